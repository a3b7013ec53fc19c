"""DFlash draft proposal (inject + propose + greedy verify) for NVIDIA B200.

The compute path is the C-ABI library ``libdflash.so`` (hand-written sm_100a
CUDA); ``dflash`` is its thin Python binding and ``synth`` the seeded
synthetic-input generator used by the tests and the benchmark.
"""

from .dflash import (DFlash, DFlashError, StepGraph, Workspace, finalize_draft_keys,  # noqa: F401
                     lib, paged_slots, prepare_proposal_inputs, status_string, verify_greedy,
                     verify_workspace_bytes, version)
