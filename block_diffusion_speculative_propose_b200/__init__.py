"""DFlash draft proposal (inject + propose + greedy verify) for NVIDIA B200.

The compute path is the C-ABI library ``libdflash.so`` (hand-written sm_100a
CUDA); ``dflash`` is its thin Python binding and ``synth`` the seeded
synthetic-input generator used by the tests and the benchmark.
"""

from .dflash import (DFlash, DFlashError, StepGraph, TargetModel, Workspace,  # noqa: F401
                     aux_capture_layers, finalize_draft_keys, lib, paged_slots,
                     prepare_proposal_inputs, set_wait_limit, status_string, verify_greedy,
                     verify_workspace_bytes, version)
