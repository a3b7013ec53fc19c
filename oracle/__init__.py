"""CPU oracle for the DFlash draft-proposal step.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library package.
"""
from .dflash_oracle import *  # noqa: F401,F403
from .dflash_oracle import (OracleConfig, Proposal, ProposalInputs, QueryBlock,  # noqa: F401
                            TPSlices, Verification,
                            STORAGE_POINTS, FP16_WEIGHTS)
