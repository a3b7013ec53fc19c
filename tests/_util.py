"""Test helpers: moving seeded inputs between torch (GPU path) and numpy (oracle)."""

from __future__ import annotations

import numpy as np
import torch

PER_LAYER = ("in_norm_w", "post_norm_w", "wq", "wk", "wv", "wo", "q_norm_w", "k_norm_w",
             "w_gate", "w_up", "w_down")


def to_np(t: torch.Tensor) -> np.ndarray:
    """bf16/fp32/int torch tensor -> numpy (bf16 widened exactly to float32)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def weights_np(W: dict) -> dict:
    out = {}
    for k, v in W.items():
        out[k] = [to_np(x) for x in v] if k in PER_LAYER else to_np(v)
    return out


def weights_to(W: dict, device) -> dict:
    out = {}
    for k, v in W.items():
        out[k] = [x.to(device) for x in v] if k in PER_LAYER else v.to(device)
    return out


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ----------------------------------------------------------------------------
# parity bookkeeping: rows whose greedy pick is a near-tie are excluded from the
# bit-exact comparison; every exclusion is recorded and summarised at the end
# of the pytest run (tests/conftest.py), and written as JSON lines to the file
# named by DFLASH_PARITY_RECORD when that variable is set.
# ----------------------------------------------------------------------------
PARITY_LOG: list = []


def record_parity(name: str, **fields) -> None:
    import json
    import os
    entry = dict(name=name, **fields)
    PARITY_LOG.append(entry)
    path = os.environ.get("DFLASH_PARITY_RECORD")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(entry) + "\n")
