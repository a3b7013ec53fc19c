"""Thin Python binding over the C ABI in include/dflash.h (libdflash.so).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Torch tensors supply device memory and streams; outputs that the
caller does not pass are allocated here with ``torch.empty``.  If the shared
library is missing this module raises — there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdflash.so")

STATUS = {
    0: "DFLASH_OK",
    -1: "DFLASH_ERR_INVALID_ARG",
    -2: "DFLASH_ERR_CUDA",
    -3: "DFLASH_ERR_WORKSPACE",
    -4: "DFLASH_ERR_UNSUPPORTED_SHAPE",
    -5: "DFLASH_ERR_DEVICE_BOUNDS",
    -6: "DFLASH_ERR_UNIMPLEMENTED",
    -7: "DFLASH_ERR_DEVICE_TIMEOUT",
    -8: "DFLASH_ERR_RANGE",
    -9: "DFLASH_ERR_EXCHANGE",
}
DEVERR_TIMEOUT, DEVERR_SLOT, DEVERR_TABLE, DEVERR_TOKEN, DEVERR_POSITION = 1, 2, 4, 8, 16
KERNEL_KINDS = 14


class DFlashError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class _Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_layers", ctypes.c_int),
                ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("intermediate", ctypes.c_int),
                ("vocab", ctypes.c_int), ("n_target_layers", ctypes.c_int),
                ("target_layer_ids", ctypes.POINTER(ctypes.c_int)),
                ("block_size", ctypes.c_int), ("mask_token_id", ctypes.c_int),
                ("page_size", ctypes.c_int), ("rms_eps", ctypes.c_float),
                ("rope_theta", ctypes.c_float), ("max_position", ctypes.c_int)]


_PP = ctypes.POINTER(ctypes.c_void_p)
# dflash_allreduce_fn: int (*)(float* data, size_t count, void* stream, void* user)
ALLREDUCE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                ctypes.c_void_p)


class _Weights(ctypes.Structure):
    _fields_ = [("fc_w", ctypes.c_void_p), ("hidden_norm_w", ctypes.c_void_p),
                ("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("final_norm_w", ctypes.c_void_p)] + [
        (n, _PP) for n in ("in_norm_w", "post_norm_w", "wq", "wk", "wv", "wo", "q_norm_w",
                           "k_norm_w", "w_gate", "w_up", "w_down")]


class _StepIO(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("n", ctypes.c_int),
                ("prev_drafts", ctypes.c_void_p), ("target_logits", ctypes.c_void_p),
                ("target_positions", ctypes.c_void_p), ("last_token_indices", ctypes.c_void_p),
                ("num_draft", ctypes.c_void_p), ("prev_sampled", ctypes.c_void_p),
                ("prev_width", ctypes.c_int), ("prev_num_draft", ctypes.c_void_p),
                ("aux", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("max_pages_per_seq", ctypes.c_int), ("k_cache", _PP), ("v_cache", _PP),
                ("num_pages", ctypes.c_int), ("out_tokens", ctypes.c_void_p),
                ("num_accepted", ctypes.c_void_p), ("positions", ctypes.c_void_p),
                ("slot_mapping", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("bonus", ctypes.c_void_p), ("draft_tokens", ctypes.c_void_p),
                ("block_tokens", ctypes.c_void_p), ("device_error", ctypes.c_void_p)]


class _TargetConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("hidden", "n_layers", "n_q_heads", "n_kv_heads",
                                            "head_dim", "intermediate", "vocab")] + \
               [("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("max_len", ctypes.c_int), ("n_capture", ctypes.c_int),
                ("capture_layers", ctypes.POINTER(ctypes.c_int))]


_TARGET_SINGLE = ("embed", "final_norm_w", "lm_head")
_TARGET_LAYER = ("in_norm_w", "post_norm_w", "wq", "wk", "wv", "wo", "q_norm_w", "k_norm_w",
                 "w_gate", "w_up", "w_down")


class _TargetWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _TARGET_SINGLE] + \
               [(n, _PP) for n in _TARGET_LAYER]


class _AttnPlan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("tcgen05", "keys_per_tile", "ring_depth",
                                            "ctas_per_sm", "chunk_keys", "max_splits",
                                            "cluster", "persistent", "transposed_pv")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdflash.so (built in-tree by ``build.py``); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "block_diffusion_speculative_propose_b200/build.py")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "dflash_create": ([ctypes.POINTER(_Config), ctypes.POINTER(_Weights), i32,
                           ctypes.POINTER(vp)], i32),
        "dflash_create_vocab_shard": ([ctypes.POINTER(_Config), ctypes.POINTER(_Weights), i32,
                                       i32, i32, ctypes.POINTER(vp)], i32),
        "dflash_destroy": ([vp], None),
        "dflash_inject_workspace_bytes": ([vp, i32], sz),
        "dflash_propose_workspace_bytes": ([vp, i32, i32], sz),
        "dflash_propose_final_rows_offset": ([vp, i32, i32], sz),
        "dflash_set_wait_limit": ([i32, ctypes.c_longlong], i32),
        "dflash_plan_gemm_info": ([i32] * 6 + [ctypes.POINTER(_GemmPlan)], i32),
        "dflash_create_tp_shard": ([ctypes.POINTER(_Config), ctypes.POINTER(_Weights), i32, i32,
                                    i32, i32, i32, ctypes.POINTER(vp)], i32),
        "dflash_propose_tp": ([vp, vp, vp, vp, i32, i32, _PP, _PP, i32, vp, vp, vp, sz, vp,
                               ALLREDUCE_FN, vp], i32),
        "dflash_aux_capture_layers": ([ctypes.POINTER(ctypes.c_int), i32, i32,
                                       ctypes.POINTER(ctypes.c_int)], i32),
        "dflash_target_create": ([ctypes.POINTER(_TargetConfig), ctypes.POINTER(_TargetWeights),
                                  i32, ctypes.POINTER(vp)], i32),
        "dflash_target_destroy": ([vp], None),
        "dflash_target_workspace_bytes": ([vp, i32], sz),
        "dflash_target_forward": ([vp, vp, i32, i32, vp, vp, vp, sz, vp], i32),
        "dflash_target_check_device_errors": ([vp, ctypes.POINTER(ctypes.c_uint)], i32),
        "dflash_selftest_wait_timeout": ([vp, vp], i32),
        "dflash_verify_workspace_bytes": ([i32, i32, i32], sz),
        "dflash_linear_workspace_bytes": ([vp, i32, i32, i32], sz),
        "dflash_attention_workspace_bytes": ([vp, i32, i32], sz),
        "dflash_paged_slots": ([vp, vp, i32, vp, i32, i32, vp, vp], i32),
        "dflash_prepare_proposal_inputs": ([vp, i32, vp, i32, vp, i32, vp, vp, i32, vp, vp,
                                            i32, i32, i32, vp, vp, vp, vp, vp, vp], i32),
        "dflash_inject_context": ([vp, vp, vp, vp, i32, _PP, _PP, i32, vp, sz, vp], i32),
        "dflash_propose": ([vp, vp, vp, vp, i32, i32, _PP, _PP, i32, vp, vp, vp, vp, sz, vp],
                           i32),
        "dflash_propose_keys": ([vp, vp, vp, vp, i32, i32, _PP, _PP, i32, vp, vp, vp, sz, vp],
                                i32),
        "dflash_finalize_draft_keys": ([vp, vp, i32, i32, i32, vp, vp, vp, vp], i32),
        "dflash_verify_greedy": ([vp, vp, i32, i32, i32, vp, vp, vp, vp, sz, vp], i32),
        "dflash_verify_greedy_noalloc": ([vp, vp, i32, i32, i32, vp, vp, vp, vp], i32),
        "dflash_spec_step_workspace_bytes": ([vp, i32, i32, i32], sz),
        "dflash_spec_step": ([vp, ctypes.POINTER(_StepIO), vp, sz, vp], i32),
        "dflash_step_graph_create": ([vp, ctypes.POINTER(_StepIO), vp, sz, ctypes.POINTER(vp)],
                                     i32),
        "dflash_step_graph_launch": ([vp, vp], i32),
        "dflash_step_graph_destroy": ([vp], None),
        "dflash_linear": ([vp, vp, vp, i32, i32, i32, vp, vp, sz, vp], i32),
        "dflash_linear_ex": ([vp, vp, vp, i32, i32, i32, vp, i32, i32, vp, sz, vp], i32),
        "dflash_block_attention": ([vp, vp, vp, vp, i32, i32, vp, vp, i32, vp, vp, sz, vp],
                                   i32),
        "dflash_plan_attention_info": ([i32] * 10 + [ctypes.POINTER(_AttnPlan)], i32),
        "dflash_check_device_errors": ([vp, ctypes.POINTER(ctypes.c_uint)], i32),
        "dflash_launch_count": ([vp], ctypes.c_ulonglong),
        "dflash_kernel_name": ([i32], ctypes.c_char_p),
        "dflash_profile_enable": ([vp, i32], i32),
        "dflash_profile_read": ([vp, i32, ctypes.POINTER(ctypes.c_int),
                                 ctypes.POINTER(ctypes.c_double)], i32),
        "dflash_profile_disable": ([vp], i32),
        "dflash_status_string": ([i32], ctypes.c_char_p),
        "dflash_version": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _check(status: int, where: str) -> None:
    if status != 0:
        raise DFlashError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _want(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr_array(ts: Sequence[torch.Tensor]):
    arr = (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])
    return ctypes.cast(arr, _PP), arr


class Workspace:
    """Device scratch owned by the caller (a uint8 tensor), grown on demand."""

    def __init__(self, device):
        self.device = torch.device(device)
        self.buf = torch.empty(0, dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


class DFlash:
    """A library handle: packed draft weights + RoPE table on one device.

    ``cfg`` uses the field names of ``dflash_config``; ``weights`` the names of
    ``dflash_weights`` (bf16 CUDA tensors; per-layer entries are lists).  The
    handle keeps references to every tensor whose pointer the library keeps.
    ``vocab_shard=(start, count)`` builds one rank's shard of the tensor-parallel
    LM head (dflash_create_vocab_shard): ``weights["lm_head"]`` is then that
    shard's [count, H] rows, and the handle proposes through propose_keys."""

    def __init__(self, cfg: Dict, weights: Dict, device: int = 0, max_position: int = 0,
                 vocab_shard: Optional[Sequence[int]] = None, tp: Optional[Sequence[int]] = None):
        L = lib()
        self.cfg = dict(cfg)
        self.device = torch.device("cuda", device)
        n_layers = cfg["n_layers"]
        self._keep: List = []
        tl = cfg.get("target_layer_ids")
        tl_arr = None
        if tl is not None:
            tl_arr = (ctypes.c_int * len(tl))(*tl)
            self._keep.append(tl_arr)
        maxpos = max_position or cfg.get("max_position", 65536)
        self.max_position = maxpos
        c = _Config(cfg["hidden"], n_layers, cfg["n_q_heads"], cfg["n_kv_heads"],
                    cfg["head_dim"], cfg["intermediate"], cfg["vocab"],
                    cfg["n_target_layers"],
                    ctypes.cast(tl_arr, ctypes.POINTER(ctypes.c_int)) if tl_arr else None,
                    cfg["block_size"], cfg["mask_token_id"], cfg.get("page_size", 16),
                    cfg.get("rms_eps", 1e-6), cfg.get("rope_theta", 1e6), maxpos)
        w = _Weights()
        for k in ("fc_w", "hidden_norm_w", "embed", "lm_head", "final_norm_w"):
            t = weights[k]
            _want(t, torch.bfloat16, k)
            self._keep.append(t)
            setattr(w, k, _ptr(t))
        for k in ("in_norm_w", "post_norm_w", "wq", "wk", "wv", "wo", "q_norm_w", "k_norm_w",
                  "w_gate", "w_up", "w_down"):
            ts = list(weights[k])
            if len(ts) != n_layers:
                raise ValueError(f"{k}: expected {n_layers} layers")
            for t in ts:
                _want(t, torch.bfloat16, k)
            self._keep.extend(ts)
            pp, arr = _ptr_array(ts)
            self._keep.append(arr)
            setattr(w, k, pp)
        h = ctypes.c_void_p()
        self.tp = (0, 1) if tp is None else (int(tp[0]), int(tp[1]))
        if tp is not None:
            # one tensor-parallel rank: `weights` is the whole model (every rank
            # passes the same); the library copies out this rank's slices
            self.vocab_shard = ((0, cfg["vocab"]) if vocab_shard is None else
                                (int(vocab_shard[0]), int(vocab_shard[1])))
            _check(L.dflash_create_tp_shard(ctypes.byref(c), ctypes.byref(w), device,
                                            self.tp[0], self.tp[1], self.vocab_shard[0],
                                            self.vocab_shard[1], ctypes.byref(h)),
                   "dflash_create_tp_shard")
        elif vocab_shard is None:
            self.vocab_shard = (0, cfg["vocab"])
            _check(L.dflash_create(ctypes.byref(c), ctypes.byref(w), device, ctypes.byref(h)),
                   "dflash_create")
        else:
            self.vocab_shard = (int(vocab_shard[0]), int(vocab_shard[1]))
            _check(L.dflash_create_vocab_shard(ctypes.byref(c), ctypes.byref(w), device,
                                               self.vocab_shard[0], self.vocab_shard[1],
                                               ctypes.byref(h)), "dflash_create_vocab_shard")
        self.h = h
        self.ws = Workspace(self.device)

    def close(self) -> None:
        if getattr(self, "h", None):
            torch.cuda.synchronize(self.device)
            lib().dflash_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---------------------------------------------------------------- sizes
    def inject_workspace_bytes(self, n: int) -> int:
        return lib().dflash_inject_workspace_bytes(self.h, n)

    def propose_workspace_bytes(self, B: int, max_pages_per_seq: int) -> int:
        return lib().dflash_propose_workspace_bytes(self.h, B, max_pages_per_seq)

    def propose_final_rows(self, workspace: torch.Tensor, B: int,
                           max_pages_per_seq: int) -> torch.Tensor:
        """View of the [B*K, hidden] fp16 rows that the last proposal with this
        workspace handed to the LM head (diagnostics)."""
        off = int(lib().dflash_propose_final_rows_offset(self.h, B, max_pages_per_seq))
        K, H = self.cfg["block_size"] - 1, self.cfg["hidden"]
        n = B * K * H * 2
        if off < 0 or off + n > workspace.numel():
            raise DFlashError(-1, "dflash_propose_final_rows_offset")
        return workspace[off:off + n].view(torch.float16).view(B * K, H)

    # ---------------------------------------------------------------- calls
    def inject_context(self, aux, positions, slot_mapping, k_cache, v_cache,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> None:
        n = int(aux.shape[0])
        _want(aux, torch.bfloat16, "aux")
        _want(positions, torch.int64, "positions")
        _want(slot_mapping, torch.int64, "slot_mapping")
        need = self.inject_workspace_bytes(n) if n else 0
        ws = workspace if workspace is not None else self.ws.get(need)
        kp, ka = _ptr_array(k_cache)
        vp, va = _ptr_array(v_cache)
        _check(lib().dflash_inject_context(self.h, _ptr(aux), _ptr(positions),
                                           _ptr(slot_mapping), n, kp, vp,
                                           int(k_cache[0].shape[0]), _ptr(ws), ws.numel(),
                                           _stream(stream)),
               "dflash_inject_context")

    def propose(self, bonus_tokens, seq_lens, block_table, k_cache, v_cache,
                draft_tokens=None, block_tokens=None, logits_out=None,
                workspace: Optional[torch.Tensor] = None, stream=None):
        B = int(bonus_tokens.shape[0])
        bs = self.cfg["block_size"]
        _want(bonus_tokens, torch.int32, "bonus_tokens")
        _want(seq_lens, torch.int32, "seq_lens")
        _want(block_table, torch.int32, "block_table")
        W = int(block_table.shape[1])
        if draft_tokens is None:
            draft_tokens = torch.empty(B, bs - 1, dtype=torch.int32, device=self.device)
        need = self.propose_workspace_bytes(B, W) if B else 0
        ws = workspace if workspace is not None else self.ws.get(need)
        kp, ka = _ptr_array(k_cache)
        vp, va = _ptr_array(v_cache)
        _check(lib().dflash_propose(self.h, _ptr(bonus_tokens), _ptr(seq_lens),
                                    _ptr(block_table), B, W, kp, vp, int(k_cache[0].shape[0]),
                                    _ptr(draft_tokens), _ptr(block_tokens), _ptr(logits_out),
                                    _ptr(ws), ws.numel(), _stream(stream)),
               "dflash_propose")
        return draft_tokens

    def spec_step_workspace_bytes(self, B: int, n: int, max_pages_per_seq: int) -> int:
        return lib().dflash_spec_step_workspace_bytes(self.h, B, n, max_pages_per_seq)

    def _step_io(self, prev_drafts, target_logits, target_positions, last_token_indices,
                 num_draft, aux, block_table, k_cache, v_cache, prev_sampled, prev_num_draft,
                 out, device_error):
        """Marshal the buffers of one speculative step into dflash_step_io;
        returns (io, outputs, objects to keep alive)."""
        B, n = int(last_token_indices.shape[0]), int(target_positions.shape[0])
        bs = self.cfg["block_size"]
        _want(prev_drafts, torch.int32, "prev_drafts")
        _want(target_logits, torch.float32, "target_logits")
        _want(target_positions, torch.int64, "target_positions")
        _want(last_token_indices, torch.int32, "last_token_indices")
        _want(num_draft, torch.int32, "num_draft")
        _want(aux, torch.bfloat16, "aux")
        _want(block_table, torch.int32, "block_table")
        if prev_sampled is not None:
            _want(prev_sampled, torch.int32, "prev_sampled")
        if prev_num_draft is not None:
            _want(prev_num_draft, torch.int32, "prev_num_draft")
        dev = self.device
        o = dict(out or {})
        shapes = {"out_tokens": ((B, bs), torch.int32), "num_accepted": ((B,), torch.int32),
                  "positions": ((n,), torch.int64), "slot_mapping": ((n,), torch.int64),
                  "seq_lens": ((B,), torch.int32), "bonus": ((B,), torch.int32),
                  "draft_tokens": ((B, bs - 1), torch.int32),
                  "block_tokens": ((B, bs), torch.int32)}
        for k, (shape, dt) in shapes.items():
            if k not in o:
                o[k] = torch.empty(shape, dtype=dt, device=dev)
            _want(o[k], dt, k)
        kp, ka = _ptr_array(k_cache)
        vp, va = _ptr_array(v_cache)
        io = _StepIO(B, n, _ptr(prev_drafts), _ptr(target_logits), _ptr(target_positions),
                     _ptr(last_token_indices), _ptr(num_draft), _ptr(prev_sampled),
                     int(prev_sampled.shape[1]) if prev_sampled is not None else 0,
                     _ptr(prev_num_draft), _ptr(aux), _ptr(block_table),
                     int(block_table.shape[1]), kp, vp, int(k_cache[0].shape[0]),
                     _ptr(o["out_tokens"]), _ptr(o["num_accepted"]), _ptr(o["positions"]),
                     _ptr(o["slot_mapping"]), _ptr(o["seq_lens"]), _ptr(o["bonus"]),
                     _ptr(o["draft_tokens"]), _ptr(o["block_tokens"]), _ptr(device_error))
        keep = [prev_drafts, target_logits, target_positions, last_token_indices, num_draft,
                aux, block_table, list(k_cache), list(v_cache), prev_sampled, prev_num_draft,
                device_error, ka, va]
        return io, o, keep

    def spec_step(self, prev_drafts, target_logits, target_positions, last_token_indices,
                  num_draft, aux, block_table, k_cache, v_cache, prev_sampled=None,
                  prev_num_draft=None, out=None, device_error=None, workspace=None,
                  stream=None) -> Dict[str, torch.Tensor]:
        """One whole speculative step (dflash_spec_step): verify -> prepare ->
        inject -> propose on the device.  Returns the outputs by name
        (out_tokens, num_accepted, positions, slot_mapping, seq_lens, bonus,
        draft_tokens, block_tokens); tensors given in ``out`` are written in place."""
        io, o, keep = self._step_io(prev_drafts, target_logits, target_positions,
                                    last_token_indices, num_draft, aux, block_table, k_cache,
                                    v_cache, prev_sampled, prev_num_draft, out, device_error)
        need = self.spec_step_workspace_bytes(io.B, io.n, io.max_pages_per_seq) if io.B else 0
        ws = workspace if workspace is not None else self.ws.get(need)
        _check(lib().dflash_spec_step(self.h, ctypes.byref(io), _ptr(ws), ws.numel(),
                                      _stream(stream)), "dflash_spec_step")
        return o

    def step_graph(self, prev_drafts, target_logits, target_positions, last_token_indices,
                   num_draft, aux, block_table, k_cache, v_cache, prev_sampled=None,
                   prev_num_draft=None, out=None, device_error=None,
                   workspace=None) -> "StepGraph":
        """The same step captured once into a library-owned CUDA graph
        (dflash_step_graph_create) over these buffers; see StepGraph."""
        io, o, keep = self._step_io(prev_drafts, target_logits, target_positions,
                                    last_token_indices, num_draft, aux, block_table, k_cache,
                                    v_cache, prev_sampled, prev_num_draft, out, device_error)
        need = self.spec_step_workspace_bytes(io.B, io.n, io.max_pages_per_seq) if io.B else 0
        ws = workspace if workspace is not None else torch.empty(
            max(need, 256), dtype=torch.uint8, device=self.device)
        g = ctypes.c_void_p()
        _check(lib().dflash_step_graph_create(self.h, ctypes.byref(io), _ptr(ws), ws.numel(),
                                              ctypes.byref(g)), "dflash_step_graph_create")
        return StepGraph(self, g, o, keep + [ws, io])

    def propose_keys(self, bonus_tokens, seq_lens, block_table, k_cache, v_cache,
                     draft_keys=None, logits_out=None, workspace: Optional[torch.Tensor] = None,
                     stream=None):
        """dflash_propose_keys: this handle's vocabulary shard's greedy-pick keys,
        [B, K] int64, ready for an all-reduce MAX across the shards."""
        B = int(bonus_tokens.shape[0])
        bs = self.cfg["block_size"]
        _want(bonus_tokens, torch.int32, "bonus_tokens")
        _want(seq_lens, torch.int32, "seq_lens")
        _want(block_table, torch.int32, "block_table")
        W = int(block_table.shape[1])
        if draft_keys is None:
            draft_keys = torch.empty(B, bs - 1, dtype=torch.int64, device=self.device)
        _want(draft_keys, torch.int64, "draft_keys")
        need = self.propose_workspace_bytes(B, W) if B else 0
        ws = workspace if workspace is not None else self.ws.get(need)
        kp, ka = _ptr_array(k_cache)
        vp, va = _ptr_array(v_cache)
        _check(lib().dflash_propose_keys(self.h, _ptr(bonus_tokens), _ptr(seq_lens),
                                         _ptr(block_table), B, W, kp, vp,
                                         int(k_cache[0].shape[0]), _ptr(draft_keys),
                                         _ptr(logits_out), _ptr(ws), ws.numel(),
                                         _stream(stream)), "dflash_propose_keys")
        return draft_keys

    def propose_tp(self, bonus_tokens, seq_lens, block_table, k_cache, v_cache, exchange,
                   draft_keys=None, logits_out=None, workspace: Optional[torch.Tensor] = None,
                   stream=None):
        """dflash_propose_tp on a tensor-parallel shard: `exchange(data_ptr,
        count, stream_ptr) -> int` must sum the `count` fp32 values at the
        device pointer over every rank, in place, ordered on that stream (0 on
        success).  Returns this rank's vocabulary shard's keys [B, K] int64."""
        B = int(bonus_tokens.shape[0])
        bs = self.cfg["block_size"]
        _want(bonus_tokens, torch.int32, "bonus_tokens")
        _want(seq_lens, torch.int32, "seq_lens")
        _want(block_table, torch.int32, "block_table")
        W = int(block_table.shape[1])
        if draft_keys is None:
            draft_keys = torch.empty(B, bs - 1, dtype=torch.int64, device=self.device)
        need = self.propose_workspace_bytes(B, W) if B else 0
        ws = workspace if workspace is not None else self.ws.get(need)
        kp, ka = _ptr_array(k_cache)
        vp, va = _ptr_array(v_cache)

        def hook(data, count, st, user):
            try:
                return int(exchange(int(data), int(count), st))
            except Exception:
                return 1
        cb = ALLREDUCE_FN(hook)
        _check(lib().dflash_propose_tp(self.h, _ptr(bonus_tokens), _ptr(seq_lens),
                                       _ptr(block_table), B, W, kp, vp,
                                       int(k_cache[0].shape[0]), _ptr(draft_keys),
                                       _ptr(logits_out), _ptr(ws), ws.numel(), _stream(stream),
                                       cb, None), "dflash_propose_tp")
        return draft_keys

    def linear(self, A, W, out=None, block_n: int = 0, splits: int = 0, workspace=None,
               stream=None):
        M, K = A.shape
        N = W.shape[0]
        _want(A, torch.bfloat16, "A")
        _want(W, torch.bfloat16, "W")
        if out is None:
            out = torch.empty(M, N, dtype=torch.float32, device=self.device)
        need = lib().dflash_linear_workspace_bytes(self.h, M, N, K) if M else 0
        if splits > 1:
            bn = block_n or 256
            tiles = -(-M // 128) * -(-N // bn)
            need = max(need, 2 * (tiles * splits + 1) * min(M, 128) * bn * 4)
        ws = workspace if workspace is not None else self.ws.get(need)
        _check(lib().dflash_linear_ex(self.h, _ptr(A), _ptr(W), M, N, K, _ptr(out), block_n,
                                      splits, _ptr(ws), ws.numel(), _stream(stream)),
               "dflash_linear")
        return out

    def block_attention(self, q, seq_lens, block_table, k_cache, v_cache, o=None,
                        workspace=None, stream=None):
        B = int(seq_lens.shape[0])
        W = int(block_table.shape[1])
        if o is None:
            o = torch.empty(q.shape[0], q.shape[1] * q.shape[2], dtype=torch.float16,
                            device=self.device)
        need = lib().dflash_attention_workspace_bytes(self.h, B, W) if B else 0
        ws = workspace if workspace is not None else self.ws.get(need)
        _check(lib().dflash_block_attention(self.h, _ptr(q), _ptr(seq_lens), _ptr(block_table),
                                            B, W, _ptr(k_cache), _ptr(v_cache),
                                            int(k_cache.shape[0]), _ptr(o), _ptr(ws),
                                            ws.numel(), _stream(stream)),
               "dflash_block_attention")
        return o

    # ---------------------------------------------------------- diagnostics
    def launch_count(self) -> int:
        return int(lib().dflash_launch_count(self.h))

    def profile_enable(self, max_launches: int) -> None:
        _check(lib().dflash_profile_enable(self.h, max_launches), "dflash_profile_enable")

    def profile_disable(self) -> None:
        _check(lib().dflash_profile_disable(self.h), "dflash_profile_disable")

    def profile_read(self) -> Dict[str, tuple]:
        """{kernel family: (launches, total ms)} since the last read."""
        n = KERNEL_KINDS
        cnt = (ctypes.c_int * n)()
        tot = (ctypes.c_double * n)()
        _check(lib().dflash_profile_read(self.h, n, cnt, tot), "dflash_profile_read")
        return {lib().dflash_kernel_name(k).decode(): (cnt[k], tot[k])
                for k in range(n) if cnt[k]}

    def check_device_errors(self) -> int:
        bits = ctypes.c_uint(0)
        lib().dflash_check_device_errors(self.h, ctypes.byref(bits))
        return int(bits.value)

    def check_device_status(self):
        """(status, bits) of dflash_check_device_errors."""
        bits = ctypes.c_uint(0)
        s = int(lib().dflash_check_device_errors(self.h, ctypes.byref(bits)))
        return s, int(bits.value)

    def selftest_wait_timeout(self, stream=None) -> None:
        """Enqueue a kernel whose one bounded wait runs out (diagnostics)."""
        _check(lib().dflash_selftest_wait_timeout(self.h, _stream(stream)),
               "dflash_selftest_wait_timeout")


def aux_capture_layers(target_layer_ids: Sequence[int], target_n_layers: int) -> List[int]:
    """Capture layers (pre-layer states) for a draft checkpoint's
    target_layer_ids (states after layer i): each id plus one."""
    n = len(target_layer_ids)
    ids = (ctypes.c_int * max(n, 1))(*target_layer_ids)
    out = (ctypes.c_int * max(n, 1))()
    _check(lib().dflash_aux_capture_layers(ids, n, int(target_n_layers), out),
           "dflash_aux_capture_layers")
    return [int(out[i]) for i in range(n)]


class TargetModel:
    """The library's small causal target model (dflash_target_*): fp32
    weights (CUDA tensors, names of ``dflash_target_weights``), one sequence.
    ``forward(tokens, start_pos)`` returns (logits [n, V] fp32, aux
    [n, n_capture * H] bf16)."""

    def __init__(self, cfg: Dict, weights: Dict, capture_layers: Sequence[int],
                 max_len: int, device: int = 0):
        L = lib()
        self.cfg = dict(cfg)
        self.device = torch.device("cuda", device)
        self.n_capture = len(capture_layers)
        self._keep: List = []
        cap = (ctypes.c_int * max(self.n_capture, 1))(*capture_layers)
        self._keep.append(cap)
        c = _TargetConfig(cfg["hidden"], cfg["n_layers"], cfg["n_q_heads"], cfg["n_kv_heads"],
                          cfg["head_dim"], cfg["intermediate"], cfg["vocab"],
                          cfg.get("rms_eps", 1e-6), cfg.get("rope_theta", 1e6), int(max_len),
                          self.n_capture, ctypes.cast(cap, ctypes.POINTER(ctypes.c_int)))
        w = _TargetWeights()
        for k in _TARGET_SINGLE:
            t = weights[k]
            _want(t, torch.float32, k)
            self._keep.append(t)
            setattr(w, k, _ptr(t))
        for k in _TARGET_LAYER:
            ts = list(weights[k])
            if len(ts) != cfg["n_layers"]:
                raise ValueError(f"{k}: expected {cfg['n_layers']} layers")
            for t in ts:
                _want(t, torch.float32, k)
            self._keep.extend(ts)
            pp, arr = _ptr_array(ts)
            self._keep.append(arr)
            setattr(w, k, pp)
        h = ctypes.c_void_p()
        _check(L.dflash_target_create(ctypes.byref(c), ctypes.byref(w), device, ctypes.byref(h)),
               "dflash_target_create")
        self.h = h
        self.ws = Workspace(self.device)

    def close(self) -> None:
        if getattr(self, "h", None):
            torch.cuda.synchronize(self.device)
            lib().dflash_target_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, tokens: torch.Tensor, start_pos: int, logits=None, aux=None, stream=None):
        _want(tokens, torch.int32, "tokens")
        n = int(tokens.numel())
        H, V = self.cfg["hidden"], self.cfg["vocab"]
        if logits is None:
            logits = torch.empty(n, V, dtype=torch.float32, device=self.device)
        if aux is None and self.n_capture:
            aux = torch.empty(n, self.n_capture * H, dtype=torch.bfloat16, device=self.device)
        ws = self.ws.get(lib().dflash_target_workspace_bytes(self.h, max(n, 1)))
        _check(lib().dflash_target_forward(self.h, _ptr(tokens), n, int(start_pos), _ptr(logits),
                                           _ptr(aux), _ptr(ws), ws.numel(), _stream(stream)),
               "dflash_target_forward")
        return logits, aux

    def check_device_errors(self) -> int:
        bits = ctypes.c_uint(0)
        lib().dflash_target_check_device_errors(self.h, ctypes.byref(bits))
        return int(bits.value)


def set_wait_limit(device: int, cycles: int) -> None:
    """Cycles after which every bounded wait of the library's kernels on
    `device` gives up (diagnostics; default 4e9)."""
    _check(lib().dflash_set_wait_limit(int(device), int(cycles)), "dflash_set_wait_limit")


class StepGraph:
    """A speculative step captured into a CUDA graph owned by the library.
    ``launch()`` replays it on a stream; ``out`` holds its output tensors.  The
    graph keeps the pointers of the buffers it was built on (held here): write
    new inputs into those tensors between launches."""

    def __init__(self, owner: DFlash, g, out: Dict[str, torch.Tensor], keep: List):
        self._owner = owner     # the handle must outlive the graph
        self.g = g
        self.out = out
        self._keep = keep

    def launch(self, stream=None) -> None:
        _check(lib().dflash_step_graph_launch(self.g, _stream(stream)),
               "dflash_step_graph_launch")

    def close(self) -> None:
        if getattr(self, "g", None):
            torch.cuda.synchronize(self._owner.device)
            lib().dflash_step_graph_destroy(self.g)
            self.g = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def finalize_draft_keys(draft_keys, bonus_tokens, block_size: int, vocab: int,
                        draft_tokens=None, block_tokens=None, device_error=None, stream=None):
    """dflash_finalize_draft_keys: drafts [B, K] (and block tokens [B, bs])
    from the keys exchanged across vocabulary shards."""
    B = int(bonus_tokens.shape[0])
    _want(draft_keys, torch.int64, "draft_keys")
    _want(bonus_tokens, torch.int32, "bonus_tokens")
    dev = draft_keys.device
    if draft_tokens is None:
        draft_tokens = torch.empty(B, block_size - 1, dtype=torch.int32, device=dev)
    if block_tokens is None:
        block_tokens = torch.empty(B, block_size, dtype=torch.int32, device=dev)
    _check(lib().dflash_finalize_draft_keys(_ptr(draft_keys), _ptr(bonus_tokens), B, block_size,
                                            vocab, _ptr(draft_tokens), _ptr(block_tokens),
                                            _ptr(device_error), _stream(stream)),
           "dflash_finalize_draft_keys")
    return draft_tokens, block_tokens


def attention_plan(B: int, n_kv_heads: int, max_pages_per_seq: int, block_size: int,
                   q_per_kv: int, head_dim: int = 128, page_size: int = 16, num_sms: int = 148,
                   forced_ring: int = 0, cluster: bool = False,
                   persistent: bool = False, tile32: bool = False) -> Dict[str, int]:
    """dflash_plan_attention_info: the attention launch plan for this geometry
    (host only)."""
    out = _AttnPlan()
    flags = (1 if cluster else 0) | (2 if persistent else 0) | (4 if tile32 else 0)
    _check(lib().dflash_plan_attention_info(B, n_kv_heads, max_pages_per_seq, page_size,
                                            block_size, q_per_kv, head_dim, num_sms,
                                            forced_ring, flags, ctypes.byref(out)),
           "dflash_plan_attention_info")
    return {n: getattr(out, n) for n, _ in _AttnPlan._fields_}


class _GemmPlan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("pair", "tile_m", "tile_n", "k_splits", "stream_k",
                                            "staged", "tiles", "grid")]


def gemm_plan(M: int, N: int, K: int, group: int = 32, num_sms: int = 148,
              pair_split_cap: int = 37) -> Dict[str, int]:
    """dflash_plan_gemm_info: the GEMM launch plan for this shape (host only)."""
    out = _GemmPlan()
    _check(lib().dflash_plan_gemm_info(M, N, K, group, num_sms, pair_split_cap,
                                       ctypes.byref(out)), "dflash_plan_gemm_info")
    return {n: getattr(out, n) for n, _ in _GemmPlan._fields_}


def verify_workspace_bytes(B: int, K: int, V: int) -> int:
    return lib().dflash_verify_workspace_bytes(B, K, V)


def verify_greedy(drafts, target_logits, out_tokens=None, num_accepted=None, bonus=None,
                  workspace=None, stream=None):
    """Greedy acceptance (dflash_verify_greedy); returns (out_tokens, n, bonus)."""
    B, K1, V = target_logits.shape
    K = K1 - 1
    dev = target_logits.device
    _want(drafts, torch.int32, "drafts")
    _want(target_logits, torch.float32, "target_logits")
    if out_tokens is None:
        out_tokens = torch.empty(B, K + 1, dtype=torch.int32, device=dev)
    if num_accepted is None:
        num_accepted = torch.empty(B, dtype=torch.int32, device=dev)
    if bonus is None:
        bonus = torch.empty(B, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(verify_workspace_bytes(B, K, V), 256), dtype=torch.uint8,
                                device=dev)
    _check(lib().dflash_verify_greedy(_ptr(drafts), _ptr(target_logits), B, K, V,
                                      _ptr(out_tokens), _ptr(num_accepted), _ptr(bonus),
                                      _ptr(workspace), workspace.numel(), _stream(stream)),
           "dflash_verify_greedy")
    return out_tokens, num_accepted, bonus


def verify_greedy_noalloc(drafts, target_logits, out_tokens=None, num_accepted=None,
                          bonus=None, stream=None):
    """Greedy acceptance without a workspace (dflash_verify_greedy_noalloc), for
    callers that cannot allocate device scratch; returns (out_tokens, n, bonus).
    The library's fixed scratch is shared by all calls: keep calls on one stream."""
    B, K1, V = target_logits.shape
    K = K1 - 1
    dev = target_logits.device
    _want(drafts, torch.int32, "drafts")
    _want(target_logits, torch.float32, "target_logits")
    if out_tokens is None:
        out_tokens = torch.empty(B, K + 1, dtype=torch.int32, device=dev)
    if num_accepted is None:
        num_accepted = torch.empty(B, dtype=torch.int32, device=dev)
    if bonus is None:
        bonus = torch.empty(B, dtype=torch.int32, device=dev)
    _check(lib().dflash_verify_greedy_noalloc(_ptr(drafts), _ptr(target_logits), B, K, V,
                                              _ptr(out_tokens), _ptr(num_accepted), _ptr(bonus),
                                              _stream(stream)),
           "dflash_verify_greedy_noalloc")
    return out_tokens, num_accepted, bonus


def paged_slots(positions, req_ids, block_table, page_size: int = 16, slots=None,
                stream=None):
    """_paged_slots on the device (dflash_paged_slots)."""
    n = int(positions.shape[0])
    _want(positions, torch.int64, "positions")
    _want(req_ids, torch.int64, "req_ids")
    _want(block_table, torch.int32, "block_table")
    if slots is None:
        slots = torch.empty(n, dtype=torch.int64, device=positions.device)
    _check(lib().dflash_paged_slots(_ptr(positions), _ptr(req_ids), n, _ptr(block_table),
                                    int(block_table.shape[1]), page_size, _ptr(slots),
                                    _stream(stream)), "dflash_paged_slots")
    return slots


def prepare_proposal_inputs(target_positions, last_token_indices, cur_sampled, cur_num_draft,
                            block_table, page_size: int, vocab: int, prev_sampled=None,
                            prev_num_draft=None, device_error=None, stream=None):
    """Proposal inputs with the async rejection correction on the device
    (dflash_prepare_proposal_inputs).  Returns (positions, slot_mapping,
    seq_lens, bonus) ready for DFlash.inject_context / DFlash.propose."""
    n, B = int(target_positions.shape[0]), int(last_token_indices.shape[0])
    _want(target_positions, torch.int64, "target_positions")
    _want(last_token_indices, torch.int32, "last_token_indices")
    _want(cur_sampled, torch.int32, "cur_sampled")
    _want(cur_num_draft, torch.int32, "cur_num_draft")
    _want(block_table, torch.int32, "block_table")
    if prev_sampled is not None:
        _want(prev_sampled, torch.int32, "prev_sampled")
        _want(prev_num_draft, torch.int32, "prev_num_draft")
    dev = target_positions.device
    positions = torch.empty(n, dtype=torch.int64, device=dev)
    slots = torch.empty(n, dtype=torch.int64, device=dev)
    seq_lens = torch.empty(B, dtype=torch.int32, device=dev)
    bonus = torch.empty(B, dtype=torch.int32, device=dev)
    pw = int(prev_sampled.shape[1]) if prev_sampled is not None else 0
    _check(lib().dflash_prepare_proposal_inputs(
        _ptr(target_positions), n, _ptr(last_token_indices), B, _ptr(cur_sampled),
        int(cur_sampled.shape[1]), _ptr(cur_num_draft), _ptr(prev_sampled), pw,
        _ptr(prev_num_draft), _ptr(block_table), int(block_table.shape[1]), page_size, vocab,
        _ptr(positions), _ptr(slots), _ptr(seq_lens), _ptr(bonus), _ptr(device_error),
        _stream(stream)), "dflash_prepare_proposal_inputs")
    return positions, slots, seq_lens, bonus


def status_string(s: int) -> str:
    return lib().dflash_status_string(s).decode()


def version() -> str:
    return lib().dflash_version().decode()
