"""GPU parity of the library's kernel families, called through the C ABI.

  * dflash_linear(_ex)        the tcgen05 GEMM, every tile width and split-K,
                              against a float64 torch matmul of the same bf16 inputs
  * dflash_block_attention    against the oracle's non-causal paged attention
  * dflash_inject_context     against the oracle's injection (bf16 storage mode)
  * dflash_verify_greedy      bit-exact against the oracle
  * dflash_paged_slots        bit-exact against the oracle
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from block_diffusion_speculative_propose_b200 import DFlash, paged_slots, synth, verify_greedy
from tests._util import rel_l2, to_np, weights_np, weights_to

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.model_config("tiny")
    Wt = synth.make_weights(cfg, seed=0)
    h = DFlash(cfg, weights_to(Wt, DEV), max_position=4096)
    yield cfg, Wt, h
    h.close()


# ----------------------------------------------------------------------------
# GEMM
# ----------------------------------------------------------------------------
GEMM_CASES = [
    # (M, N, K, block_n, splits)   0 = automatic plan
    (1, 256, 64, 0, 0),
    (16, 4096, 4096, 0, 0),
    (15, 4096, 1024, 32, 1),
    (15, 4096, 1024, 64, 1),
    (15, 4096, 1024, 128, 1),
    (15, 4096, 1024, 256, 1),
    (16, 1024, 4096, 128, 4),
    (16, 1024, 4096, 32, 3),
    # staged epilogue (M <= 32): boundary rows, ragged N, many pieces per tile
    (32, 2048, 2048, 0, 0),
    (33, 2048, 2048, 0, 0),
    (7, 1056, 640, 0, 0),
    (17, 4096, 2048, 64, 5),
    (1, 4096, 4096, 0, 0),
    (129, 96, 192, 32, 1),
    (129, 96, 192, 32, 3),
    (300, 1536, 512, 0, 0),
    (512, 4096, 4096, 256, 1),
    (1000, 2080, 640, 0, 0),
    (2048, 1024, 1024, 256, 1),
    # whole 256-wide tiles over several M tiles: CTA pairs (256 x 256 tiles),
    # each cluster walking several tiles; ragged M and N; a pair whose second
    # half lies wholly past M (300 rows)
    (1024, 4096, 4096, 0, 0),
    (2048, 6144, 1024, 0, 0),
    (1000, 8224, 704, 0, 0),
    (300, 6400, 256, 0, 0),
    # 256 x 128 pair tiles (too few 256-wide ones to fill the SMs): 512 rows
    # against a 4096-wide output, and ragged M and N in place of a stream-K plan
    (512, 4096, 1024, 0, 0),
    (500, 4128, 704, 0, 0),
    # few wide pair tiles with a long K: K split over two pairs (clusters of
    # four, the second pair's partial reduced through distributed shared memory)
    (512, 4096, 6144, 0, 0),
    (500, 4128, 6144, 0, 0),
]


@pytest.mark.parametrize("M,N,K,bn,splits", GEMM_CASES)
def test_linear_matches_float64_matmul(tiny, M, N, K, bn, splits):
    h = tiny[2]
    g = torch.Generator().manual_seed(M * 7919 + N * 31 + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16)
    ref = A.double() @ W.double().T
    out = h.linear(A.to(DEV), W.to(DEV), block_n=bn, splits=splits)
    torch.cuda.synchronize()
    got = out.cpu().double()
    err = (got - ref).abs().max().item()
    scale = ref.abs().max().item()
    assert err <= 2e-5 * scale + 1e-6, (err, scale)
    assert h.check_device_errors() == 0


def test_linear_pair_and_single_sm_agree(monkeypatch, tiny):
    """The same many-row product through CTA pairs (default) and through the
    one-SM kernel (DFLASH_GEMM_PAIR=0 when the handle is created): both within
    the float64 bound, and within a few fp32 ulps of each other."""
    monkeypatch.setenv("DFLASH_GEMM_PAIR", "0")
    cfg = tiny[0]
    single = DFlash(cfg, weights_to(tiny[1], DEV), max_position=256)
    try:
        g = torch.Generator().manual_seed(11)
        A = torch.randn(700, 1024, generator=g).to(torch.bfloat16)
        W = (0.05 * torch.randn(5024, 1024, generator=g)).to(torch.bfloat16)
        ref = A.double() @ W.double().T
        a = tiny[2].linear(A.to(DEV), W.to(DEV)).cpu().double()
        b = single.linear(A.to(DEV), W.to(DEV)).cpu().double()
        scale = ref.abs().max().item()
        for got in (a, b):
            assert (got - ref).abs().max().item() <= 2e-5 * scale + 1e-6
        assert (a - b).abs().max().item() <= 1e-6 * scale
        assert tiny[2].check_device_errors() == 0 and single.check_device_errors() == 0
    finally:
        single.close()


def test_linear_pair_split_k_matches_unsplit(monkeypatch, tiny):
    """512 rows against a 4096-wide output with K = 6144: the split-K pair plan
    (default) and the narrow pair tiles (DFLASH_GEMM_SPLIT=0) both within the
    float64 bound, and the split plan deterministic.  (The two accumulate the
    6144 products in different orders and MMA shapes; the tensor cores' fp32
    accumulation is not exactly rounded, so they are compared with float64,
    not with each other.)"""
    monkeypatch.setenv("DFLASH_GEMM_SPLIT", "0")
    unsplit = DFlash(tiny[0], weights_to(tiny[1], DEV), max_position=256)
    try:
        g = torch.Generator().manual_seed(12)
        A = torch.randn(512, 6144, generator=g).to(torch.bfloat16)
        W = (0.05 * torch.randn(4096, 6144, generator=g)).to(torch.bfloat16)
        ref = A.double() @ W.double().T
        a = tiny[2].linear(A.to(DEV), W.to(DEV)).cpu().double()
        a2 = tiny[2].linear(A.to(DEV), W.to(DEV)).cpu().double()
        b = unsplit.linear(A.to(DEV), W.to(DEV)).cpu().double()
        scale = ref.abs().max().item()
        for got in (a, b):
            assert (got - ref).abs().max().item() <= 2e-5 * scale + 1e-6
        assert torch.equal(a, a2)
        assert tiny[2].check_device_errors() == 0 and unsplit.check_device_errors() == 0
    finally:
        unsplit.close()


def test_linear_split_k_is_deterministic(tiny):
    h = tiny[2]
    g = torch.Generator().manual_seed(5)
    A = torch.randn(16, 4096, generator=g).to(torch.bfloat16).to(DEV)
    W = (0.05 * torch.randn(2048, 4096, generator=g)).to(torch.bfloat16).to(DEV)
    a = h.linear(A, W, block_n=64, splits=8).clone()
    b = h.linear(A, W, block_n=64, splits=8).clone()
    assert torch.equal(a, b)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
def _pool(cfg, seq_lens, seed, extra=5):
    """Shuffled page pool large enough for every request's seq_len + bs keys."""
    rng = np.random.default_rng(seed)
    P, bs = cfg["page_size"], cfg["block_size"]
    need = [-(-(s + bs) // P) for s in seq_lens]
    W = max(need) + 2
    num_pages = sum(need) + extra
    perm = rng.permutation(num_pages)
    table = np.zeros((len(seq_lens), W), dtype=np.int32)
    cur = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[cur:cur + n]
        cur += n
    return table, num_pages


def assert_attention_close(got, ref, vc, seq_lens, block_size):
    """Element-wise bound on one layer of block attention.  Each output is a
    convex combination of V rows computed in fp32 and stored in fp16: its error
    is at most the fp16 rounding (2^-11 |o|) plus the error of P carried as
    bf16 hi + lo (about 2^-16 relative per weight, so 2^-16 of the V scale);
    the bound allows twice and four times those."""
    v = to_np(vc).astype(np.float64)
    v_rms = float(np.sqrt(np.mean(np.square(v[np.isfinite(v)]))))
    tol = 2.0 ** -10 * np.abs(ref) + 2.0 ** -14 * v_rms
    err = np.abs(got - ref)
    worst = float(np.max(err / tol))
    bad = np.argwhere(err > tol)
    assert bad.size == 0, (f"{len(bad)} elements outside the bound, first {bad[:5].tolist()}, "
                           f"worst err/tol {worst:.2f}")
    return worst


def _attention_case(cfg, seq_lens, seed):
    oc = O.OracleConfig.from_mapping(cfg)
    table, num_pages = _pool(cfg, seq_lens, seed)
    g = torch.Generator().manual_seed(seed)
    shape = (num_pages, cfg["n_kv_heads"], cfg["page_size"], cfg["head_dim"])
    kc = torch.randn(shape, generator=g).to(torch.bfloat16)
    vc = torch.randn(shape, generator=g).to(torch.bfloat16)
    # NaN wherever no request reads (past each request's last key in its last
    # page, and unused pages) must not leak into results
    used = set()
    P = cfg["page_size"]
    for b, s in enumerate(seq_lens):
        n = s + cfg["block_size"]
        used.update(int(x) for x in table[b, :-(-n // P)])
        if n % P:
            last = int(table[b, (n - 1) // P])
            kc[last, :, n % P:] = float("nan")
            vc[last, :, n % P:] = float("nan")
    for pg in set(range(num_pages)) - used:
        kc[pg] = float("nan")
        vc[pg] = float("nan")
    B = len(seq_lens)
    q = torch.randn(B * cfg["block_size"], cfg["n_q_heads"], cfg["head_dim"],
                    generator=g).to(torch.bfloat16)
    ref = O.block_attention(oc, to_np(q).astype(np.float64), to_np(kc).astype(np.float64),
                            to_np(vc).astype(np.float64), table, seq_lens)
    assert np.isfinite(ref).all()
    return q, kc, vc, table, ref


@pytest.mark.parametrize("model,seq_lens", [
    ("tiny", [64]),
    ("tiny", [0, 1, 15, 16, 17, 63, 64, 65, 200]),
    ("qwen3_8b", [2048]),
    ("qwen3_8b", [0, 7, 100, 1000, 5000]),
    ("llama31_8b", [3, 333, 4097]),
    # 8 query heads per kv head: 128 rows per kv group (the mma.sync kernel)
    ("qwen3_8b_g8", [0, 77, 3000]),
])
def test_block_attention_matches_oracle(model, seq_lens):
    if model == "qwen3_8b_g8":
        cfg = dict(synth.model_config("qwen3_8b"), n_kv_heads=4)
    else:
        cfg = synth.model_config(model)
    # the attention entry point needs only geometry: a handle with tiny weights
    # of the same head layout
    small = dict(cfg, intermediate=256, vocab=1024, n_layers=1, mask_token_id=1023,
                 n_target_layers=1)
    W = synth.make_weights(small, seed=1)
    h = DFlash(small, weights_to(W, DEV), max_position=4096)
    try:
        q, kc, vc, table, ref = _attention_case(cfg, seq_lens, seed=len(seq_lens))
        o = h.block_attention(q.to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
                              torch.tensor(table, device=DEV), kc.to(DEV), vc.to(DEV))
        torch.cuda.synchronize()
        got = to_np(o).astype(np.float64).reshape(ref.shape)
        assert np.isfinite(got).all()
        # bf16 inputs are exact in the oracle; what remains is the fp32
        # accumulation, P carried as bf16 hi + lo and the fp16 output
        worst = assert_attention_close(got, ref, vc, seq_lens, cfg["block_size"])
        print(f"attention worst err/bound {worst:.3f}")
        assert h.check_device_errors() == 0
    finally:
        h.close()


@pytest.mark.parametrize("model,seq_lens", [
    ("qwen3_8b", [2048]),
    ("qwen3_8b", [0, 7, 100, 1000, 5000]),
    ("llama31_8b", [3, 333, 4097]),
])
def test_block_attention_cluster_combine(monkeypatch, model, seq_lens):
    """The opt-in plan that combines a request's key splits inside a thread-
    block cluster (distributed shared memory) instead of a second kernel."""
    monkeypatch.setenv("DFLASH_ATTN_CLUSTER", "1")
    cfg = synth.model_config(model)
    small = dict(cfg, intermediate=256, vocab=1024, n_layers=1, mask_token_id=1023,
                 n_target_layers=1)
    h = DFlash(small, weights_to(synth.make_weights(small, seed=1), DEV), max_position=4096)
    try:
        q, kc, vc, table, ref = _attention_case(cfg, seq_lens, seed=len(seq_lens) + 7)
        h.profile_enable(64)
        o = h.block_attention(q.to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
                              torch.tensor(table, device=DEV), kc.to(DEV), vc.to(DEV))
        torch.cuda.synchronize()
        prof = h.profile_read()
        h.profile_disable()
        assert prof["attention"][0] == 1 and "attn_combine" not in prof   # combined in-cluster
        got = to_np(o).astype(np.float64).reshape(ref.shape)
        assert_attention_close(got, ref, vc, seq_lens, cfg["block_size"])
        assert h.check_device_errors() == 0
    finally:
        h.close()


@pytest.mark.parametrize("ring", [2, 6])
@pytest.mark.parametrize("model,seq_lens", [
    ("tiny", [0, 1, 15, 16, 17, 63, 64, 65, 200]),
    ("qwen3_8b", [0, 7, 100, 1000, 5000]),
    ("llama31_8b", [3, 333, 4097]),
])
def test_block_attention_ring_depth(monkeypatch, ring, model, seq_lens):
    """Both K/V ring depths of the 64-key kernel (two stages at two CTAs per
    SM, six stages at one), forced regardless of what the planner picks."""
    monkeypatch.setenv("DFLASH_ATTN_STAGES", str(ring))
    cfg = synth.model_config(model)
    small = dict(cfg, intermediate=256, vocab=1024, n_layers=1, mask_token_id=1023,
                 n_target_layers=1)
    h = DFlash(small, weights_to(synth.make_weights(small, seed=1), DEV), max_position=4096)
    try:
        q, kc, vc, table, ref = _attention_case(cfg, seq_lens, seed=len(seq_lens) + 11)
        o = h.block_attention(q.to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
                              torch.tensor(table, device=DEV), kc.to(DEV), vc.to(DEV))
        torch.cuda.synchronize()
        got = to_np(o).astype(np.float64).reshape(ref.shape)
        assert np.isfinite(got).all()
        assert_attention_close(got, ref, vc, seq_lens, cfg["block_size"])
        assert h.check_device_errors() == 0
    finally:
        h.close()


@pytest.mark.parametrize("model,seq_lens", [
    ("tiny", [0, 1, 15, 16, 17, 63, 64, 65, 200]),
    ("qwen3_8b", [0, 7, 100, 1000, 5000]),
    ("qwen3_8b", [3000] * 40 + [0, 64, 17]),
    ("llama31_8b", [3, 333, 4097]),
])
def test_block_attention_persistent(monkeypatch, model, seq_lens):
    """The persistent six-deep-ring kernel (CTAs walking the (split, head,
    request) items, counters carried across items) gives the same bits as the
    one-item-per-CTA six-deep-ring kernel, and the oracle's values."""
    cfg = synth.model_config(model)
    small = dict(cfg, intermediate=256, vocab=1024, n_layers=1, mask_token_id=1023,
                 n_target_layers=1)
    W = weights_to(synth.make_weights(small, seed=1), DEV)
    q, kc, vc, table, ref = _attention_case(cfg, seq_lens, seed=len(seq_lens) + 5)
    args = (q.to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
            torch.tensor(table, device=DEV), kc.to(DEV), vc.to(DEV))
    outs = []
    for persist in ("0", "1"):
        monkeypatch.setenv("DFLASH_ATTN_STAGES", "6")
        monkeypatch.setenv("DFLASH_ATTN_PERSIST", persist)
        h = DFlash(small, W, max_position=8192)
        try:
            h.profile_enable(16)
            outs.append(h.block_attention(*args))
            torch.cuda.synchronize()
            assert h.profile_read()["attention"][0] == 1
            h.profile_disable()
            assert h.check_device_errors() == 0
        finally:
            h.close()
    assert torch.equal(outs[0], outs[1])
    got = to_np(outs[1]).astype(np.float64).reshape(ref.shape)
    assert_attention_close(got, ref, vc, seq_lens, cfg["block_size"])


@pytest.mark.parametrize("model,seq_lens", [
    ("qwen3_8b", [0, 7, 100, 1000, 5000]),
    ("llama31_8b", [3, 333, 4097]),
])
def test_block_attention_tile32(monkeypatch, model, seq_lens):
    """The two-CTA-per-SM head_dim-128 kernel with 32-key tiles (a four-deep
    ring, two P buffers), as DFLASH_ATTN_TILE=32 selects it."""
    monkeypatch.setenv("DFLASH_ATTN_TILE", "32")
    cfg = synth.model_config(model)
    small = dict(cfg, intermediate=256, vocab=1024, n_layers=1, mask_token_id=1023,
                 n_target_layers=1)
    h = DFlash(small, weights_to(synth.make_weights(small, seed=1), DEV), max_position=8192)
    try:
        q, kc, vc, table, ref = _attention_case(cfg, seq_lens, seed=len(seq_lens) + 13)
        o = h.block_attention(q.to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
                              torch.tensor(table, device=DEV), kc.to(DEV), vc.to(DEV))
        torch.cuda.synchronize()
        got = to_np(o).astype(np.float64).reshape(ref.shape)
        assert np.isfinite(got).all()
        assert_attention_close(got, ref, vc, seq_lens, cfg["block_size"])
        assert h.check_device_errors() == 0
    finally:
        h.close()


@pytest.mark.parametrize("tile", ["32", "64"])
@pytest.mark.parametrize("seq_lens", [[300, 1000], [5000]])
def test_block_attention_growing_scores(monkeypatch, tile, seq_lens):
    """Scores that jump by more than 2^64 after the first tile of a split:
    the head_dim-128 kernel's references must be raised and its transposed
    accumulator rescaled (the rare path), and still agree element-wise with the
    oracle.  q = 1 everywhere; keys in even 64-key tiles are ~0, keys in odd
    tiles ~4.3 in every dimension, so the scaled scores (log2 units) step from
    ~0 to ~70 at every odd tile (every split starts on an even tile)."""
    monkeypatch.setenv("DFLASH_ATTN_TILE", tile)
    cfg = synth.model_config("qwen3_8b")
    small = dict(cfg, intermediate=256, vocab=1024, n_layers=1, mask_token_id=1023,
                 n_target_layers=1)
    h = DFlash(small, weights_to(synth.make_weights(small, seed=1), DEV), max_position=8192)
    try:
        oc = O.OracleConfig.from_mapping(cfg)
        P, bs, Hkv, d = 16, cfg["block_size"], cfg["n_kv_heads"], cfg["head_dim"]
        need = [-(-(s + bs) // P) for s in seq_lens]
        num_pages = sum(need) + 1
        rng = np.random.default_rng(3)
        perm = rng.permutation(num_pages)
        table = np.zeros((len(seq_lens), max(need)), dtype=np.int32)
        cur = 0
        for b, n in enumerate(need):
            table[b, :n] = perm[cur:cur + n]
            cur += n
        g = torch.Generator().manual_seed(9)
        kc = 0.05 * torch.randn(num_pages, Hkv, P, d, generator=g)
        vc = torch.randn(num_pages, Hkv, P, d, generator=g)
        for b, s in enumerate(seq_lens):
            for j in range(s + bs):
                if (j // 64) % 2:
                    kc[int(table[b, j // P]), :, j % P, :] += 4.3
        kc, vc = kc.to(torch.bfloat16), vc.to(torch.bfloat16)
        q = torch.ones(len(seq_lens) * bs, cfg["n_q_heads"], d).to(torch.bfloat16)
        ref = O.block_attention(oc, to_np(q).astype(np.float64), to_np(kc).astype(np.float64),
                                to_np(vc).astype(np.float64), table, seq_lens)
        o = h.block_attention(q.to(DEV), torch.tensor(seq_lens, dtype=torch.int32, device=DEV),
                              torch.tensor(table, device=DEV), kc.to(DEV), vc.to(DEV))
        torch.cuda.synchronize()
        got = to_np(o).astype(np.float64).reshape(ref.shape)
        assert np.isfinite(got).all()
        assert_attention_close(got, ref, vc, seq_lens, bs)
        assert h.check_device_errors() == 0
    finally:
        h.close()


# ----------------------------------------------------------------------------
# verify / paged slots
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("B,K,V", [(1, 3, 1024), (3, 15, 151936), (37, 9, 128256),
                                   (5, 0, 1000), (4, 4, 1027)])
def test_verify_bit_exact(B, K, V):
    g = torch.Generator().manual_seed(B * 100 + K)
    n_acc = torch.randint(0, K + 1, (B,), generator=g)
    drafts = torch.randint(0, V, (B, K), generator=g, dtype=torch.int32)
    T = synth.make_target_logits(g, drafts, n_acc, V)
    if B > 2 and K > 1:
        T[0, 1, :] = 0.5                        # all-equal row -> index 0
        T[1, 0, 7] = float("nan")
        T[2, 1, :] = float("-inf")
        T[0, 2, :] = float("nan")               # all NaN: counts as -inf -> index 0
        T[1, 1, :] = -1.0                       # -0 ties +0 as the maximum -> lower index
        T[1, 1, 5] = -0.0
        T[1, 1, V - 7] = 0.0
        T[2, 0, :] = 0.0                        # ties inside one thread's elements
        T[2, 0, 1027 % V] = 100.0               # (indices 3 and 1027) and across chunks
        T[2, 0, 3] = 100.0
        T[2, 0, V - 1] = 100.0
    ref = O.verify_greedy(to_np(drafts), to_np(T))
    out, n, bonus = verify_greedy(drafts.to(DEV), T.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(out), ref.out_tokens)
    np.testing.assert_array_equal(to_np(n), ref.num_accepted)
    np.testing.assert_array_equal(to_np(bonus), ref.bonus)


def test_verify_full_size_logits():
    """[128, 16, 151936] fp32 logits with geometric acceptance (mean tau ~ 6)."""
    cfg = synth.model_config("qwen3_8b")
    sb = synth.make_step_batch(cfg, 128, 8192, 32768, accept="geometric", seed=3,
                               with_aux=False)
    ref = O.verify_greedy(to_np(sb.prev_drafts), to_np(sb.target_logits))
    np.testing.assert_array_equal(ref.num_accepted, to_np(sb.n_accept))
    out, n, bonus = verify_greedy(sb.prev_drafts.to(DEV), sb.target_logits.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(out), ref.out_tokens)
    np.testing.assert_array_equal(to_np(n), ref.num_accepted)
    np.testing.assert_array_equal(to_np(bonus), ref.bonus)


def test_paged_slots_bit_exact():
    rng = np.random.default_rng(0)
    table = rng.integers(0, 10000, (7, 33)).astype(np.int32)
    pos = rng.integers(0, 33 * 16 + 40, 5000)          # includes clamped positions
    req = rng.integers(0, 7, 5000)
    ref = O.paged_slots(pos, req, table, 16)
    got = paged_slots(torch.tensor(pos, device=DEV), torch.tensor(req, device=DEV),
                      torch.tensor(table, device=DEV))
    np.testing.assert_array_equal(to_np(got), ref)
    neg = paged_slots(torch.tensor([-1, 3], device=DEV), torch.tensor([0, 0], device=DEV),
                      torch.tensor(table, device=DEV))
    assert to_np(neg).tolist() == [-1, int(table[0, 0]) * 16 + 3]


# ----------------------------------------------------------------------------
# injection
# ----------------------------------------------------------------------------
def _inject_case(cfg, Wt, h, n, seed, sample=None):
    oc = O.OracleConfig.from_mapping(cfg)
    rng = np.random.default_rng(seed)
    P = cfg["page_size"]
    num_pages = -(-(n + 40) // P) + 7
    table = rng.permutation(num_pages)[None, :].astype(np.int32)
    pos = np.arange(n, dtype=np.int64) + 40
    slots = O.paged_slots(pos, np.zeros(n, np.int64), table, P)
    slots[rng.random(n) < 0.1] = -1                      # padding rows
    aux = synth.make_aux(n, cfg, seed)
    shape = (num_pages, cfg["n_kv_heads"], P, cfg["head_dim"])
    sentinel = 7.0
    kc = [torch.full(shape, sentinel, dtype=torch.bfloat16, device=DEV)
          for _ in range(cfg["n_layers"])]
    vc = [torch.full(shape, sentinel, dtype=torch.bfloat16, device=DEV)
          for _ in range(cfg["n_layers"])]
    h.inject_context(aux.to(DEV), torch.tensor(pos, device=DEV),
                     torch.tensor(slots, device=DEV), kc, vc)
    torch.cuda.synchronize()
    assert h.check_device_errors() == 0
    rows = np.arange(n) if sample is None else sample
    W = weights_np(Wt) if not isinstance(Wt["fc_w"], np.ndarray) else Wt
    auxn = to_np(aux)[rows].astype(np.float64)
    ctx_io = O.context_fusion(oc, W, auxn, "device")
    k_io, v_io = O.context_kv(oc, W, ctx_io, pos[rows], "device")
    ctx_ex = O.context_fusion(oc, W, auxn, "exact")
    k_ex, v_ex = O.context_kv(oc, W, ctx_ex, pos[rows], "exact")
    for l in range(cfg["n_layers"]):
        kg, vg = to_np(kc[l]), to_np(vc[l])
        for j, r in enumerate(rows):
            s = slots[r]
            if s < 0:
                continue
            gk, gv = kg[s // P, :, s % P], vg[s // P, :, s % P]
            # Against the storage-precision oracle: one bf16 ulp of the larger
            # value plus 2e-3 of the head's RMS (pre-rounding values differ by
            # fp32 accumulation order, which can move a value across a bf16
            # rounding boundary); against the exact oracle: 1e-2 relative L2.
            for got, want in ((gk, k_io[l][j]), (gv, v_io[l][j])):
                tol = (2.0 ** -7 * np.maximum(np.abs(got), np.abs(want))
                       + 2e-3 * np.sqrt(np.mean(want ** 2, axis=-1, keepdims=True)))
                assert np.all(np.abs(got - want) <= tol), (l, r)
            assert rel_l2(gk, k_ex[l][j]) < 1e-2 and rel_l2(gv, v_ex[l][j]) < 1e-2
        # padding rows and untouched slots keep the sentinel
        for r in np.nonzero(slots < 0)[0][:8]:
            s = O.paged_slots(pos[r:r + 1], np.zeros(1, np.int64), table, P)[0]
            assert (kg[s // P, :, s % P] == sentinel).all()


def test_inject_tiny(tiny):
    cfg, Wt, h = tiny
    for n in (1, 5, 64, 130):
        _inject_case(cfg, Wt, h, n, seed=n)


def test_inject_qwen3_shape_sampled():
    cfg = synth.model_config("qwen3_8b")
    Wt = synth.make_weights(cfg, seed=0)
    h = DFlash(cfg, weights_to(Wt, DEV), max_position=40960)
    try:
        rng = np.random.default_rng(1)
        W = weights_np({k: Wt[k] for k in ("fc_w", "hidden_norm_w", "wk", "wv", "k_norm_w")})
        for n in (16, 2048):
            sample = np.sort(rng.choice(n, size=min(n, 12), replace=False))
            _inject_case(cfg, W, h, n, seed=n, sample=sample)
    finally:
        h.close()
