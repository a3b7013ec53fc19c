// attention_tc2.cuh — non-causal block attention for head_dim 128, two CTAs per
// SM, with P V computed transposed.
//
// Same contract as attn_block_tc_kernel (attention_tc.cuh): one CTA per
// (request b, kv head h, key split); the kv group's query rows (bs block slots x
// G heads, zero-padded to 64) attend to the request's keys [split * chunk, ...)
// of [0, seq_len + bs) with no mask inside the range ("DFlash Speculative
// Decoding in the vLLM Neuron Framework", §What is DFlash: every block query
// sees the injected context and the whole block).
//
// What is different, and why (measured on B200 at 128 requests x 8k-32k keys):
//   - Two CTAs per SM (99 KB of shared memory each, 64 KB of it a K/V ring: two
//     64-key tiles, or four 32-key tiles).  A single CTA streaming paged K/V
//     through TMA tops out near 5 TB/s whatever its ring depth; two CTAs per SM
//     reach 7 TB/s.
//   - With 32-key tiles the one 16 KB P area holds two P buffers (the two
//     halves of its 128-byte rows), so the softmax of tile t+1 writes P while
//     P V of tile t runs, and ring slots are released at half the grain.
//   - O is accumulated transposed: O^T[d][r] += V^T[d][k] P^T[k][r], an MMA
//     with M = head_dim = 128 (the full-rate shape) instead of M = 64 rows;
//     V (MN-major) and P (K-major) keep their shared-memory layouts, only the
//     roles swap.  O^T lives in TMEM as 128 lanes (d) x 64 columns (rows).
//   - The grid is split-major (x = kv head, y = request, z = split): the CTAs
//     are dispatched roughly in linear block order, so every request's full
//     first splits go out before the later ones, and the last wave is made of
//     the partial last splits (shorter by half on average) instead of full
//     8192-key splits of the last requests.  Outputs are unchanged (each CTA
//     writes its own partial); 128 requests x 8k-32k keys: 5.46 -> 5.60 TB/s
//     alone, 0.64 -> 0.70 of the copy figure inside the whole step.
//   - The softmax keeps one reference m_r per row, fixed at the first tile's
//     row maximum.  Later tiles compute p = 2^(s * scale - m_r) directly, with
//     no per-tile maximum: exp2 of anything up to 2^kTc2Headroom stays well
//     inside fp32 and bf16 range.  All four softmax warps vote once per tile
//     (one bar.red.or); only if some score exceeds its reference by more than
//     the headroom are that tile's references raised and O^T's columns, the
//     row sums and the tile's exponents rescaled (the reference cancels
//     exactly in O / l either way).  The mask runs on partial tiles only.
//
//   warp 0      TMA producer (one thread): K and V of 16-key pages (two
//               64-column boxes per page, 128-byte swizzle), each tensor into
//               its own ring: a K slot is released as soon as S of its tile
//               has run, a V slot once P V has.  Measured per tile in one CTA
//               (128 requests x 8k-32k keys): a load takes ~3100 cycles to
//               land and a tile holds its slot ~2400 cycles, so with one K+V
//               slot per tile a two-deep ring paced the CTA at ~3000 cycles
//               per tile; releasing K after S lets the next K load start
//               ~1900 cycles earlier.
//   warp 1      MMA issuer (one thread): S = Q K^T (M = 64, N = 64 keys) into a
//               double-buffered TMEM S; O^T += V^T P_hi^T + V^T P_lo^T
//   warps 2..5  softmax: 16 rows of S each (tcgen05.ld.16x256b), P split into
//               bf16 hi + lo parts in shared memory; then the epilogue, one
//               TMEM lane (d) per thread over the 64 rows
//
// Every mbarrier wait is bounded; after a wait runs out the warp keeps walking
// its loop with every further wait skipped, so that all four softmax warps
// still reach each of their named barriers and the CTA winds down.
#pragma once

#include "attention_tc.cuh"

namespace dflash {

constexpr int kTc2RingBytes = 65536;   // K/V ring per CTA
constexpr float kTc2Headroom = 64.f;   // log2 of the largest p = 2^(s - m) kept unscaled
constexpr int kTc2VoteBar = 1;         // named barrier of the four softmax warps

// KT = keys per tile (64 or 32); ring depth ST and P buffers follow from it.
template <int KT>
struct Tc2Cfg {
  static constexpr int D = 128;
  static constexpr int kKVBytes = (D / 64) * KT * 128;         // one K (or V) tile
  static constexpr int ST = kTc2RingBytes / (2 * kKVBytes);    // K/V ring depth
  static constexpr int kPBufs = 64 / KT;                       // P buffers in the P rows
  static constexpr int kQBytes = (D / 64) * kTcM * 128;        // 16 KB
  static constexpr int kPBytes = kTcM * 128;                   // P hi (or lo): 8 KB
  static constexpr int kOffV = ST * kKVBytes;
  static constexpr int kOffQ = 2 * ST * kKVBytes;
  static constexpr int kOffP = kOffQ + kQBytes;
  static constexpr int kOffAlpha = kOffP + 2 * kPBytes;        // [2][64] fp32 rescale factors
  static constexpr int kOffL = kOffAlpha + 2 * kTcM * 4;       // [64] fp32 row sums
  static constexpr int kOffM = kOffL + kTcM * 4;               // [64] fp32 row references
  static constexpr int kOffBar = kOffM + kTcM * 4;
  static constexpr int kOffPages = kOffBar + 256;              // the split's page rows
  static constexpr int kMaxPages = 8192 / 16 + 1;              // pages of the longest split
  static constexpr int kSmem = 1024 + kOffPages + kMaxPages * 4;
  static constexpr int kOCol = 2 * KT;                         // TMEM column of O^T
  static constexpr int kTmemCols = KT == 64 ? 256 : 128;
  static_assert(KT == 64 || KT == 32, "tile width");
  static_assert(ST >= 2 && ST <= 4, "ring depth");
  static_assert(kOCol + kTcM <= kTmemCols, "TMEM budget");
  static_assert(2 * (kSmem + 1024) <= 233472, "two CTAs per SM");
};

__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// CTA-wide OR of `pred` over the `n` threads of named barrier `id` (a barrier).
__device__ __forceinline__ bool bar_red_or(int id, int n, bool pred) {
  uint32_t r;
  __syncwarp();
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// kind::f16 instruction descriptor, bf16 A and B with the given major-ness
// (bit 15: A MN-major, bit 16: B MN-major), fp32 accumulator.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_ab(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const float* v) {
  uint32_t r[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

template <int KT>
__global__ void __launch_bounds__(kTcThreads, 2)
    attn_block_tc2_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = Tc2Cfg<KT>;
  constexpr int D = C::D, ST = C::ST, NB = C::kPBufs;
  pdl_trigger();
  pdl_wait();
  const int h = blockIdx.x, b = blockIdx.y, split = blockIdx.z;   // split-major grid
  const int n_keys = p.seq_lens[b] + p.bs;
  const int k0 = split * p.chunk_keys;
  if (k0 >= n_keys) return;
  const int k1 = min(n_keys, k0 + p.chunk_keys);
  const int n_splits_b = (n_keys + p.chunk_keys - 1) / p.chunk_keys;
  const int n_tiles = (k1 - k0 + KT - 1) / KT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sPh = smem + C::kOffP;
  uint8_t* sPl = smem + C::kOffP + C::kPBytes;
  float* sAlpha = reinterpret_cast<float*>(smem + C::kOffAlpha);   // [2][64]
  float* sL = reinterpret_cast<float*>(smem + C::kOffL);
  float* sM = reinterpret_cast<float*>(smem + C::kOffM);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* k_full = bars;         // [ST] K ring
  uint64_t* k_empty = bars + 4;    // [ST]
  uint64_t* v_full = bars + 8;     // [ST] V ring
  uint64_t* v_empty = bars + 12;   // [ST]
  uint64_t* s_full = bars + 16;    // [2] S buffers (tile t -> t % 2)
  uint64_t* s_empty = bars + 18;   // [2]
  uint64_t* p_full = bars + 20;    // [2] barrier t % 2 (P buffer t % NB)
  uint64_t* p_empty = bars + 22;   // [2] two P buffers: P V of the buffer's last tile landed
  uint64_t* o_ready = bars + 24;   // one phase per tile: its P V landed
  uint64_t* q_full = bars + 25;
  uint64_t* o_final = bars + 26;   // the last tile's P V landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 27);
  // rows of this split's pages in the [pages * Hkv * 16, D] views of the pools,
  // (-16: a page past the table or the pool; the loads then fill zeros)
  int* s_rows = reinterpret_cast<int*>(smem + C::kOffPages);
  auto sK = [&](int s) { return smem + s * C::kKVBytes; };
  auto sV = [&](int s) { return smem + C::kOffV + s * C::kKVBytes; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(o_ready, 1);
    mbar_init(q_full, 4);
    mbar_init(o_final, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // One thread feeds both rings, polling them in turn: K of tile tk as soon
    // as S of tile tk - ST has run, V of tile tv (never ahead of K) as soon as
    // P V of tile tv - ST has.  (One thread, so that the two rings never wait
    // on each other through a divergent warp.)
    // the split's page rows, read from the block table once (all 32 lanes),
    // checked against the table width and the pool
    const int pg0 = k0 >> 4, npg = min(C::kMaxPages, ((k1 - 1) >> 4) - pg0 + 1);
    const int* bt = p.block_table + static_cast<size_t>(b) * p.W;
    for (int j = lane; j < npg; j += 32) {
      const int pg = pg0 + j;
      int y = -16;
      if (pg >= p.W) {
        raise_error(p.err, DFLASH_DEVERR_TABLE);
      } else {
        const int page = bt[pg];
        if (page < 0 || page >= p.num_pages) raise_error(p.err, DFLASH_DEVERR_SLOT);
        else y = (page * p.Hkv + h) * 16;
      }
      s_rows[j] = y;
    }
    __syncwarp();
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      // the rows of tile t's pages (-16 past the split: TMA fills zeros)
      auto page_rows = [&](int t, int* y) {
        const int npages = (min(KT, k1 - (k0 + t * KT)) + 15) >> 4;
#pragma unroll
        for (int j = 0; j < KT / 16; ++j) y[j] = j < npages ? s_rows[t * (KT / 16) + j] : -16;
      };
      auto issue = [&](int t, bool is_v) {
        const int s = t % ST;
        uint64_t* full = is_v ? &v_full[s] : &k_full[s];
        const CUtensorMap* map = is_v ? &tmV : &tmK;
        uint8_t* dst = is_v ? sV(s) : sK(s);
        int y[KT / 16];
        page_rows(t, y);
        mbar_arrive_expect_tx(full, static_cast<uint32_t>(C::kKVBytes));
#pragma unroll
        for (int j = 0; j < KT / 16; ++j)
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_2d(dst + hf * KT * 128 + j * 2048, map, full, hf * 64, y[j]);
      };
      int tk = 0, tv = 0;
      long long idle_since = clock64();
      while (tv < n_tiles) {
        bool progress = false;
        // V first: P V of tile tv waits on it, while K of tile tk (released
        // right after S) still has the softmax and P V of a tile as slack
        if (tv < tk && mbar_test_wait(&v_empty[tv % ST], ((tv / ST) & 1) ^ 1u)) {
          issue(tv++, true);
          progress = true;
        }
        if (tk < n_tiles && mbar_test_wait(&k_empty[tk % ST], ((tk / ST) & 1) ^ 1u)) {
          issue(tk++, false);
          progress = true;
        }
        if (progress) {
          idle_since = clock64();
        } else if (clock64() - idle_since >
                   *reinterpret_cast<volatile long long*>(&g_wait_limit_cycles)) {
          raise_error(p.err, DFLASH_DEVERR_TIMEOUT);
          break;
        } else if (p.err &&
                   (*reinterpret_cast<volatile unsigned*>(p.err) & DFLASH_DEVERR_TIMEOUT)) {
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc_bf16_ab(kTcM, KT, false, false);
      const uint32_t idesc_pv = umma_idesc_bf16_ab(D, kTcM, true, false);
      bool ok = mbar_wait(q_full, 0, p.err);
      tc_fence_after();
      auto issue_qk = [&](int t) -> bool {
        const int kv = t % ST, kvu = t / ST;
        const int s = t & 1, u = t >> 1;
        if (!mbar_wait(&k_full[kv], kvu & 1, p.err)) return false;
        if (!mbar_wait(&s_empty[s], (u & 1) ^ 1u, p.err)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int half = kk >> 2, w = kk & 3;
          const uint64_t ad = umma_desc_sw128(smem_u32(sQ + half * kTcM * 128 + w * 32));
          const uint64_t bd = umma_desc_sw128(smem_u32(sK(kv) + half * KT * 128 + w * 32));
          umma_f16kind(tmem_base + s * KT, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[s]);
        umma_commit(&k_empty[kv]);      // K of this tile is no longer needed
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int t = 0; ok && t < n_tiles; ++t) {
        // S of tile t+1 ahead of P V of tile t when its K/V have landed
        const int s1 = (t + 1) & 1, u1 = (t + 1) >> 1;
        const int kv1 = (t + 1) % ST, kvu1 = (t + 1) / ST;
        const bool qk_first = t + 1 < n_tiles && mbar_try_wait(&k_full[kv1], kvu1 & 1) &&
                              mbar_try_wait(&s_empty[s1], (u1 & 1) ^ 1u);
        if (qk_first && !issue_qk(t + 1)) break;
        const int s = t & 1, u = t >> 1;
        if (!mbar_wait(&p_full[s], u & 1, p.err)) break;
        if (!mbar_wait(&v_full[t % ST], (t / ST) & 1, p.err)) break;
        tc_fence_after();
        // O^T[d][r] += V^T[d][k] P^T[k][r]: A = V (MN-major, 64-column halves
        // KT * 128 bytes apart), B = P (K-major, rows = query rows; buffer
        // t % NB at byte column (t % NB) * 2 KT of the 128-byte rows)
        const int pb = (t % NB) * (KT / 16);
#pragma unroll
        for (int lohi = 0; lohi < 2; ++lohi) {
#pragma unroll
          for (int kk = 0; kk < KT / 16; ++kk) {
            const uint64_t ad =
                umma_desc_sw128_mn(smem_u32(sV(t % ST) + kk * 16 * 128), KT * 128, 1024);
            const uint64_t bd = umma_desc_sw128(smem_u32((lohi ? sPl : sPh) + (pb + kk) * 32));
            umma_f16kind(tmem_base + C::kOCol, ad, bd, idesc_pv,
                         (t > 0 || lohi > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&v_empty[t % ST]);
        if (NB == 2) umma_commit(&p_empty[s]);
        umma_commit(o_ready);
        if (t + 1 == n_tiles) umma_commit(o_final);
        if (!qk_first && t + 1 < n_tiles && !issue_qk(t + 1)) break;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int sp = warp & 3;                    // TMEM sub-partition
    const int tid = threadIdx.x - 64;           // 0..127
    {
      // Q rows r = i * G + g of this kv group -> K-major, 128B-swizzled operand
      constexpr int kQPer = kTcM * (D / 8) / 128;
      uint4 qv[kQPer];
#pragma unroll
      for (int u = 0; u < kQPer; ++u) {
        const int e = tid + u * 128;
        const int r = e / (D / 8), c = e - r * (D / 8);
        qv[u] = make_uint4(0, 0, 0, 0);
        if (r < p.R) {
          const int i = r / p.G, g = r - (r / p.G) * p.G;
          const bf16* src = p.q + (static_cast<size_t>(b * p.bs + i) * p.Hq + h * p.G + g) * D;
          qv[u] = *reinterpret_cast<const uint4*>(src + c * 8);
        }
      }
#pragma unroll
      for (int u = 0; u < kQPer; ++u) {
        const int e = tid + u * 128;
        const int r = e / (D / 8), c = e - r * (D / 8);
        *reinterpret_cast<uint4*>(sQ + (c >> 3) * kTcM * 128 + r * 128 +
                                  (((c & 7) ^ (r & 7)) << 4)) = qv[u];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    }

    const uint32_t lane_base = static_cast<uint32_t>(32 * sp) << 16;
    const int r0 = 16 * sp + (lane >> 2);       // this thread's S rows r0 and r0 + 8
    const float scale = p.scale_log2;
    float m_ref[2] = {0.f, 0.f};
    float l_run[2] = {0.f, 0.f};
    int apar = 0;                               // sAlpha buffer of the next rescale
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int s = t & 1, u = t >> 1;
      if (ok) ok = mbar_wait(&s_full[s], u & 1, p.err);
      tc_fence_after();
      constexpr int NX = KT / 2;            // S values of this thread: rows r0, r0 + 8
      float x[NX];
      if constexpr (KT == 64)
        tmem_ld_16x256b_x8(tmem_base + lane_base + s * KT, x);
      else
        tmem_ld_16x256b_x4(tmem_base + lane_base + s * KT, x);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[s]);

      const int nvalid = min(KT, k1 - (k0 + t * KT));
      if (nvalid < KT) {
        // partial tile: keys past the range score -inf (p = 0)
#pragma unroll
        for (int j = 0; j < KT / 8; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (j * 8 + 2 * (lane & 3) + (e & 1) >= nvalid) x[4 * j + e] = -INFINITY;
      }
      if (t == 0) {
        // the rows' references: the first tile's maxima (key 0 is always valid)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int q = 0; q < NX; ++q) mx[(q >> 1) & 1] = fmaxf(mx[(q >> 1) & 1], x[q]);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
          mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
          m_ref[hh] = mx[hh] * scale;
        }
#pragma unroll
        for (int q = 0; q < NX; ++q) x[q] = fmaf(x[q], scale, -m_ref[(q >> 1) & 1]);
      } else {
        bool over = false;
#pragma unroll
        for (int q = 0; q < NX; ++q) {
          x[q] = fmaf(x[q], scale, -m_ref[(q >> 1) & 1]);
          over |= x[q] > kTc2Headroom;
        }
        if (bar_red_or(kTc2VoteBar, 128, over)) {
          // rare: raise the references of the rows that outgrew them and
          // rescale their O^T columns, row sums and this tile's exponents
          float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
          for (int q = 0; q < NX; ++q) mx[(q >> 1) & 1] = fmaxf(mx[(q >> 1) & 1], x[q]);
          float alpha[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
            mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
            const float raise = mx[hh] > 0.f ? mx[hh] : 0.f;
            alpha[hh] = ex2_ftz(-raise);
            m_ref[hh] += raise;
            l_run[hh] *= alpha[hh];
            mx[hh] = raise;
          }
#pragma unroll
          for (int q = 0; q < NX; ++q) x[q] -= mx[(q >> 1) & 1];
          float* al = sAlpha + apar * kTcM;
          if ((lane & 3) == 0) {
            al[r0] = alpha[0];
            al[r0 + 8] = alpha[1];
          }
          named_bar_sync(kTc2VoteBar, 128);
          // O^T holds P V of tiles < t: rescale its columns once P V(t-1) landed
          if (ok) ok = mbar_wait(o_ready, (t - 1) & 1, p.err);
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < kTcM / 32; ++c) {
            float ov[32];
            tmem_ld_32x32b_x32(tmem_base + lane_base + C::kOCol + c * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) ov[q] *= al[c * 32 + q];
            tmem_st_32x32b_x32(tmem_base + lane_base + C::kOCol + c * 32, ov);
          }
          tmem_st_wait();
          tc_fence_before();
          apar ^= 1;
        }
      }
#pragma unroll
      for (int q = 0; q < NX; ++q) {
        x[q] = ex2_ftz(x[q]);
        l_run[(q >> 1) & 1] += x[q];
      }
      // the P buffer is free once P V of the last tile that used it landed
      // (one buffer: tile t-1, via o_ready; two: tile t-2, via p_empty)
      if (NB == 1) {
        if (t > 0 && ok) ok = mbar_wait(o_ready, (t - 1) & 1, p.err);
      } else {
        if (ok) ok = mbar_wait(&p_empty[s], (u & 1) ^ 1u, p.err);
      }
      const int cb = (t % NB) * (KT / 8);     // the buffer's first 16-byte chunk of a row
#pragma unroll
      for (int j = 0; j < KT / 8; ++j) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int r = r0 + 8 * hh;
          uint32_t hi, lo;
          split_bf16x2(x[4 * j + 2 * hh], x[4 * j + 2 * hh + 1], hi, lo);
          const int off = r * 128 + (((cb + j) ^ (r & 7)) << 4) + (lane & 3) * 4;
          *reinterpret_cast<uint32_t*>(sPh + off) = hi;
          *reinterpret_cast<uint32_t*>(sPl + off) = lo;
        }
      }
      if (sp == 0 && (nvalid & 15)) {
        // V rows past the last key of a partly used page may hold anything
        // (NaN patterns included): zero them so that P = 0 columns add 0,
        // once this tile's V has landed
        if (ok) ok = mbar_wait(&v_full[t % ST], (t / ST) & 1, p.err);
        const int jp = nvalid >> 4, rr0 = nvalid & 15;
        const int n16 = (16 - rr0) * (D / 64) * 8;
        for (int e = lane; e < n16; e += 32) {
          const int hf = e / ((16 - rr0) * 8);
          const int rem = e - hf * (16 - rr0) * 8;
          const int rr = rr0 + rem / 8, cc = rem & 7;
          *reinterpret_cast<uint4*>(sV(t % ST) + hf * KT * 128 + jp * 2048 + rr * 128 + cc * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[s]);
    }

    // ---------------------------------------------------------------- epilogue
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 1);
      l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 2);
    }
    if ((lane & 3) == 0) {
      // one split: the rows' 1 / l for the normalised output; several: l
      sL[r0] = n_splits_b == 1 ? 1.f / l_run[0] : l_run[0];
      sL[r0 + 8] = n_splits_b == 1 ? 1.f / l_run[1] : l_run[1];
      sM[r0] = m_ref[0];
      sM[r0 + 8] = m_ref[1];
    }
    named_bar_sync(kTc2VoteBar, 128);
    if (ok) ok = mbar_wait(o_final, 0, p.err);
    tc_fence_after();
    // this thread: TMEM lane 32 sp + lane = output dim d, over the 64 rows
    const int d = 32 * sp + lane;
    float o[kTcM];
#pragma unroll
    for (int c = 0; c < kTcM / 32; ++c)
      tmem_ld_32x32b_x32(tmem_base + lane_base + C::kOCol + c * 32, o + 32 * c);
    tmem_ld_wait();
    if (ok) {
      if (n_splits_b == 1) {
        // row r = i * G + g -> output row (b * bs + i), head h * G + g
        f16* base = p.o + (static_cast<size_t>(b * p.bs) * p.Hq + h * p.G) * D + d;
        int i = 0, g = 0;
#pragma unroll
        for (int r = 0; r < kTcM; ++r) {
          if (r < p.R) base[static_cast<size_t>(i * p.Hq + g) * D] = __float2half_rn(o[r] * sL[r]);
          if (++g == p.G) {
            g = 0;
            ++i;
          }
        }
      } else {
        const size_t prow = (static_cast<size_t>(split) * p.B + b) * p.Hkv + h;
        float* dst = p.part_o + prow * p.R * D + d;
#pragma unroll
        for (int r = 0; r < kTcM; ++r)
          if (r < p.R) dst[static_cast<size_t>(r) * D] = o[r];
        if (tid < p.R)
          *reinterpret_cast<float2*>(p.part_ml + (prow * p.R + tid) * 2) =
              make_float2(sM[tid], sL[tid]);
      }
    }
  }

  tc_fence_before();
  cta_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace dflash
