// attention_tc.cuh — non-causal block attention on the 5th-generation tensor
// cores (tcgen05 MMA, accumulators in tensor memory).
//
// Same contract as attn_block_kernel (attention.cuh): one CTA per (request b,
// kv head h, key split); every query row of the kv group (bs block slots x G
// heads, zero-padded to 64 rows) attends to the request's keys
// [split * chunk, ...) of [0, seq_len + bs) with no mask inside the range.
//
//   warp 0      TMA producer: walks the block table, stages KT-key tiles of K
//               and V (KT / 16 pages of 16 keys, 128-byte swizzle) in a ring of
//               ST tiles
//   warp 1      MMA issuer (one thread): S = Q K^T into a double-buffered TMEM
//               S (M=64 rows x KT keys), then O += P_hi V + P_lo V into TMEM O
//               (64 x d); S of tile t+1 is issued before P V of tile t when its
//               K/V have landed
//   warps 2..5  softmax: each reads its 16 rows of S with tcgen05.ld.16x256b
//               (the mma.sync accumulator-fragment layout), applies the online
//               softmax (row statistics by quad shuffles), writes P split into
//               bf16 hi + lo parts to shared memory as the next MMA's operand.
//               O is rescaled in TMEM only when a row maximum grows by more than
//               2^8 since the last rescale (the reference maximum is shared by P,
//               the row sum and O, so the result is exact either way).
//
// Variants <D, KT, ST>: 128-key tiles with a 2-deep ring and two P buffers
// (the opt-in cluster mode below); 64-key tiles with one P buffer and a 2-deep
// ring (100 KB of shared memory: two CTAs per SM) or a 6-deep ring (231 KB:
// one CTA per SM, six tiles in flight, for long key splits).
//
// Shared memory: K/V ring ST x (K + V) tiles, Q (64 x d), P hi/lo x 1 or 2
// buffers, barriers.  TMEM: S buffers at columns [0, 2 KT), O at
// [2 KT, 2 KT + d).  Every wait is bounded; a wait that runs out sets the
// timeout bit and the CTA winds down.
//
// Cluster mode (opt-in; few requests: splitting the keys is what fills the GPU): the
// splits of one (request, kv head) are the CTAs of one cluster; CTA rank q
// owns rows q, q + S, ...  Once every CTA of the cluster is past its key loop
// (first cluster barrier), each pushes its unnormalised O rows and (m, l)
// with remote shared-memory stores into the owners' (now idle) K/V rings;
// after the second barrier each owner combines its rows from local shared
// memory over the S pieces in rank order and writes the fp16 output.  No
// partials reach global memory and no combine kernel runs.  A split past the
// request's last key contributes (m, l) = (-inf, 0).
#pragma once

#include "attention.cuh"

namespace dflash {

constexpr int kTcKeys = 128;        // keys per tile of the few-request (cluster) variant
constexpr int kTcKeysSmall = 64;    // keys per tile of the many-request variant (2 CTAs per SM)
constexpr int kTcStages = 2;        // K/V ring depth
constexpr int kTcDeepStages = 6;    // K/V ring depth of the one-CTA-per-SM 64-key variant
constexpr int kTcM = 64;            // MMA M: query rows of a kv group, zero-padded
constexpr int kTcThreads = 192;     // warp 0 TMA, warp 1 MMA, warps 2..5 softmax
constexpr float kTcLazyRescale = 8.f;  // log2 of the growth that forces an O rescale

// Per tile width KT (keys) and ring depth ST: 128-key tiles keep more keys in
// flight per CTA (the cluster mode); 64-key tiles with one P buffer and a
// 2-deep ring fit two CTAs per SM (shared memory 100 KB, 256 TMEM columns) so
// that their pipelines hide each other's latency; with a 6-deep ring one CTA
// per SM keeps six tiles in flight.
template <int D, int KT, int ST = kTcStages>
struct TcAttnCfg {
  static constexpr int kHalves = D / 64;                      // 64-element halves of a row
  static constexpr int kKVBytes = kHalves * KT * 128;         // one K (or V) tile
  static constexpr int kQBytes = kHalves * kTcM * 128;
  static constexpr int kPBytes = (KT / 64) * kTcM * 128;      // P hi (or lo) of one tile
  static constexpr int kPBufs = KT == 64 ? 1 : 2;             // P buffers (ring of tiles)
  static constexpr int kStages = ST;                          // K/V ring depth
  static constexpr int kOffV = ST * kKVBytes;
  static constexpr int kOffQ = 2 * ST * kKVBytes;
  static constexpr int kOffP = kOffQ + kQBytes;
  static constexpr int kOffBar = kOffP + 2 * kPBufs * kPBytes;
  static constexpr int kSmem = 1024 + kOffBar + 256;
  static constexpr int kOCol = 2 * KT;                        // TMEM column of O
  static constexpr int kTmemCols = kOCol + D <= 256 ? 256 : 512;
  static constexpr int kMinBlocks = (KT == 64 && ST == 2) ? 2 : 1;
  // cluster combine, inside the (then idle) K/V ring: received O rows
  // [lr * S + src][D + 8] and (m, l) [lr * S + src] (S * ceil(64 / S) <= 71 slots)
  static constexpr int kCombSlots = kTcM + 7;
  static constexpr int kCombOffML = kCombSlots * (D + 8) * 4;
  static_assert(KT == 64 || KT == 128, "tile width");
  static_assert(kCombOffML + kCombSlots * 8 <= 2 * ST * kKVBytes, "combine buffers");
  static_assert(ST >= 2 && ST <= 8, "ring depth");
  static_assert(kSmem <= 232448, "shared memory");
  static_assert(kOCol + D <= 512, "TMEM budget");
};

template <int D, int KT, int ST = kTcStages>
__global__ void __launch_bounds__(kTcThreads, TcAttnCfg<D, KT, ST>::kMinBlocks)
    attn_block_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = TcAttnCfg<D, KT, ST>;
  pdl_trigger();
  pdl_wait();
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n_keys = p.seq_lens[b] + p.bs;
  const int k0 = split * p.chunk_keys;
  // (every CTA of a cluster stays to the end: its peers read its shared memory)
  if (k0 >= n_keys && !p.cluster) return;
  const int k1 = min(n_keys, k0 + p.chunk_keys);
  const int n_splits_b = (n_keys + p.chunk_keys - 1) / p.chunk_keys;
  const int n_tiles = k0 < n_keys ? (k1 - k0 + KT - 1) / KT : 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;        // [ST] K/V ring (tile t -> stage t % ST)
  uint64_t* kv_empty = bars + 8;   // [ST]
  uint64_t* s_full = bars + 16;    // [2] S buffers (tile t -> t % 2)
  uint64_t* s_empty = bars + 18;   // [2]
  uint64_t* p_full = bars + 20;    // [2] P buffers
  uint64_t* p_empty = bars + 22;   // [2]
  uint64_t* o_ready = bars + 24;   // one phase per tile: P V of that tile landed
  uint64_t* q_full = bars + 25;
  uint64_t* o_final = bars + 26;   // the last tile's P V landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 27);
  auto sK = [&](int s) { return smem + s * C::kKVBytes; };
  auto sV = [&](int s) { return smem + C::kOffV + s * C::kKVBytes; };
  auto sP = [&](int lohi, int buf) {
    return smem + C::kOffP + ((C::kPBufs == 1 ? 0 : buf) * 2 + lohi) * C::kPBytes;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
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
  // softmax warps, cluster mode: this thread's O rows (r0, r0 + 8) and (m, l)
  float o[D / 8][4];
  float m_fin[2] = {-INFINITY, -INFINITY}, l_fin[2] = {0.f, 0.f};
  bool have = false;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int* bt = p.block_table + static_cast<size_t>(b) * p.W;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % ST, u = t / ST;
        if (!mbar_wait(&kv_empty[s], (u & 1) ^ 1u, p.err)) break;
        const int t0 = k0 + t * KT;
        const int nvalid = min(KT, k1 - t0);
        const int npages = (nvalid + 15) >> 4;
        mbar_arrive_expect_tx(&kv_full[s],
                              static_cast<uint32_t>((KT / 16) * C::kHalves * 2048 * 2));
        for (int j = 0; j < KT / 16; ++j) {
          int y = -16;  // pages past the range: fully out of bounds, TMA fills zeros
          if (j < npages) {
            const int pg = (t0 >> 4) + j;
            if (pg >= p.W) {
              raise_error(p.err, DFLASH_DEVERR_TABLE);
            } else {
              const int page = bt[pg];
              if (page < 0 || page >= p.num_pages) raise_error(p.err, DFLASH_DEVERR_SLOT);
              else y = (page * p.Hkv + h) * 16;
            }
          }
#pragma unroll
          for (int hf = 0; hf < C::kHalves; ++hf) {
            const int off = hf * KT * 128 + j * 2048;
            tma_load_2d(sK(s) + off, &tmK, &kv_full[s], hf * 64, y);
            tma_load_2d(sV(s) + off, &tmV, &kv_full[s], hf * 64, y);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc_bf16(kTcM, KT, false);
      const uint32_t idesc_pv = umma_idesc_bf16(kTcM, D, true);
      bool ok = n_tiles > 0 && mbar_wait(q_full, 0, p.err);
      tc_fence_after();
      auto issue_qk = [&](int t) -> bool {
        const int kv = t % ST, kvu = t / ST;      // K/V ring stage
        const int s = t & 1, u = t >> 1;          // S buffer
        if (!mbar_wait(&kv_full[kv], kvu & 1, p.err)) return false;
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
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int t = 0; ok && t < n_tiles; ++t) {
        // S of tile t+1 goes ahead of P V of tile t when its K/V have landed
        // (its softmax then overlaps P V); otherwise P V(t) is issued first
        // instead of waiting on the load
        const int s1 = (t + 1) & 1, u1 = (t + 1) >> 1;
        const int kv1 = (t + 1) % ST, kvu1 = (t + 1) / ST;
        const bool qk_first = t + 1 < n_tiles && mbar_try_wait(&kv_full[kv1], kvu1 & 1) &&
                              mbar_try_wait(&s_empty[s1], (u1 & 1) ^ 1u);
        if (qk_first && !issue_qk(t + 1)) break;
        const int s = t & 1, u = t >> 1;
        if (!mbar_wait(&p_full[s], u & 1, p.err)) break;
        tc_fence_after();
#pragma unroll
        for (int lohi = 0; lohi < 2; ++lohi) {
#pragma unroll
          for (int kk = 0; kk < KT / 16; ++kk) {
            const int kh = kk >> 2, w = kk & 3;
            const uint64_t ad = umma_desc_sw128(smem_u32(sP(lohi, s) + kh * kTcM * 128 + w * 32));
            const uint64_t bd = umma_desc_sw128_mn(smem_u32(sV(t % ST) + kk * 16 * 128),
                                                   KT * 128, 1024);
            umma_f16kind(tmem_base + C::kOCol, ad, bd, idesc_pv,
                         (t > 0 || lohi > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&kv_empty[t % ST]);
        umma_commit(&p_empty[s]);
        umma_commit(o_ready);
        if (t + 1 == n_tiles) umma_commit(o_final);
        if (!qk_first && t + 1 < n_tiles && !issue_qk(t + 1)) break;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int sp = warp & 3;                    // TMEM sub-partition = 16-row group
    const int tid = threadIdx.x - 64;           // 0..127
    // Q rows r = i * G + g of this kv group -> K-major, 128B-swizzled operand;
    // all of a thread's loads are issued before any store
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
      *reinterpret_cast<uint4*>(sQ + (c >> 3) * kTcM * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4)) =
          qv[u];
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(q_full);

    const uint32_t lane_base = static_cast<uint32_t>(32 * sp) << 16;
    const int r0 = 16 * sp + (lane >> 2);       // this thread's rows r0 and r0 + 8
    float m_ref[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int s = t & 1, u = t >> 1;
      if (!mbar_wait(&s_full[s], u & 1, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[4 * (KT / 8)];
#pragma unroll
      for (int c = 0; c < KT / 64; ++c)
        tmem_ld_16x256b_x8(tmem_base + lane_base + s * KT + c * 64, sv + 32 * c);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[s]);

      const int t0 = k0 + t * KT;
      const int nvalid = min(KT, k1 - t0);
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < KT / 8; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kt = j * 8 + 2 * (lane & 3) + (e & 1);
          const float v = sv[4 * j + e] * p.scale_log2;
          sv[4 * j + e] = (kt < nvalid) ? v : -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], sv[4 * j + e]);
        }
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
      }
      bool need[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        need[hh] = mx[hh] != -INFINITY &&
                   (m_ref[hh] == -INFINITY || mx[hh] > m_ref[hh] + kTcLazyRescale);
      if (__any_sync(0xffffffffu, need[0] || need[1])) {
        float nref[2], alpha[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          nref[hh] = need[hh] ? mx[hh] : m_ref[hh];
          alpha[hh] = (m_ref[hh] == -INFINITY) ? 0.f : exp2f(m_ref[hh] - nref[hh]);
        }
        if (t > 0) {
          // O holds P V of tiles < t against the old reference: rescale it once
          // the previous tile's P V has landed.  (s_full of tile t implies P V
          // of tile t-2 is complete, so o_ready is at most one phase behind and
          // its parity names tile t-1 unambiguously.)
          if (!mbar_wait(o_ready, (t - 1) & 1, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            float ov[32];
            tmem_ld_16x256b_x8(tmem_base + lane_base + C::kOCol + c * 64, ov);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) ov[q] *= alpha[(q >> 1) & 1];
            tmem_st_16x256b_x8(tmem_base + lane_base + C::kOCol + c * 64, ov);
          }
          tmem_st_wait();
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          l_run[hh] *= alpha[hh];
          m_ref[hh] = nref[hh];
        }
      }
      float ref[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) ref[hh] = (m_ref[hh] == -INFINITY) ? 0.f : m_ref[hh];
#pragma unroll
      for (int q = 0; q < 4 * (KT / 8); ++q) {
        const float pv = exp2f(sv[q] - ref[(q >> 1) & 1]);
        sv[q] = pv;
        l_run[(q >> 1) & 1] += pv;
      }
      // the P buffer must be free: P V of the tile that used it has landed
      // (two buffers: tile t-2, via p_empty; one buffer: tile t-1, via o_ready,
      // which is at most one phase behind here)
      const bool p_free = C::kPBufs == 2 ? mbar_wait(&p_empty[s], (u & 1) ^ 1u, p.err)
                          : (t == 0 || mbar_wait(o_ready, (t - 1) & 1, p.err));
      if (!p_free) {
        ok = false;
        break;
      }
      uint8_t* ph = sP(0, s);
      uint8_t* pl = sP(1, s);
#pragma unroll
      for (int j = 0; j < KT / 8; ++j) {
        const int kh = j >> 3, ch = j & 7;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int r = r0 + 8 * hh;
          uint32_t hi, lo;
          split_bf16x2(sv[4 * j + 2 * hh], sv[4 * j + 2 * hh + 1], hi, lo);
          const int off = kh * kTcM * 128 + r * 128 + ((ch ^ (r & 7)) << 4) + (lane & 3) * 4;
          *reinterpret_cast<uint32_t*>(ph + off) = hi;
          *reinterpret_cast<uint32_t*>(pl + off) = lo;
        }
      }
      if (sp == 0 && (nvalid & 15)) {
        // rows past the last key of a partly used page may hold anything
        // (NaN patterns included): zero them so that P = 0 rows add 0
        const int jp = nvalid >> 4, rr0 = nvalid & 15;
        const int n16 = (16 - rr0) * C::kHalves * 8;
        for (int e = lane; e < n16; e += 32) {
          const int hf = e / ((16 - rr0) * 8);
          const int rem = e - hf * (16 - rr0) * 8;
          const int rr = rr0 + rem / 8, cc = rem & 7;
          *reinterpret_cast<uint4*>(sV(t % ST) + hf * KT * 128 + jp * 2048 + rr * 128 +
                                    cc * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[s]);
    }

    if (p.cluster) {
      // keep this split's unnormalised O rows and (m, l) in registers for the
      // push below (every TMA load and MMA of the CTA has completed once
      // o_final fired)
      have = ok && n_tiles > 0 && mbar_wait(o_final, 0, p.err);
#pragma unroll
      for (int db = 0; db < D / 8; ++db)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[db][e] = 0.f;
      if (have) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          float ov[32];
          tmem_ld_16x256b_x8(tmem_base + lane_base + C::kOCol + c * 64, ov);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[c * 8 + jj][e] = ov[4 * jj + e];
        }
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 1);
        l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 2);
        m_fin[hh] = have ? m_ref[hh] : -INFINITY;
        l_fin[hh] = have ? l_run[hh] : 0.f;
      }
    } else if (ok && mbar_wait(o_final, 0, p.err)) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        float ov[32];
        tmem_ld_16x256b_x8(tmem_base + lane_base + C::kOCol + c * 64, ov);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[c * 8 + jj][e] = ov[4 * jj + e];
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 1);
        l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 2);
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = r0 + hh * 8;
        if (r >= p.R) continue;
        if (n_splits_b == 1) {
          const int i = r / p.G, g = r - (r / p.G) * p.G;
          f16* dst = p.o + (static_cast<size_t>(b * p.bs + i) * p.Hq + h * p.G + g) * D;
          const float inv = 1.f / l_run[hh];
#pragma unroll
          for (int db = 0; db < D / 8; ++db) {
            const int d = db * 8 + 2 * (lane & 3);
            *reinterpret_cast<uint32_t*>(dst + d) =
                pack_f16x2(o[db][2 * hh] * inv, o[db][2 * hh + 1] * inv);
          }
        } else {
          const size_t prow = (static_cast<size_t>(split) * p.B + b) * p.Hkv + h;
          float* dst = p.part_o + (prow * p.R + r) * D;
#pragma unroll
          for (int db = 0; db < D / 8; ++db) {
            const int d = db * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2*>(dst + d) = make_float2(o[db][2 * hh], o[db][2 * hh + 1]);
          }
          if ((lane & 3) == 0) {
            *reinterpret_cast<float2*>(p.part_ml + (prow * p.R + r) * 2) =
                make_float2(m_ref[hh], l_run[hh]);
          }
        }
      }
    }
  }

  if (p.cluster) {
    const int S = p.max_splits;
    const int q = static_cast<int>(cluster_rank());
    cluster_sync();  // every CTA of the cluster is done with its K/V ring
    if (warp >= 2) {
      float* recv = reinterpret_cast<float*>(smem);                  // [slot][D + 8]
      float2* recv_ml = reinterpret_cast<float2*>(smem + C::kCombOffML);
      const int r0 = 16 * (warp & 3) + (lane >> 2);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = r0 + 8 * hh;
        if (r >= p.R) continue;
        const uint32_t owner = static_cast<uint32_t>(r % S);
        const int slot = (r / S) * S + q;
#pragma unroll
        for (int db = 0; db < D / 8; ++db) {
          const int d = db * 8 + 2 * (lane & 3);
          st_peer_f2(recv + slot * (D + 8) + d, owner, o[db][2 * hh], o[db][2 * hh + 1]);
        }
        if ((lane & 3) == 0) st_peer_f2(recv_ml + slot, owner, m_fin[hh], l_fin[hh]);
      }
    }
    cluster_sync();  // every push has landed
    if (warp >= 2) {
      const float* recv = reinterpret_cast<const float*>(smem);
      const float2* recv_ml = reinterpret_cast<const float2*>(smem + C::kCombOffML);
      const int tid = threadIdx.x - 64;
      const int my_rows = (p.R - q + S - 1) / S;  // rows q, q + S, ...
      for (int item = tid; item < my_rows * (D / 4); item += 128) {
        const int lr = item / (D / 4), d = (item - lr * (D / 4)) * 4;
        const int r = q + lr * S;
        float M = -INFINITY;
        for (int src = 0; src < S; ++src) M = fmaxf(M, recv_ml[lr * S + src].x);
        float L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int src = 0; src < S; ++src) {
          const float2 ml = recv_ml[lr * S + src];
          const float w = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
          L += w * ml.y;
          const float4 t = *reinterpret_cast<const float4*>(recv + (lr * S + src) * (D + 8) + d);
          acc.x += w * t.x;
          acc.y += w * t.y;
          acc.z += w * t.z;
          acc.w += w * t.w;
        }
        const float inv = 1.f / L;
        const int i = r / p.G, g = r - (r / p.G) * p.G;
        f16* dst = p.o + (static_cast<size_t>(b * p.bs + i) * p.Hq + h * p.G + g) * D + d;
        *reinterpret_cast<uint2*>(dst) =
            make_uint2(pack_f16x2(acc.x * inv, acc.y * inv), pack_f16x2(acc.z * inv, acc.w * inv));
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


// ---------------------------------------------------------------------------
// Persistent variant of the 64-key, six-deep-ring kernel: gridDim.x CTAs (one
// per SM) walk the (key split, kv head, request) items in the order of the
// non-persistent grid (split fastest), CTA c taking items c, c + gridDim.x, ...
// Every ring, S/P buffer and O barrier runs on a tile counter that continues
// across items, so the producer streams the next item's K/V while the softmax
// warps finish the previous item: the softmax warps load the next item's Q as
// soon as the MMA warp has issued the current item's last S (q_empty), then
// write the current item's output, then start the next item's tiles.  The
// barrier / TMEM set-up is paid once per CTA instead of once per item.  No
// cluster mode.  Same results as attn_block_tc_kernel<D, 64, ST> item by item.
// ---------------------------------------------------------------------------
template <int D, int ST>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_block_tc_persistent_kernel(const __grid_constant__ CUtensorMap tmK,
                                    const __grid_constant__ CUtensorMap tmV,
                                    const AttnParams p) {
  constexpr int KT = kTcKeysSmall;
  using C = TcAttnCfg<D, KT, ST>;
  static_assert(C::kPBufs == 1, "one P buffer");
  pdl_trigger();
  pdl_wait();
  const int n_items = p.max_splits * p.Hkv * p.B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // item -> (split, head, request, key range); false when it has no keys
  auto item_at = [&](int it, int& split, int& h, int& b, int& k0, int& k1, int& n_tiles) {
    split = it % p.max_splits;
    const int r = it / p.max_splits;
    h = r % p.Hkv;
    b = r / p.Hkv;
    const int n_keys = p.seq_lens[b] + p.bs;
    k0 = split * p.chunk_keys;
    k1 = min(n_keys, k0 + p.chunk_keys);
    n_tiles = k0 < n_keys ? (k1 - k0 + KT - 1) / KT : 0;
    return n_tiles > 0;
  };

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;        // [ST] K/V ring (tile g -> stage g % ST)
  uint64_t* kv_empty = bars + 8;   // [ST]
  uint64_t* s_full = bars + 16;    // [2] S buffers (tile g -> g % 2)
  uint64_t* s_empty = bars + 18;   // [2]
  uint64_t* p_full = bars + 20;    // [2] (one P buffer: barrier g % 2 of it)
  uint64_t* o_ready = bars + 24;   // one phase per tile: P V of that tile landed
  uint64_t* q_full = bars + 25;    // one phase per item: its Q is in shared memory
  uint64_t* o_final = bars + 26;   // one phase per item: its last P V landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 27);
  uint64_t* q_empty = bars + 28;   // one phase per item: its last S was issued and ran
  auto sK = [&](int s) { return smem + s * C::kKVBytes; };
  auto sV = [&](int s) { return smem + C::kOffV + s * C::kKVBytes; };
  uint8_t* sPh = smem + C::kOffP;
  uint8_t* sPl = smem + C::kOffP + C::kPBytes;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4);
    }
    mbar_init(o_ready, 1);
    mbar_init(q_full, 4);
    mbar_init(o_final, 1);
    mbar_init(q_empty, 1);
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
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      uint32_t g = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        int split, h, b, k0, k1, n_tiles;
        if (!item_at(it, split, h, b, k0, k1, n_tiles)) continue;
        const int* bt = p.block_table + static_cast<size_t>(b) * p.W;
        for (int t = 0; t < n_tiles; ++t, ++g) {
          const int s = static_cast<int>(g % ST);
          const uint32_t u = g / ST;
          if (!mbar_wait(&kv_empty[s], (u & 1) ^ 1u, p.err)) {
            ok = false;
            break;
          }
          const int t0 = k0 + t * KT;
          const int nvalid = min(KT, k1 - t0);
          const int npages = (nvalid + 15) >> 4;
          mbar_arrive_expect_tx(&kv_full[s],
                                static_cast<uint32_t>((KT / 16) * C::kHalves * 2048 * 2));
          for (int j = 0; j < KT / 16; ++j) {
            int y = -16;  // pages past the range: fully out of bounds, TMA fills zeros
            if (j < npages) {
              const int pg = (t0 >> 4) + j;
              if (pg >= p.W) {
                raise_error(p.err, DFLASH_DEVERR_TABLE);
              } else {
                const int page = bt[pg];
                if (page < 0 || page >= p.num_pages) raise_error(p.err, DFLASH_DEVERR_SLOT);
                else y = (page * p.Hkv + h) * 16;
              }
            }
#pragma unroll
            for (int hf = 0; hf < C::kHalves; ++hf) {
              const int off = hf * KT * 128 + j * 2048;
              tma_load_2d(sK(s) + off, &tmK, &kv_full[s], hf * 64, y);
              tma_load_2d(sV(s) + off, &tmV, &kv_full[s], hf * 64, y);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc_bf16(kTcM, KT, false);
      const uint32_t idesc_pv = umma_idesc_bf16(kTcM, D, true);
      uint32_t g = 0, q_phase = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        int split, h, b, k0, k1, n_tiles;
        if (!item_at(it, split, h, b, k0, k1, n_tiles)) continue;
        if (!mbar_wait(q_full, q_phase & 1, p.err)) break;
        ++q_phase;
        tc_fence_after();
        const uint32_t g0 = g;
        // S of the item's tile t; the item's last S also releases its Q
        auto issue_qk = [&](int t) -> bool {
          const uint32_t gt = g0 + t;
          const int kv = static_cast<int>(gt % ST);
          const uint32_t kvu = gt / ST;
          const int s = static_cast<int>(gt & 1);
          const uint32_t u = gt >> 1;
          if (!mbar_wait(&kv_full[kv], kvu & 1, p.err)) return false;
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
          if (t == n_tiles - 1) umma_commit(q_empty);
          return true;
        };
        ok = issue_qk(0);
        for (int t = 0; ok && t < n_tiles; ++t) {
          const uint32_t gt = g0 + t, g1 = gt + 1;
          const bool qk_first = t + 1 < n_tiles &&
                                mbar_try_wait(&kv_full[g1 % ST], (g1 / ST) & 1) &&
                                mbar_try_wait(&s_empty[g1 & 1], ((g1 >> 1) & 1) ^ 1u);
          if (qk_first && !issue_qk(t + 1)) {
            ok = false;
            break;
          }
          const int s = static_cast<int>(gt & 1);
          if (!mbar_wait(&p_full[s], (gt >> 1) & 1, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int kv = static_cast<int>(gt % ST);
#pragma unroll
          for (int lohi = 0; lohi < 2; ++lohi) {
#pragma unroll
            for (int kk = 0; kk < KT / 16; ++kk) {
              const int kh = kk >> 2, w = kk & 3;
              const uint64_t ad =
                  umma_desc_sw128(smem_u32((lohi ? sPl : sPh) + kh * kTcM * 128 + w * 32));
              const uint64_t bd = umma_desc_sw128_mn(smem_u32(sV(kv) + kk * 16 * 128),
                                                     KT * 128, 1024);
              umma_f16kind(tmem_base + C::kOCol, ad, bd, idesc_pv,
                           (t > 0 || lohi > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&kv_empty[kv]);
          umma_commit(o_ready);
          if (t + 1 == n_tiles) umma_commit(o_final);
          if (!qk_first && t + 1 < n_tiles && !issue_qk(t + 1)) {
            ok = false;
            break;
          }
        }
        g += n_tiles;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int sp = warp & 3;                    // TMEM sub-partition = 16-row group
    const int tid = threadIdx.x - 64;           // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(32 * sp) << 16;
    const int r0 = 16 * sp + (lane >> 2);       // this thread's rows r0 and r0 + 8
    // Q rows r = i * G + g of item (h, b) -> K-major, 128B-swizzled operand
    auto load_q = [&](int h, int b) {
      constexpr int kQPer = kTcM * (D / 8) / 128;
      uint4 qv[kQPer];
#pragma unroll
      for (int u = 0; u < kQPer; ++u) {
        const int e = tid + u * 128;
        const int r = e / (D / 8), c = e - r * (D / 8);
        qv[u] = make_uint4(0, 0, 0, 0);
        if (r < p.R) {
          const int i = r / p.G, gq = r - (r / p.G) * p.G;
          const bf16* src = p.q + (static_cast<size_t>(b * p.bs + i) * p.Hq + h * p.G + gq) * D;
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
    };
    // the next item with keys at or after `it` (n_items if none)
    auto next_item = [&](int it) {
      int split, h, b, k0, k1, n_tiles;
      while (it < n_items && !item_at(it, split, h, b, k0, k1, n_tiles)) it += gridDim.x;
      return it;
    };

    uint32_t g = 0, item_phase = 0;
    bool ok = true;
    int it = next_item(blockIdx.x);
    if (it < n_items) {
      int split, h, b, k0, k1, n_tiles;
      item_at(it, split, h, b, k0, k1, n_tiles);
      load_q(h, b);
    }
    while (ok && it < n_items) {
      int split, h, b, k0, k1, n_tiles;
      item_at(it, split, h, b, k0, k1, n_tiles);
      const int n_keys = p.seq_lens[b] + p.bs;
      const int n_splits_b = (n_keys + p.chunk_keys - 1) / p.chunk_keys;
      float m_ref[2] = {-INFINITY, -INFINITY};
      float l_run[2] = {0.f, 0.f};
      for (int t = 0; t < n_tiles; ++t) {
        const uint32_t gt = g + t;
        const int s = static_cast<int>(gt & 1);
        if (!mbar_wait(&s_full[s], (gt >> 1) & 1, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float sv[4 * (KT / 8)];
        tmem_ld_16x256b_x8(tmem_base + lane_base + s * KT, sv);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[s]);

        const int t0 = k0 + t * KT;
        const int nvalid = min(KT, k1 - t0);
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < KT / 8; ++j) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int kt = j * 8 + 2 * (lane & 3) + (e & 1);
            const float v = sv[4 * j + e] * p.scale_log2;
            sv[4 * j + e] = (kt < nvalid) ? v : -INFINITY;
            mx[e >> 1] = fmaxf(mx[e >> 1], sv[4 * j + e]);
          }
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
          mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
        }
        bool need[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          need[hh] = mx[hh] != -INFINITY &&
                     (m_ref[hh] == -INFINITY || mx[hh] > m_ref[hh] + kTcLazyRescale);
        if (__any_sync(0xffffffffu, need[0] || need[1])) {
          float nref[2], alpha[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            nref[hh] = need[hh] ? mx[hh] : m_ref[hh];
            alpha[hh] = (m_ref[hh] == -INFINITY) ? 0.f : exp2f(m_ref[hh] - nref[hh]);
          }
          if (t > 0) {
            // O holds this item's P V of tiles < t: rescale it once the
            // previous tile's P V has landed (o_ready is at most one phase
            // behind, so its parity names tile gt - 1)
            if (!mbar_wait(o_ready, (gt - 1) & 1, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              float ov[32];
              tmem_ld_16x256b_x8(tmem_base + lane_base + C::kOCol + c * 64, ov);
              tmem_ld_wait();
#pragma unroll
              for (int q = 0; q < 32; ++q) ov[q] *= alpha[(q >> 1) & 1];
              tmem_st_16x256b_x8(tmem_base + lane_base + C::kOCol + c * 64, ov);
            }
            tmem_st_wait();
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            l_run[hh] *= alpha[hh];
            m_ref[hh] = nref[hh];
          }
        }
        float ref[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) ref[hh] = (m_ref[hh] == -INFINITY) ? 0.f : m_ref[hh];
#pragma unroll
        for (int q = 0; q < 4 * (KT / 8); ++q) {
          const float pv = exp2f(sv[q] - ref[(q >> 1) & 1]);
          sv[q] = pv;
          l_run[(q >> 1) & 1] += pv;
        }
        // the P buffer is free once P V of the previous tile (any item) landed
        if (gt > 0 && !mbar_wait(o_ready, (gt - 1) & 1, p.err)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int j = 0; j < KT / 8; ++j) {
          const int kh = j >> 3, ch = j & 7;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int r = r0 + 8 * hh;
            uint32_t hi, lo;
            split_bf16x2(sv[4 * j + 2 * hh], sv[4 * j + 2 * hh + 1], hi, lo);
            const int off = kh * kTcM * 128 + r * 128 + ((ch ^ (r & 7)) << 4) + (lane & 3) * 4;
            *reinterpret_cast<uint32_t*>(sPh + off) = hi;
            *reinterpret_cast<uint32_t*>(sPl + off) = lo;
          }
        }
        if (sp == 0 && (nvalid & 15)) {
          // rows past the last key of a partly used page may hold anything
          // (NaN patterns included): zero them so that P = 0 rows add 0
          const int jp = nvalid >> 4, rr0 = nvalid & 15;
          const int n16 = (16 - rr0) * C::kHalves * 8;
          for (int e = lane; e < n16; e += 32) {
            const int hf = e / ((16 - rr0) * 8);
            const int rem = e - hf * (16 - rr0) * 8;
            const int rr = rr0 + rem / 8, cc = rem & 7;
            *reinterpret_cast<uint4*>(sV(static_cast<int>(gt % ST)) + hf * KT * 128 + jp * 2048 +
                                      rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[s]);
      }
      if (!ok) break;
      g += n_tiles;
      // the next item's Q, as soon as this item's last S has run
      const int nxt = next_item(it + gridDim.x);
      if (nxt < n_items) {
        if (!mbar_wait(q_empty, item_phase & 1, p.err)) break;
        int s2, h2, b2, a0, a1, nt2;
        item_at(nxt, s2, h2, b2, a0, a1, nt2);
        load_q(h2, b2);
      }
      // this item's output
      if (!mbar_wait(o_final, item_phase & 1, p.err)) break;
      ++item_phase;
      tc_fence_after();
      float o[D / 8][4];
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        float ov[32];
        tmem_ld_16x256b_x8(tmem_base + lane_base + C::kOCol + c * 64, ov);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[c * 8 + jj][e] = ov[4 * jj + e];
      }
      tc_fence_before();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 1);
        l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 2);
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = r0 + hh * 8;
        if (r >= p.R) continue;
        if (n_splits_b == 1) {
          const int i = r / p.G, gq = r - (r / p.G) * p.G;
          f16* dst = p.o + (static_cast<size_t>(b * p.bs + i) * p.Hq + h * p.G + gq) * D;
          const float inv = 1.f / l_run[hh];
#pragma unroll
          for (int db = 0; db < D / 8; ++db) {
            const int d = db * 8 + 2 * (lane & 3);
            *reinterpret_cast<uint32_t*>(dst + d) =
                pack_f16x2(o[db][2 * hh] * inv, o[db][2 * hh + 1] * inv);
          }
        } else {
          const size_t prow = (static_cast<size_t>(split) * p.B + b) * p.Hkv + h;
          float* dst = p.part_o + (prow * p.R + r) * D;
#pragma unroll
          for (int db = 0; db < D / 8; ++db) {
            const int d = db * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2*>(dst + d) = make_float2(o[db][2 * hh], o[db][2 * hh + 1]);
          }
          if ((lane & 3) == 0) {
            *reinterpret_cast<float2*>(p.part_ml + (prow * p.R + r) * 2) =
                make_float2(m_ref[hh], l_run[hh]);
          }
        }
      }
      it = nxt;
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
