// gemm_tcgen05.cuh — persistent, warp-specialised bf16 GEMM for sm_100a with
// fused epilogues.
//
//   D[m, n] = sum_k A[m, k] * W[n, k]      A: [M, K], W: [N, K], both K-major and both
//                                          fp16 or both bf16; fp32 accumulation
//
// Tile 128 x BN x 64.  Warp 0 streams A and W tiles with TMA (128-byte swizzle)
// into a ring of shared-memory stages; warp 1 issues tcgen05.mma (M=128, N=BN,
// K=16, one thread) into a double-buffered fp32 accumulator in tensor memory;
// warps 2..5 drain the accumulator with tcgen05.ld and run the epilogue functor
// while the next tile accumulates.  A tile's K=16 steps are spread over `nacc`
// independent accumulator chains (summed in chain order by the epilogue) so
// that narrow, weight-streaming tiles are not paced by the latency of one
// dependent MMA chain.
//
// Scheduling: whole tiles round-robin over one CTA per SM when there are
// enough of them to fill the GPU evenly; for a few rows (the staged epilogue)
// and fewer tiles than SMs, cluster split-K — the S CTAs of a thread-block
// cluster share one tile, each taking 1/S of its k-blocks, and reduce the
// pieces through distributed shared memory (no global partials, no fence, no
// arrival counter); otherwise stream-K — every CTA takes an equal contiguous
// range of the (tile, k-block) iteration space, so every SM streams weights.  A tile split across CTAs has each piece written as an
// fp32 partial (at most two slots per CTA); the CTA that finishes the tile's
// last piece (a per-tile arrival counter, no waiting) sums the pieces in CTA
// order — so the result is deterministic — and runs the epilogue.  The
// counters are left at zero.
//
// Every pipeline wait is bounded (see mbar_wait); a wait that runs out sets the
// timeout bit and the CTA winds down, frees its tensor memory and returns.
#pragma once

#include "dflash_device.cuh"

namespace dflash {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmThreads = 192;
constexpr int kGemmSmemLimit = 232448;  // max dynamic shared memory per block on sm_100

constexpr int kGemmMaxStages = 32;
// full/empty per stage, tfull/tempty per accumulator, then 4 words: TMEM base,
// last-arriver flag and the two epilogue wait verdicts
constexpr int kGemmBarrierBytes = 2 * kGemmMaxStages * 8 + 4 * 8 + 16;

template <int BN>
struct GemmCfg {
  static constexpr int kBBytes = BN * kGemmBK * 2;
  static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "UMMA N for M=128");
};

// Tiles of at most this many rows (M <= 32) take the staged epilogue: one warp
// copies the accumulator from tensor memory into a shared-memory tile, then all
// 128 epilogue threads run the stream-K fixup and the epilogue functor over it,
// so that a handful of rows does not leave 3/4 of the threads idle and the
// rest walking the tile with one dependent global round trip per step.
constexpr int kGemmStagedRows = 32;

__host__ __device__ inline bool gemm_staged(int a_rows) { return a_rows <= kGemmStagedRows; }

// fp32 staging tile [a_rows][bn + 4] (the pad spreads rows over the banks)
__host__ __device__ inline int gemm_staging_bytes(int a_rows, int bn) {
  return gemm_staged(a_rows) ? a_rows * (bn + 4) * 4 : 0;
}

// Shared memory of one launch: [a_rows x 128 B A slots][BN x 128 B W slots]
// [barriers][staging tile].  With fewer than 128 rows of A (a_rows < 128) the
// MMA still reads a full 128-row A operand; the rows past a_rows alias the
// following slots, which only feeds accumulator rows that the epilogue never
// stores.
__host__ __device__ inline int gemm_smem_bytes(int a_rows, int bn, int stages) {
  const int tail = kGemmBM * 128 - a_rows * 128 - stages * bn * 128;  // keep A overreads inside
  return 1024 + stages * (a_rows + bn) * 128 + kGemmBarrierBytes +
         gemm_staging_bytes(a_rows, bn) + (tail > 0 ? tail : 0);
}

struct GemmParams {
  int M, N, K;
  int m_tiles, n_tiles, k_blocks;
  int tiles;           // m_tiles * n_tiles
  int stream_k;        // 0: whole tiles round-robin; 1: equal ranges of (tile, k-block) iterations
  int cluster_s;       // > 1: cluster split-K, S CTAs per tile (grid = tiles * S, cluster S x 1 x 1)
  int ipc;             // stream-K: k-block iterations per CTA
  int total_iters;     // stream-K: tiles * k_blocks
  int nacc;            // independent accumulator chains per tile (1, 2 or 4)
  int nbuf;            // accumulator buffers (2: next tile accumulates during the epilogue)
  int tmem_cols;       // allocated TMEM columns (>= nbuf * nacc * BN, power of two)
  int a_rows;          // rows of the A box / slot (128, or M rounded up to 16 when M < 128)
  int stages;          // pipeline depth (<= kGemmMaxStages)
  int f16;             // operands are fp16 (1) or bf16 (0)
  int w_packed;        // W in the tile-contiguous layout (BN = 256 row chunks), else row-major
  int slot_rows;       // rows held per partial slot (min(M, 128))
  float* partials;     // stream-K: [gridDim.x * 2][slot_rows][BN] fp32
  unsigned* counters;  // [tiles], zero on entry, zero on exit
  unsigned* err;
};

// One contiguous piece of one output tile's K range, as processed by one CTA.
struct GemmSeg {
  int tile, m_tile, n_tile, kb0, kb1;
  int first_cta, nseg;  // CTAs contributing to this tile (stream-K), 1 for whole tiles
  int slot;             // this CTA's partial slot for the tile when nseg > 1
};

// Iterates the segments of this CTA.  Every warp role walks the same sequence.
struct GemmSegIter {
  int cur, end, step;
  __device__ __forceinline__ explicit GemmSegIter(const GemmParams& p) {
    if (p.cluster_s > 1) {
      cur = blockIdx.x;  // one segment: this CTA's share of tile blockIdx.x / S
      end = blockIdx.x + 1;
      step = 1;
    } else if (p.stream_k) {
      cur = blockIdx.x * p.ipc;
      end = min(p.total_iters, cur + p.ipc);
      step = 0;
    } else {
      cur = blockIdx.x;
      end = p.tiles;
      step = gridDim.x;
    }
  }
  __device__ __forceinline__ bool next(const GemmParams& p, GemmSeg& s) {
    if (cur >= end) return false;
    if (p.cluster_s > 1) {
      const int S = p.cluster_s;
      s.tile = cur / S;
      const int rank = cur - s.tile * S;
      s.kb0 = rank * p.k_blocks / S;
      s.kb1 = (rank + 1) * p.k_blocks / S;
      s.first_cta = s.tile * S;
      s.nseg = 1;  // reduced through the cluster, not through global partials
      s.slot = 0;
      cur += 1;
    } else if (p.stream_k) {
      s.tile = cur / p.k_blocks;
      s.kb0 = cur - s.tile * p.k_blocks;
      s.kb1 = min(p.k_blocks, s.kb0 + (end - cur));
      const int tile_beg = s.tile * p.k_blocks;
      s.first_cta = tile_beg / p.ipc;
      s.nseg = (tile_beg + p.k_blocks - 1) / p.ipc - s.first_cta + 1;
      s.slot = blockIdx.x * 2 + (cur == static_cast<int>(blockIdx.x) * p.ipc ? 0 : 1);
      cur += s.kb1 - s.kb0;
    } else {
      s.tile = cur;
      s.kb0 = 0;
      s.kb1 = p.k_blocks;
      s.first_cta = 0;
      s.nseg = 1;
      s.slot = 0;
      cur += step;
    }
    s.n_tile = s.tile / p.m_tiles;
    s.m_tile = s.tile - s.n_tile * p.m_tiles;
    return true;
  }
};

// Partial slot that CTA c used for `tile` (the slot index rule of GemmSegIter).
__device__ __forceinline__ int gemm_slot_of(const GemmParams& p, int tile, int c) {
  const int seg_beg = max(tile * p.k_blocks, c * p.ipc);
  return c * 2 + (seg_beg == c * p.ipc ? 0 : 1);
}

// Sum of the nacc accumulator chains for 32 columns at TMEM address taddr
// (chains BN columns apart), in chain order.
template <int BN>
__device__ __forceinline__ void tmem_load_sum32(uint32_t taddr, int nacc, float* v) {
  tmem_ld_32x32b_x32(taddr, v);
  tmem_ld_wait();
  for (int j = 1; j < nacc; ++j) {
    float t[32];
    tmem_ld_32x32b_x32(taddr + j * BN, t);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] += t[i];
  }
}

// Coordinates of the W box of (n_tile, k-block kb): row-major W is addressed by
// (k, row); the tile-contiguous layout stores each 256 x 64 tile as one chunk
// of 256 consecutive 128-byte rows, so a BN-row tile (BN dividing 256) is a
// contiguous part of one chunk.
__device__ __forceinline__ int w_x(const GemmParams& p, int kb) {
  return p.w_packed ? 0 : kb * kGemmBK;
}
template <int BN>
__device__ __forceinline__ int w_y(const GemmParams& p, int n_tile, int kb) {
  static_assert(256 % BN == 0, "tile width divides the packed chunk");
  const int row0 = n_tile * BN;
  return p.w_packed ? ((row0 >> 8) * p.k_blocks + kb) * 256 + (row0 & 255) : row0;
}

// Shared-memory carve-up, barriers and tensor-memory base of one CTA, common
// to every phase of a launch.
template <int BN>
struct GemmCta {
  uint8_t* sA;
  uint8_t* sB;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint32_t* tmem_slot;
  volatile int* last_flag;
  // [2]: verdict of the elected epilogue wait, alternating by segment (a
  // thread can be at most one segment ahead of the slowest reader)
  volatile int* wait_flag;
  float* staging;
  int stages;
  int a_bytes;
  uint32_t stage_tx;
  uint32_t tmem_base;
  int acc_cols;   // TMEM columns of one accumulator buffer
};

// Ring positions of the producer / MMA thread and of the epilogue, carried
// from one phase of a launch to the next.
struct GemmRing {
  uint32_t stage = 0, phase = 0;
  bool ok = true;
};
struct GemmAccRing {
  uint32_t acc = 0, acc_phase = 0, nseen = 0;
  bool ok = true;
};

// Bounded wait until *ctr >= target (acquire): the arrival count of the CTAs
// of this launch that finished an earlier phase.  Gives up like mbar_wait.
__device__ __forceinline__ bool wait_count(const unsigned* ctr, unsigned target, unsigned* err) {
  const long long t0 = clock64();
  for (unsigned spin = 0;; ++spin) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if ((spin & 63u) == 63u) {
      if (clock64() - t0 > *reinterpret_cast<volatile long long*>(&g_wait_limit_cycles)) {
        raise_error(err, DFLASH_DEVERR_TIMEOUT);
        return false;
      }
      if (err && (*reinterpret_cast<volatile unsigned*>(err) & DFLASH_DEVERR_TIMEOUT)) return false;
    }
    __nanosleep(64);
  }
}

// Barrier init, the first weight stages of phase `p0` (thread 0), tensor-memory
// allocation (warp 1) and the CTA barrier.  Returns the carve-up; `pre` = the
// k-blocks of p0 whose W tile thread 0 has requested.
template <int BN>
__device__ __forceinline__ GemmCta<BN> gemm_setup(const GemmParams& p0, const CUtensorMap* tA,
                                                  const CUtensorMap* tW, int& pre) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  GemmCta<BN> S;
  S.stages = p0.stages;
  S.a_bytes = p0.a_rows * 128;
  S.stage_tx = static_cast<uint32_t>(S.a_bytes + C::kBBytes);
  S.sA = smem;
  S.sB = smem + S.stages * S.a_bytes;
  S.full = reinterpret_cast<uint64_t*>(S.sB + S.stages * C::kBBytes);
  S.empty = S.full + kGemmMaxStages;
  S.tfull = S.empty + kGemmMaxStages;
  S.tempty = S.tfull + 2;
  S.tmem_slot = reinterpret_cast<uint32_t*>(S.tempty + 2);
  S.last_flag = reinterpret_cast<volatile int*>(S.tmem_slot + 1);
  S.wait_flag = reinterpret_cast<volatile int*>(S.tmem_slot + 2);
  S.staging = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(S.full) + kGemmBarrierBytes);
  S.acc_cols = p0.nacc * BN;
  const int warp = threadIdx.x >> 5;
  // The weights are never written by an earlier kernel: thread 0 (the TMA
  // producer) requests the W tiles of the first `stages` k-blocks right after
  // the barriers exist — before the tensor-memory allocation, which may wait
  // for a co-resident CTA of the previous kernel to free its columns, and
  // before waiting for the grid that produces A.  Fresh stages need no
  // empty-slot wait.
  pre = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S.stages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&S.tfull[a], 1);
      mbar_init(&S.tempty[a], 4);
    }
    fence_barrier_init();
    tma_prefetch_desc(tA);
    tma_prefetch_desc(tW);
    const uint64_t pol_w = policy_evict_first();
    GemmSegIter it0(p0);
    GemmSeg s0;
    while (pre < S.stages && it0.next(p0, s0)) {
      for (int kb = s0.kb0; kb < s0.kb1 && pre < S.stages; ++kb, ++pre) {
        mbar_arrive_expect_tx(&S.full[pre], S.stage_tx);
        tma_load_2d_hint(S.sB + pre * C::kBBytes, tW, &S.full[pre], w_x(p0, kb),
                         w_y<BN>(p0, s0.n_tile, kb), pol_w);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(S.tmem_slot, static_cast<uint32_t>(p0.tmem_cols));
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  S.tmem_base = *S.tmem_slot;
  return S;
}

// TMA producer (one thread), one phase.  The W tiles of the first `pre`
// k-blocks were already requested (with the whole stage's byte count).  With
// `dep`, the phase's A operand is written by an earlier phase of the same
// launch: the producer first requests the W tiles of as many k-blocks as there
// are free stages, then waits (bounded) until `dep_target` CTAs have arrived
// on *dep, then loads A (after a proxy fence, since A was written by other
// CTAs through the generic proxy and is read here by TMA).
template <int BN>
__device__ void gemm_produce(const GemmParams& q, const CUtensorMap* tA, const CUtensorMap* tW,
                             const GemmCta<BN>& S, GemmRing& R, int pre, const unsigned* dep,
                             unsigned dep_target) {
  using C = GemmCfg<BN>;
  const uint64_t pol_w = policy_evict_first();
  const uint64_t pol_a = policy_evict_last();
  if (dep) {
    GemmSegIter it0(q);
    GemmSeg s0;
    uint32_t stage = R.stage, phase = R.phase;
    pre = 0;
    while (R.ok && pre < S.stages && it0.next(q, s0)) {
      for (int kb = s0.kb0; kb < s0.kb1 && pre < S.stages; ++kb, ++pre) {
        if (!mbar_wait(&S.empty[stage], phase ^ 1u, q.err)) {
          R.ok = false;
          break;
        }
        mbar_arrive_expect_tx(&S.full[stage], S.stage_tx);
        tma_load_2d_hint(S.sB + stage * C::kBBytes, tW, &S.full[stage], w_x(q, kb),
                         w_y<BN>(q, s0.n_tile, kb), pol_w);
        if (++stage == static_cast<uint32_t>(S.stages)) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (R.ok && !wait_count(dep, dep_target, q.err)) R.ok = false;
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  int idx = 0;
  GemmSegIter it(q);
  GemmSeg sg;
  while (R.ok && it.next(q, sg)) {
    for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++idx) {
      if (idx >= pre) {
        if (!mbar_wait(&S.empty[R.stage], R.phase ^ 1u, q.err)) {
          R.ok = false;
          break;
        }
        mbar_arrive_expect_tx(&S.full[R.stage], S.stage_tx);
        tma_load_2d_hint(S.sB + R.stage * C::kBBytes, tW, &S.full[R.stage], w_x(q, kb),
                         w_y<BN>(q, sg.n_tile, kb), pol_w);
      }
      tma_load_2d_hint(S.sA + R.stage * S.a_bytes, tA, &S.full[R.stage], kb * kGemmBK,
                       sg.m_tile * kGemmBM, pol_a);
      if (++R.stage == static_cast<uint32_t>(S.stages)) {
        R.stage = 0;
        R.phase ^= 1u;
      }
    }
  }
}

// MMA issuer (one thread), one phase.
template <int BN>
__device__ void gemm_mma(const GemmParams& q, const GemmCta<BN>& S, GemmRing& R,
                         GemmAccRing& A) {
  using C = GemmCfg<BN>;
  const uint32_t idesc = umma_idesc_f32acc(kGemmBM, BN, q.f16 != 0);
  GemmSegIter it(q);
  GemmSeg sg;
  while (R.ok && it.next(q, sg)) {
    if (!mbar_wait(&S.tempty[A.acc], A.acc_phase ^ 1u, q.err)) {
      R.ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t d_base = S.tmem_base + A.acc * S.acc_cols;
    int t = 0;   // K=16 step index within the segment; chain = t % nacc
    for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
      if (!mbar_wait(&S.full[R.stage], R.phase, q.err)) {
        R.ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t adesc = umma_desc_sw128(smem_u32(S.sA + R.stage * S.a_bytes));
      const uint64_t bdesc = umma_desc_sw128(smem_u32(S.sB + R.stage * C::kBBytes));
#pragma unroll
      for (int k = 0; k < kGemmBK / 16; ++k, ++t) {
        // +32 bytes along K inside the 128-byte swizzle atom = +2 in the
        // descriptor's (address >> 4) field
        const int chain = t % q.nacc;
        umma_f16kind(d_base + chain * BN, adesc + 2 * k, bdesc + 2 * k, idesc,
                     t >= q.nacc ? 1u : 0u);
      }
      umma_commit(&S.empty[R.stage]);
      if (++R.stage == static_cast<uint32_t>(S.stages)) {
        R.stage = 0;
        R.phase ^= 1u;
      }
    }
    if (!R.ok) break;
    umma_commit(&S.tfull[A.acc]);
    if (++A.acc == static_cast<uint32_t>(q.nbuf)) {
      A.acc = 0;
      A.acc_phase ^= 1u;
    }
  }
}

template <int BN, class Epi>
__device__ void gemm_staged_epilogue(const GemmParams& p, const Epi& epi, const GemmCta<BN>& S,
                                     GemmAccRing& A) {
  constexpr int G = Epi::kGroup;
  constexpr int LD = BN + 4;
  constexpr int F4 = BN / 4;             // float4 per row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x - 64;      // 0..127
  const int sp = warp & 3;
  float* staging = S.staging;
  volatile int* wait_flag = S.wait_flag;
  volatile int* last_flag = S.last_flag;
  uint64_t* tfull = S.tfull;
  uint64_t* tempty = S.tempty;
  const uint32_t tmem_base = S.tmem_base;
  const int acc_cols = S.acc_cols;
  uint32_t& acc = A.acc;
  uint32_t& acc_phase = A.acc_phase;
  uint32_t& nseen = A.nseen;
  GemmSegIter it(p);
  GemmSeg sg;
  while (A.ok && it.next(p, sg)) {
      // one thread waits (bounded) and the verdict is shared, so that the
      // named barriers below are always reached by all 128 threads or none
      if (tid == 0) wait_flag[nseen & 1] = mbar_wait(&tfull[acc], acc_phase, p.err) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!wait_flag[nseen++ & 1]) {
        A.ok = false;
        break;
      }
      tc_fence_after();
      if (sp == 0) {
        // rows 0..31 live in TMEM lanes 0..31: the sub-partition-0 warp reads
        // them (the load is warp-wide), one row per lane, and the lanes below
        // a_rows park theirs in the staging tile, which holds a_rows rows
        const uint32_t taddr = tmem_base + acc * acc_cols;
        const bool keep = lane < p.a_rows;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_load_sum32<BN>(taddr + c * 32, p.nacc, v);
          float* dst = staging + lane * LD + c * 32;
          if (keep) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == static_cast<uint32_t>(p.nbuf)) {
        acc = 0;
        acc_phase ^= 1u;
      }
      named_bar_sync(1, 128);
      if (p.cluster_s > 1) break;          // reduced across the cluster below
      const int rows = p.M;                // one M tile: M <= a_rows <= 32
      const int nf4 = rows * F4;
      if (sg.nseg > 1) {
        float* part = p.partials + static_cast<size_t>(sg.slot) * p.slot_rows * BN;
        for (int i = tid; i < nf4; i += 128) {
          const int r = i / F4, c4 = i - r * F4;
          __stcg(reinterpret_cast<float4*>(part) + i,
                 *reinterpret_cast<const float4*>(staging + r * LD + c4 * 4));
        }
        __threadfence();
        named_bar_sync(1, 128);
        if (tid == 0) {
          const unsigned prev = atomicAdd(&p.counters[sg.tile], 1u);
          const int last = (prev == static_cast<unsigned>(sg.nseg - 1)) ? 1 : 0;
          if (last) p.counters[sg.tile] = 0u;
          *last_flag = last;
        }
        named_bar_sync(1, 128);
        if (!*last_flag) {
          named_bar_sync(1, 128);  // last_flag and staging are rewritten by the next segment
          continue;
        }
        __threadfence();
        // sum the pieces in CTA order; up to 8 float4 per thread in flight per piece
        for (int i0 = tid; i0 < nf4; i0 += 128 * 8) {
          float4 sum[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) sum[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
          for (int c = sg.first_cta; c < sg.first_cta + sg.nseg; ++c) {
            const float4* src = reinterpret_cast<const float4*>(
                p.partials + static_cast<size_t>(gemm_slot_of(p, sg.tile, c)) * p.slot_rows * BN);
            float4 q[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = i0 + u * 128;
              q[u] = i < nf4 ? __ldcg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              sum[u].x += q[u].x;
              sum[u].y += q[u].y;
              sum[u].z += q[u].z;
              sum[u].w += q[u].w;
            }
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * 128;
            if (i < nf4) {
              const int r = i / F4, c4 = i - r * F4;
              *reinterpret_cast<float4*>(staging + r * LD + c4 * 4) = sum[u];
            }
          }
        }
        named_bar_sync(1, 128);
      }
      // epilogue items (row, group of G columns); adjacent threads take adjacent
      // rows of one group, which keeps the staging reads free of bank conflicts
      constexpr int NG = BN / G;
      for (int item = tid; item < rows * NG; item += 128) {
        const int g = item / rows, r = item - g * rows;
        const int n0 = sg.n_tile * BN + g * G;
        if (n0 >= p.N) continue;
        float v[G];
        const float* src = staging + r * LD + g * G;
#pragma unroll
        for (int j = 0; j < G; j += 4) {
          const float4 q = *reinterpret_cast<const float4*>(src + j);
          v[j] = q.x;
          v[j + 1] = q.y;
          v[j + 2] = q.z;
          v[j + 3] = q.w;
        }
        typename Epi::State st;
        epi.begin(st);
        epi.apply(st, r, n0, min(G, p.N - n0), v);
        epi.end(st, r, true);
      }
      named_bar_sync(1, 128);  // staging and last_flag are rewritten by the next segment
    }
}

template <int BN, class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmW, const GemmParams p,
                        const Epi epi) {
  constexpr int G = Epi::kGroup;
  static_assert(BN % G == 0, "epilogue group must divide the tile width");
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_trigger();
  int pre = 0;
  const GemmCta<BN> S = gemm_setup<BN>(p, &tmA, &tmW, pre);
  float* staging = S.staging;
  volatile int* wait_flag = S.wait_flag;
  volatile int* last_flag = S.last_flag;
  uint64_t* tfull = S.tfull;
  uint64_t* tempty = S.tempty;
  const uint32_t tmem_base = S.tmem_base;
  const int acc_cols = S.acc_cols;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      pdl_wait();
      GemmRing R;
      gemm_produce<BN>(p, &tmA, &tmW, S, R, pre, nullptr, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      GemmRing R;
      GemmAccRing A;
      gemm_mma<BN>(p, S, R, A);
    }
  } else if (gemm_staged(p.a_rows)) {
    // ------------------------------------------------------------ staged epilogue
    pdl_wait();
    GemmAccRing A;
    gemm_staged_epilogue<BN, Epi>(p, epi, S, A);
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();
    const int ew = warp - 2;        // 0..3
    const int sp = warp & 3;        // TMEM sub-partition this warp may read
    const int row = sp * 32 + lane;
    uint32_t acc = 0, acc_phase = 0, nseen = 0;
    GemmSegIter it(p);
    GemmSeg sg;
    while (it.next(p, sg)) {
      if (ew == 0 && lane == 0) wait_flag[nseen & 1] = mbar_wait(&tfull[acc], acc_phase, p.err) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!wait_flag[nseen++ & 1]) break;
      tc_fence_after();
      const int m = sg.m_tile * kGemmBM + row;
      const bool row_ok = m < p.M;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(sp * 32) << 16) + acc * acc_cols;
      if (sg.nseg == 1) {
        typename Epi::State st;
        epi.begin(st);
#pragma unroll 1
        for (int g = 0; g < BN / G; ++g) {
          float v[G];
#pragma unroll
          for (int c = 0; c < G / 32; ++c) tmem_load_sum32<BN>(taddr + g * G + c * 32, p.nacc, v + c * 32);
          const int n0 = sg.n_tile * BN + g * G;
          if (row_ok && n0 < p.N) epi.apply(st, m, n0, min(G, p.N - n0), v);
        }
        epi.end(st, m, row_ok);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
      } else {
        float* part = p.partials + static_cast<size_t>(sg.slot) * p.slot_rows * BN;
#pragma unroll 1
        for (int g = 0; g < BN / G; ++g) {
          float v[G];
#pragma unroll
          for (int c = 0; c < G / 32; ++c) tmem_load_sum32<BN>(taddr + g * G + c * 32, p.nacc, v + c * 32);
          if (row_ok) {
            float* dst = part + static_cast<size_t>(row) * BN + g * G;
#pragma unroll
            for (int j = 0; j < G; j += 4)
              __stcg(reinterpret_cast<float4*>(dst + j),
                     make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
          }
        }
        __threadfence();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        named_bar_sync(1, 128);
        if (ew == 0 && lane == 0) {
          const unsigned prev = atomicAdd(&p.counters[sg.tile], 1u);
          const int last = (prev == static_cast<unsigned>(sg.nseg - 1)) ? 1 : 0;
          if (last) p.counters[sg.tile] = 0u;
          *last_flag = last;
        }
        named_bar_sync(1, 128);
        const int last = *last_flag;
        if (last) {
          __threadfence();
          typename Epi::State st;
          epi.begin(st);
#pragma unroll 1
          for (int g = 0; g < BN / G; ++g) {
            const int n0 = sg.n_tile * BN + g * G;
            if (row_ok && n0 < p.N) {
              float v[G];
#pragma unroll
              for (int j = 0; j < G; ++j) v[j] = 0.f;
              for (int c = sg.first_cta; c < sg.first_cta + sg.nseg; ++c) {
                const float* src = p.partials +
                                   (static_cast<size_t>(gemm_slot_of(p, sg.tile, c)) *
                                        p.slot_rows + row) * BN + g * G;
#pragma unroll
                for (int j = 0; j < G; j += 4) {
                  const float4 q = __ldcg(reinterpret_cast<const float4*>(src + j));
                  v[j] += q.x;
                  v[j + 1] += q.y;
                  v[j + 2] += q.z;
                  v[j + 3] += q.w;
                }
              }
              epi.apply(st, m, n0, min(G, p.N - n0), v);
            }
          }
          epi.end(st, m, row_ok);
        }
        named_bar_sync(1, 128);  // last_flag is rewritten by the next segment
      }
      if (++acc == static_cast<uint32_t>(p.nbuf)) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }


  if (p.cluster_s > 1) {
    // Every thread of every CTA of the cluster reaches both barriers exactly
    // once (no early exits above, all waits bounded).  Between them, CTA rank q
    // owns the column groups g = q, q + S, ... of the tile: first all 128
    // epilogue threads sum, per float4 of those groups, the S staging tiles in
    // rank order (deterministic; S independent peer loads in flight per
    // thread) into this CTA's own staging tile — peers only read the groups
    // they own, never these — then each (row, group) item runs the epilogue.
    cluster_sync();
    if (warp >= 2) {
      constexpr int LD = BN + 4;
      constexpr int NG = BN / G;
      constexpr int GF4 = G / 4;
      const int S = p.cluster_s;
      const int rank = static_cast<int>(cluster_rank());
      const int tile = blockIdx.x / S;
      const int n_tile = tile / p.m_tiles;
      const int rows = p.M;
      const int my_groups = (NG - rank + S - 1) / S;
      const int tid = threadIdx.x - 64;
      for (int it = tid; it < my_groups * rows * GF4; it += 128) {
        const int c4 = it % GF4, rest = it / GF4;
        const int r = rest % rows, lg = rest / rows;
        float* src = staging + r * LD + (rank + lg * S) * G + c4 * 4;
        float4 t[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < S) t[q] = ld_peer_f4(src, static_cast<uint32_t>(q));
        float4 acc = t[0];
#pragma unroll
        for (int q = 1; q < 8; ++q) {
          if (q < S) {
            acc.x += t[q].x;
            acc.y += t[q].y;
            acc.z += t[q].z;
            acc.w += t[q].w;
          }
        }
        *reinterpret_cast<float4*>(src) = acc;
      }
      named_bar_sync(1, 128);
      for (int item = tid; item < my_groups * rows; item += 128) {
        const int lg = item / rows, r = item - lg * rows;
        const int g = rank + lg * S;
        const int n0 = n_tile * BN + g * G;
        if (n0 >= p.N) continue;
        float v[G];
        const float* src = staging + r * LD + g * G;
#pragma unroll
        for (int j = 0; j < G; j += 4) {
          const float4 q4 = *reinterpret_cast<const float4*>(src + j);
          v[j] = q4.x;
          v[j + 1] = q4.y;
          v[j + 2] = q4.z;
          v[j + 3] = q4.w;
        }
        typename Epi::State st;
        epi.begin(st);
        epi.apply(st, r, n0, min(G, p.N - n0), v);
        epi.end(st, r, true);
      }
    }
    cluster_sync();  // no CTA leaves while a peer may still read its staging tile
  }

  tc_fence_before();
  cta_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, static_cast<uint32_t>(p.tmem_cols));
  }
}

// Two GEMMs in one launch (few rows, staged epilogue, no clusters): phase 1
// (A1 x W1^T, epilogue e1) then phase 2 (A2 x W2^T, e2) on the same CTAs, the
// same pipeline ring and the same accumulator, where A2 is written by phase 1.
// Every CTA's epilogue arrives on dep[0] once its phase-1 stores are out; a
// producer loads A2 only after all gridDim.x CTAs have arrived, and meanwhile
// streams phase 2's first weight stages — so the second weight stream starts
// while the first one drains, without a kernel boundary.  The last CTA to
// finish resets dep[0] and dep[1] to zero for the next launch.  Every CTA of
// the grid must be able to become resident (the grid is at most one CTA per
// SM, and nothing the CTAs wait on depends on them), so the wait ends.
template <int BN, class Epi1, class Epi2>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_chain_kernel(const __grid_constant__ CUtensorMap tmA1,
                      const __grid_constant__ CUtensorMap tmW1, const GemmParams p1,
                      const Epi1 e1, const __grid_constant__ CUtensorMap tmA2,
                      const __grid_constant__ CUtensorMap tmW2, const GemmParams p2,
                      const Epi2 e2, unsigned* dep) {
  static_assert(BN % Epi1::kGroup == 0 && BN % Epi2::kGroup == 0, "epilogue groups");
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_trigger();
  int pre = 0;
  const GemmCta<BN> S = gemm_setup<BN>(p1, &tmA1, &tmW1, pre);

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();
      GemmRing R;
      gemm_produce<BN>(p1, &tmA1, &tmW1, S, R, pre, nullptr, 0);
      if (R.ok) {
        tma_prefetch_desc(&tmA2);
        tma_prefetch_desc(&tmW2);
      }
      gemm_produce<BN>(p2, &tmA2, &tmW2, S, R, 0, dep, gridDim.x);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      GemmRing R;
      GemmAccRing A;
      gemm_mma<BN>(p1, S, R, A);
      gemm_mma<BN>(p2, S, R, A);
    }
  } else {
    pdl_wait();
    GemmAccRing A;
    gemm_staged_epilogue<BN, Epi1>(p1, e1, S, A);
    // phase-1 stores of this CTA are out: arrive
    named_bar_sync(1, 128);
    if (threadIdx.x == 64) {
      __threadfence();
      atomicAdd(&dep[0], 1u);
    }
    gemm_staged_epilogue<BN, Epi2>(p2, e2, S, A);
  }

  tc_fence_before();
  cta_sync();
  if (threadIdx.x == 0) {
    // the last CTA out resets the arrival counters for the next launch
    const unsigned prev = atomicAdd(&dep[1], 1u);
    if (prev == gridDim.x - 1) {
      dep[0] = 0u;
      dep[1] = 0u;
      __threadfence();
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(S.tmem_base, static_cast<uint32_t>(p1.tmem_cols));
  }
}

// ---------------------------------------------------------------------------
// epilogue functors
//   kGroup columns (one contiguous group of output features) are handed to
//   apply() at a time, as fp32 values of one output row.
// ---------------------------------------------------------------------------
struct EpiNoState {};

// out[m, n] = acc  (fp32)
struct EpiStoreF32 {
  static constexpr int kGroup = 32;
  using State = EpiNoState;
  float* out;
  int ldo;
  __device__ void begin(State&) const {}
  __device__ void end(State&, int, bool) const {}
  __device__ void apply(State&, int m, int n0, int nv, const float* v) const {
    float* dst = out + static_cast<size_t>(m) * ldo + n0;
    if (nv == kGroup) {
#pragma unroll
      for (int j = 0; j < kGroup; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < kGroup; ++j)
        if (j < nv) dst[j] = v[j];
    }
  }
};

// x[m, n] += acc  (fp32 residual stream)
struct EpiResidAdd {
  static constexpr int kGroup = 32;
  using State = EpiNoState;
  float* x;
  int ldx;
  __device__ void begin(State&) const {}
  __device__ void end(State&, int, bool) const {}
  __device__ void apply(State&, int m, int n0, int nv, const float* v) const {
    float* dst = x + static_cast<size_t>(m) * ldx + n0;
    if (nv == kGroup) {
#pragma unroll
      for (int j = 0; j < kGroup; j += 4) {
        float4 r = *reinterpret_cast<float4*>(dst + j);
        r.x += v[j];
        r.y += v[j + 1];
        r.z += v[j + 2];
        r.w += v[j + 3];
        *reinterpret_cast<float4*>(dst + j) = r;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kGroup; ++j)
        if (j < nv) dst[j] += v[j];
    }
  }
};

// Gate/up weights are packed in blocks of 32 rows: 16 gate rows then the 16 up
// rows of the same features.  h[m, f] = bf16(silu(gate) * up).
struct EpiSwiGLU {
  static constexpr int kGroup = 32;
  using State = EpiNoState;
  bf16* h;
  int ldh;
  __device__ void begin(State&) const {}
  __device__ void end(State&, int, bool) const {}
  __device__ void apply(State&, int m, int n0, int nv, const float* v) const {
    (void)nv;  // the packed width is a multiple of 32
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float g0 = v[j], g1 = v[j + 1];
      const float a0 = g0 / (1.f + expf(-g0)) * v[16 + j];
      const float a1 = g1 / (1.f + expf(-g1)) * v[17 + j];
      w[j / 2] = pack_bf16x2(a0, a1);
    }
    uint4* dst = reinterpret_cast<uint4*>(h + static_cast<size_t>(m) * ldh + (n0 >> 1));
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
};

// Per-head RMSNorm (weight w) then rotate-half RoPE with the (cos, sin) table
// row `cs`, in place on D values.
template <int D>
__device__ __forceinline__ void head_norm_rope(float* v, const bf16* w, const float2* cs,
                                               float eps) {
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < D; ++j) ss += v[j] * v[j];
  const float r = rsqrtf(ss / D + eps);
#pragma unroll
  for (int j = 0; j < D; ++j) v[j] = v[j] * r * bf2f(w[j]);
#pragma unroll
  for (int j = 0; j < D / 2; ++j) {
    const float2 c = cs[j];
    const float a = v[j], b = v[j + D / 2];
    v[j] = a * c.x - b * c.y;
    v[j + D / 2] = b * c.x + a * c.y;
  }
}

template <int D>
__device__ __forceinline__ void store_bf16_row(bf16* dst, const float* v) {
#pragma unroll
  for (int j = 0; j < D; j += 8) {
    uint4 q;
    q.x = pack_bf16x2(v[j], v[j + 1]);
    q.y = pack_bf16x2(v[j + 2], v[j + 3]);
    q.z = pack_bf16x2(v[j + 4], v[j + 5]);
    q.w = pack_bf16x2(v[j + 6], v[j + 7]);
    *reinterpret_cast<uint4*>(dst + j) = q;
  }
}

// Draft-layer QKV projection of the query block.  Output features are
// [q heads | k heads | v heads], one head per group.  q, k: per-head RMSNorm +
// RoPE at the block position seq_len + i; q goes to the q buffer, k and v to
// the request's paged slot of this layer's cache.
template <int D>
struct EpiQKV {
  static constexpr int kGroup = D;
  using State = EpiNoState;
  bf16* q;
  const bf16* q_norm_w;
  const bf16* k_norm_w;
  const float2* rope;
  bf16* k_cache;
  bf16* v_cache;
  const int* seq_lens;
  const int* block_table;
  int max_pos, W, bs, Hq, Hkv, P, num_pages;
  float eps;
  unsigned* err;
  __device__ void begin(State&) const {}
  __device__ void end(State&, int, bool) const {}
  __device__ void apply(State&, int m, int n0, int nv, float* v) const {
    (void)nv;
    const int head = n0 / D;
    const int b = m / bs, i = m - (m / bs) * bs;
    const int pos = seq_lens[b] + i;
    if (head < Hq + Hkv) {
      if (pos < 0 || pos >= max_pos) {
        raise_error(err, DFLASH_DEVERR_POSITION);
        return;
      }
      head_norm_rope<D>(v, head < Hq ? q_norm_w : k_norm_w,
                        rope + static_cast<size_t>(pos) * (D / 2), eps);
    }
    if (head < Hq) {
      store_bf16_row<D>(q + (static_cast<size_t>(m) * Hq + head) * D, v);
      return;
    }
    const int pg = pos / P;
    if (pg >= W) {
      raise_error(err, DFLASH_DEVERR_TABLE);
      return;
    }
    const int page = block_table[static_cast<size_t>(b) * W + pg];
    if (page < 0 || page >= num_pages) {
      raise_error(err, DFLASH_DEVERR_SLOT);
      return;
    }
    const bool is_k = head < Hq + Hkv;
    const int kh = is_k ? head - Hq : head - Hq - Hkv;
    bf16* cache = is_k ? k_cache : v_cache;
    store_bf16_row<D>(cache + ((static_cast<size_t>(page) * Hkv + kh) * P + (pos - pg * P)) * D, v);
  }
};

constexpr int kMaxLayers = 64;

// Context K/V injection.  Output features are ordered per layer as
// [k heads | v heads]; a group is one (layer, k|v, head).  Keys get the layer's
// k_norm and RoPE at the row's own position; rows with a negative slot are
// padding and are skipped.
template <int D>
struct EpiKVInject {
  static constexpr int kGroup = D;
  using State = EpiNoState;
  bf16* k_cache[kMaxLayers];
  bf16* v_cache[kMaxLayers];
  const bf16* k_norm_w;  // [L][D]
  const float2* rope;
  const int64_t* positions;
  const int64_t* slots;
  int max_pos, Hkv, P, num_pages;
  float eps;
  unsigned* err;
  __device__ void begin(State&) const {}
  __device__ void end(State&, int, bool) const {}
  __device__ void apply(State&, int m, int n0, int nv, float* v) const {
    (void)nv;
    const int64_t slot = slots[m];
    if (slot < 0) return;
    if (slot >= static_cast<int64_t>(num_pages) * P) {
      raise_error(err, DFLASH_DEVERR_SLOT);
      return;
    }
    const int hi = n0 / D;
    const int l = hi / (2 * Hkv);
    const int kind = (hi / Hkv) & 1;
    const int kh = hi - (hi / Hkv) * Hkv;
    if (kind == 0) {
      const int64_t pos = positions[m];
      if (pos < 0 || pos >= max_pos) {
        raise_error(err, DFLASH_DEVERR_POSITION);
        return;
      }
      head_norm_rope<D>(v, k_norm_w + static_cast<size_t>(l) * D,
                        rope + static_cast<size_t>(pos) * (D / 2), eps);
    }
    const int64_t page = slot / P, off = slot - (slot / P) * P;
    bf16* cache = kind == 0 ? k_cache[l] : v_cache[l];
    store_bf16_row<D>(cache + ((page * Hkv + kh) * P + off) * D, v);
  }
};

// LM head with greedy pick: per row, the ordered key of (max logit, lowest id)
// is folded into keys[m] with one 64-bit atomicMax per tile.  Optionally also
// writes the fp32 logits (debug).
struct EpiArgmax {
  static constexpr int kGroup = 32;
  struct State {
    unsigned long long best;
  };
  unsigned long long* keys;
  float* logits;
  int ldl;
  uint32_t idx_base;   // vocabulary id of column 0 (a shard's first row)
  __device__ void begin(State& s) const { s.best = 0ull; }
  __device__ void apply(State& s, int m, int n0, int nv, const float* v) const {
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      if (j < nv) {
        const unsigned long long k =
            argmax_key(v[j], idx_base + static_cast<uint32_t>(n0 + j));
        s.best = k > s.best ? k : s.best;
      }
    }
    if (logits) {
      float* dst = logits + static_cast<size_t>(m) * ldl + n0;
#pragma unroll
      for (int j = 0; j < kGroup; ++j)
        if (j < nv) dst[j] = v[j];
    }
  }
  __device__ void end(State& s, int m, bool row_ok) const {
    if (row_ok && s.best) atomicMax(keys + m, s.best);
  }
};

}  // namespace dflash
