// gemm_pair.cuh — the many-row GEMM on CTA pairs: one tcgen05.mma with
// cta_group::2 computes a 256 x 256 x 16 (or 256 x 128 x 16) block over two SMs.
//
// Same product and epilogue functors as gemm_tcgen05_kernel
// (D[m, n] = sum_k A[m, k] W[n, k], fp32 accumulation, the epilogue applied per
// output row and column group), for plans of whole tiles over several 128-row
// M tiles (the proposal's GEMMs at batch >= 16, the LM head at batch >= 9, the
// injection of >= 129 rows).  Tiles are 256 x 256, or 256 x 128 where only the
// narrower tiles keep the SMs busy (few rows against a narrow output).
//
// Why: on one SM a 128 x 256 x 16 MMA takes ~128 cycles and reads 12 KB of
// operands from shared memory, while TMA writes the next 12 KB of the ring: about
// 190 bytes per cycle against the ~128 that shared memory delivers, so the
// tensor pipe idles about a third of the time (measured: 45-56% active in the
// many-row GEMMs of the 128-request draft step).  On a CTA pair each SM holds
// 128 rows of A and 128 of the tile's 256 W rows; the pair's MMA reads the W
// halves of both SMs, so per SM and per 128 cycles it reads 8 KB and receives
// 8 KB.
//
// A cluster of two CTAs; rank 0 leads.  In each CTA warp 0 is the TMA producer
// for its own rows (A rows [m0 + 128 rank, +128) and W rows
// [n0 + rank BN / 2, +BN / 2) of every k-block, into its own ring) and counts
// the bytes on the leader's full barrier; warp 1 of the leader issues the MMAs
// and commits to both CTAs' barriers at once; warps 2..5 of each CTA drain its
// 128 accumulator rows (TMEM lanes) x BN columns and release the buffer on the
// leader's barrier.  Both CTAs allocate the same TMEM columns.  No TMA load
// here multicasts: each CTA loads only the rows it holds.
//
// Every wait is bounded; after a wait runs out the CTA winds down like
// gemm_tcgen05_kernel.
#pragma once

#include "gemm_tcgen05.cuh"

namespace dflash {

constexpr int kPairRows = 128;                           // A rows per CTA
constexpr int kPairHalfBytes = kPairRows * kGemmBK * 2;  // one 128 x 64 A box

// A pair tile is 256 rows x BN columns (BN = 256, or 128 when only the
// narrower tiles fill the SMs); each CTA holds BN / 2 of its W rows.
template <int BN>
struct PairCfg {
  static_assert(BN == 256 || BN == 128, "pair tile width");
  static constexpr int kWRows = BN / 2;                       // W rows per CTA
  static constexpr int kWBytes = kWRows * kGemmBK * 2;        // its W box
  static constexpr int kStageBytes = kPairHalfBytes + kWBytes;
  static constexpr int kTmemCols = 2 * BN;                    // two accumulators
  static constexpr int kMaxStages = (kGemmSmemLimit - 1024 - kGemmBarrierBytes) / kStageBytes;
  static constexpr int kStages = kMaxStages < kGemmMaxStages ? kMaxStages : kGemmMaxStages;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + kGemmBarrierBytes;
};

// Address of this CTA's shared variable at `saddr` in the CTA of cluster rank
// `rank` (shared::cluster window).
__device__ __forceinline__ uint32_t cluster_addr(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Arrive (release, cluster scope) on an mbarrier given by its cluster address.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}
// Paired TMEM allocation: the same warp of both CTAs allocates the same columns.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (+)= A B^T over the pair: A rows 0..127 and W rows 0..127 from the leader's
// shared memory at the descriptors' addresses, rows 128..255 from the peer's
// at the same addresses; D rows split the same way over the CTAs' TMEM.
__device__ __forceinline__ void umma_pair_f16kind(uint32_t d_tmem, uint64_t a_desc,
                                                  uint64_t b_desc, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Once the pair's earlier MMAs retired: arrive on the barrier at `bar`'s
// offset in both CTAs of the pair (cluster ranks given by `mask`).
__device__ __forceinline__ void umma_pair_commit_both(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}
// 2-D tiled TMA load into this CTA's shared memory whose completed bytes are
// counted on the mbarrier at cluster address `bar_cluster` (the leader's).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int c0, int c1,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

// p.m_tiles = 256-row pair tiles, p.n_tiles = BN-column tiles, p.tiles their
// product (m fastest); p.stages ring depth; W boxes are BN / 2 rows.
//
// KS = 2 (split K over two pairs, a cluster of four, one tile per cluster):
// pair q (cluster ranks 2q, 2q + 1) accumulates k-blocks [q * kh, (q+1) * kh);
// once every MMA of the cluster has retired, each CTA of pair 1 writes its
// fp32 accumulator rows into the idle stage ring of the CTA of pair 0 that
// holds the same rows (distributed shared memory), and pair 0 adds them to its
// own, in that fixed order, and runs the epilogue.
template <int BN, int KS, class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmW, const GemmParams p,
                     const Epi epi) {
  using PC = PairCfg<BN>;
  constexpr int G = Epi::kGroup;
  static_assert(BN % G == 0, "epilogue group must divide the tile width");
  static_assert(KS == 1 || KS == 2, "K splits");
  constexpr int LD = BN + 4;   // padded row of the split-K partial (fp32)
  static_assert(KS == 1 || kPairRows * LD * 4 <= 7 * PC::kStageBytes, "partial fits the ring");
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t pr = rank & 1u;          // CTA of the pair: rows [128 pr, +128) of a tile
  const uint32_t q = rank >> 1;           // K part (0 when KS == 1)
  const uint32_t lead = rank & ~1u;       // the pair's leader
  const uint16_t pair_mask = static_cast<uint16_t>(3u << lead);
  const int kh = (p.k_blocks + KS - 1) / KS;
  const int kb0 = static_cast<int>(q) * kh, kb1 = min(p.k_blocks, kb0 + kh);
  pdl_trigger();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  uint8_t* sA = smem;                                   // [stages][128 x 128 B]
  uint8_t* sW = smem + stages * kPairHalfBytes;         // [stages][BN / 2 x 128 B]
  uint64_t* full = reinterpret_cast<uint64_t*>(sW + stages * PC::kWBytes);
  uint64_t* empty = full + kGemmMaxStages;
  uint64_t* tfull = empty + kGemmMaxStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* wait_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);    // leader's: its producer's arrival + both CTAs' bytes
      mbar_init(&empty[s], 1);   // each CTA's: the leader's commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);   // each CTA's: the leader's commit
      mbar_init(&tempty[a], 8);  // leader's: the 4 epilogue warps of both CTAs
    }
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, PC::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // both CTAs' barriers exist before any remote arrival or byte count
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n_cl = static_cast<int>(gridDim.x) / (2 * KS);
  const int cl = static_cast<int>(blockIdx.x) / (2 * KS);
  bool epi_ok = false;   // split K: this CTA's accumulator is complete

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      pdl_wait();
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      const uint32_t full_lead = cluster_addr(smem_u32(full), lead);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int t = cl; ok && t < p.tiles; t += n_cl) {
        const int mp = t % p.m_tiles, nt = t / p.m_tiles;
        const int a_row = mp * 2 * kPairRows + static_cast<int>(pr) * kPairRows;
        const int w_tile = nt * 2 + static_cast<int>(pr);   // BN / 2-row W tile index
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) {
            ok = false;
            break;
          }
          if (pr == 0) mbar_arrive_expect_tx(&full[stage], 2u * PC::kStageBytes);
          const uint32_t fb = full_lead + stage * 8u;
          tma_load_2d_pair(sW + stage * PC::kWBytes, &tmW, fb, w_x(p, kb),
                           w_y<PC::kWRows>(p, w_tile, kb), pol_w);
          tma_load_2d_pair(sA + stage * kPairHalfBytes, &tmA, fb, kb * kGemmBK, a_row, pol_a);
          if (++stage == static_cast<uint32_t>(stages)) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every stage this CTA filled is released before it may exit, so that no
      // commit of the leader arrives on a barrier of a finished CTA
      for (int s = 0; ok && s < stages; ++s) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) break;
        if (++stage == static_cast<uint32_t>(stages)) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (pr == 0 && lane == 0) {
      const uint32_t idesc = umma_idesc_f32acc(2 * kPairRows, BN, p.f16 != 0);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int t = cl; ok && t < p.tiles; t += n_cl) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.err)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128(smem_u32(sA + stage * kPairHalfBytes));
          const uint64_t bd = umma_desc_sw128(smem_u32(sW + stage * PC::kWBytes));
#pragma unroll
          for (int k = 0; k < kGemmBK / 16; ++k)
            umma_pair_f16kind(d, ad + 2 * k, bd + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          umma_pair_commit_both(&empty[stage], pair_mask);
          if (++stage == static_cast<uint32_t>(stages)) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_pair_commit_both(&tfull[acc], pair_mask);
        if (++acc == 2u) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();
    const int ew = warp - 2;
    const int sp = warp & 3;            // TMEM sub-partition this warp may read
    const int row = sp * 32 + lane;
    const uint32_t tempty_lead = cluster_addr(smem_u32(tempty), lead);
    uint32_t acc = 0, acc_phase = 0, nseen = 0;
    for (int t = cl; t < p.tiles; t += n_cl) {
      if (ew == 0 && lane == 0)
        wait_flag[nseen & 1] = mbar_wait(&tfull[acc], acc_phase, p.err) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!wait_flag[nseen++ & 1]) break;
      tc_fence_after();
      if constexpr (KS == 2) {
        epi_ok = true;   // one tile per cluster: reduced and stored below
        break;
      }
      const int mp = t % p.m_tiles, nt = t / p.m_tiles;
      const int m = mp * 2 * kPairRows + static_cast<int>(pr) * kPairRows + row;
      const bool row_ok = m < p.M;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(sp * 32) << 16) + acc * BN;
      typename Epi::State st;
      epi.begin(st);
#pragma unroll 1
      for (int g = 0; g < BN / G; ++g) {
        float v[G];
#pragma unroll
        for (int c = 0; c < G / 32; ++c) tmem_ld_32x32b_x32(taddr + g * G + c * 32, v + c * 32);
        tmem_ld_wait();
        const int n0 = nt * BN + g * G;
        if (row_ok && n0 < p.N) epi.apply(st, m, n0, min(G, p.N - n0), v);
      }
      epi.end(st, m, row_ok);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_lead + acc * 8u);
      if (++acc == 2u) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  if constexpr (KS == 2) {
    // every MMA of the cluster has retired (each epilogue saw its tfull): the
    // stage rings are idle and pair 1 can write its partial into pair 0's
    float* stg = reinterpret_cast<float*>(smem);   // [128][LD] fp32, over the ring
    const int sp = warp & 3, row = sp * 32 + lane;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(sp * 32) << 16);
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp >= 2 && q == 1 && epi_ok) {
      const uint32_t dst = cluster_addr(smem_u32(stg + row * LD), rank - 2u);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld_32x32b_x32(taddr + c * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                           dst + static_cast<uint32_t>((c * 32 + 4 * j) * 4)),
                       "f"(v[4 * j]), "f"(v[4 * j + 1]), "f"(v[4 * j + 2]), "f"(v[4 * j + 3])
                       : "memory");
      }
    }
    tc_fence_before();
    cluster_sync();   // pair 1's partials are in pair 0's shared memory
    tc_fence_after();
    if (warp >= 2 && q == 0 && epi_ok) {
      const int t = cl;
      const int mp = t % p.m_tiles, nt = t / p.m_tiles;
      const int m = mp * 2 * kPairRows + static_cast<int>(pr) * kPairRows + row;
      const bool row_ok = m < p.M;
      const float* own = stg + row * LD;
      typename Epi::State st;
      epi.begin(st);
#pragma unroll 1
      for (int g = 0; g < BN / G; ++g) {
        float v[G];
#pragma unroll
        for (int c = 0; c < G / 32; ++c) tmem_ld_32x32b_x32(taddr + g * G + c * 32, v + c * 32);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < G; j += 4) {
          const float4 r4 = *reinterpret_cast<const float4*>(own + g * G + j);
          v[j] += r4.x;
          v[j + 1] += r4.y;
          v[j + 2] += r4.z;
          v[j + 3] += r4.w;
        }
        const int n0 = nt * BN + g * G;
        if (row_ok && n0 < p.N) epi.apply(st, m, n0, min(G, p.N - n0), v);
      }
      epi.end(st, m, row_ok);
    }
  }

  tc_fence_before();
  cluster_sync();   // the pair's MMAs, TMEM reads and remote arrivals are over
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, PC::kTmemCols);
  }
}

}  // namespace dflash
