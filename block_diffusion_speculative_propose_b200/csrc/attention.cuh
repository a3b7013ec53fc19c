// attention.cuh — non-causal block attention over a paged KV cache (sm_100a).
//
// One CTA serves one (request b, kv head h, key split): all bs * G query rows
// of the kv group (bs block slots x G = Hq / Hkv query heads) attend, with no
// mask inside the range, to keys [split * chunk, ...) of the request's logical
// keys [0, seq_len + bs) — its injected context plus its whole block.  Each K
// and V byte is read from HBM once per kv group.  Compute warps are laid out as
// (row group of 16 query rows) x (key part of each 64-key tile); the parts'
// softmax states are merged in shared memory after the last tile.
//
// Pages are staged with TMA tile loads (128-byte swizzle, one 16-row x 128-byte
// box per page and 64-wide half of head_dim) into a ring of shared-memory
// stages of 64 keys; a producer warp walks the block table.  Compute warps own
// 16 query rows each and run bf16 mma.sync (m16n8k16) for Q K^T and P V with an
// fp32 online softmax whose row statistics are reduced with quad shuffles.
// When the request needs more than one split, partial (O, m, l) go to a
// workspace and attn_combine_kernel merges them in split order.
#pragma once

#include "dflash_device.cuh"

namespace dflash {

constexpr int kAttnTileKeys = 64;
constexpr int kAttnStages = 4;
constexpr int kAttnMaxComputeWarps = 8;

template <int D>
struct AttnCfg {
  static constexpr int kBoxBytes = 16 * 128;          // 16 keys x 64 bf16
  static constexpr int kBoxesPerPage = D / 64;
  static constexpr int kPagesPerTile = kAttnTileKeys / 16;
  static constexpr int kKVBytes = kPagesPerTile * kBoxesPerPage * kBoxBytes;
  static constexpr int kQStride = D + 8;              // padded row (bf16 elements)
  static constexpr int smem_bytes(int n_compute_warps) {
    return 1024 + kAttnStages * 2 * kKVBytes + n_compute_warps * 16 * kQStride * 2 + 256;
  }
  static_assert(kAttnStages * 2 * kKVBytes >= 7 * 16 * D * 4 + 7 * 32 * 16,
                "the stage buffers hold the key-part merge");
};

struct AttnParams {
  int row_groups;      // ceil(R / 16)
  int key_parts;       // compute warps per row group (each takes 64 / key_parts keys of a tile)
  const bf16* q;       // [M, Hq, D]
  f16* o;              // [M, Hq * D] (convex combinations of V rows: fp16)
  float* part_o;       // [max_splits][B][Hkv][R][D]
  float* part_ml;      // [max_splits][B][Hkv][R][2]
  const int* seq_lens;
  const int* block_table;
  int B, W, bs, Hq, Hkv, G, R, num_pages, chunk_keys, max_splits;
  int cluster;         // tcgen05 kernel: the max_splits splits of a (request, kv head) form one
                       // thread-block cluster and are combined through distributed shared memory
  float scale_log2;    // log2(e) / sqrt(D)
  unsigned* err;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte offset of (key kt in tile, 16-byte chunk c of the D-wide row) inside a
// K or V stage laid out as [page][box half][16 rows x 128 B, 128B-swizzled].
template <int D>
__device__ __forceinline__ uint32_t kv_off(int kt, int c) {
  const int jp = kt >> 4, rp = kt & 15;
  const int hf = c >> 3, cc = c & 7;
  return static_cast<uint32_t>((jp * AttnCfg<D>::kBoxesPerPage + hf) * AttnCfg<D>::kBoxBytes +
                               rp * 128 + ((cc ^ (rp & 7)) << 4));
}

template <int D, int KP>
__global__ void __launch_bounds__(32 * (kAttnMaxComputeWarps + 1), 1)
    attn_block_kernel(const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = AttnCfg<D>;
  constexpr int NB = KP / 8;    // 8-key blocks of this warp's part of a tile
  constexpr int KS = KP / 16;   // 16-key (one page) PV steps
  pdl_trigger();
  pdl_wait();
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n_keys = p.seq_lens[b] + p.bs;
  const int k0 = split * p.chunk_keys;
  if (k0 >= n_keys) return;
  const int k1 = min(n_keys, k0 + p.chunk_keys);
  const int n_splits_b = (n_keys + p.chunk_keys - 1) / p.chunk_keys;
  const int nwc = p.row_groups * p.key_parts;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + kAttnStages * C::kKVBytes;
  bf16* sQ = reinterpret_cast<bf16*>(sV + kAttnStages * C::kKVBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(sQ + nwc * 16 * C::kQStride);
  uint64_t* empty = full + kAttnStages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], nwc);
    }
    fence_barrier_init();
  }
  cta_sync();

  const int n_tiles = (k1 - k0 + kAttnTileKeys - 1) / kAttnTileKeys;

  if (warp == nwc) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int* bt = p.block_table + static_cast<size_t>(b) * p.W;
      uint32_t stage = 0, phase = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int t0 = k0 + t * kAttnTileKeys;
        const int nvalid = min(kAttnTileKeys, k1 - t0);
        const int npages = (nvalid + 15) >> 4;
        if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) break;
        mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(npages * C::kBoxesPerPage *
                                                                  C::kBoxBytes * 2));
        for (int j = 0; j < npages; ++j) {
          const int pg = (t0 >> 4) + j;
          int y;
          if (pg >= p.W) {
            raise_error(p.err, DFLASH_DEVERR_TABLE);
            y = -16;  // fully out of bounds: TMA fills zeros
          } else {
            const int page = bt[pg];
            if (page < 0 || page >= p.num_pages) {
              raise_error(p.err, DFLASH_DEVERR_SLOT);
              y = -16;
            } else {
              y = (page * p.Hkv + h) * 16;
            }
          }
#pragma unroll
          for (int hf = 0; hf < C::kBoxesPerPage; ++hf) {
            const uint32_t off = (j * C::kBoxesPerPage + hf) * C::kBoxBytes;
            tma_load_2d(sK + stage * C::kKVBytes + off, &tmK, &full[stage], hf * 64, y);
            tma_load_2d(sV + stage * C::kKVBytes + off, &tmV, &full[stage], hf * 64, y);
          }
        }
        if (++stage == kAttnStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- compute warps
  const int rg = warp % p.row_groups;   // query rows rg*16 .. rg*16+15
  const int kp = warp / p.row_groups;   // keys kp*KP .. kp*KP+KP-1 of every tile
  // Q rows of this warp: r = i * G + g  ->  q[(b*bs + i), h*G + g, :]
  bf16* sQw = sQ + warp * 16 * C::kQStride;
  {
    // all of a lane's loads are issued before any store
    constexpr int kQPer = 16 * (D / 8) / 32;
    uint4 qv[kQPer];
#pragma unroll
    for (int u = 0; u < kQPer; ++u) {
      const int e = lane + u * 32;
      const int rr = e / (D / 8), c = e - rr * (D / 8);
      const int r = rg * 16 + rr;
      qv[u] = make_uint4(0, 0, 0, 0);
      if (r < p.R) {
        const int i = r / p.G, g = r - (r / p.G) * p.G;
        const bf16* src = p.q + (static_cast<size_t>(b * p.bs + i) * p.Hq + h * p.G + g) * D;
        qv[u] = *reinterpret_cast<const uint4*>(src + c * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < kQPer; ++u) {
      const int e = lane + u * 32;
      const int rr = e / (D / 8), c = e - rr * (D / 8);
      *reinterpret_cast<uint4*>(sQw + rr * C::kQStride + c * 8) = qv[u];
    }
  }
  __syncwarp();
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int row = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int col = ks * 16 + (lane >> 4) * 8;
    ldmatrix_x4(smem_u32(sQw + row * C::kQStride + col), qa[ks][0], qa[ks][1], qa[ks][2],
                qa[ks][3]);
  }

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};

  uint32_t stage = 0, phase = 0;
  for (int t = 0; t < n_tiles; ++t) {
    const int t0 = k0 + t * kAttnTileKeys;
    const int nvalid = min(kAttnTileKeys, k1 - t0) - kp * KP;   // valid keys of this part
    if (!mbar_wait(&full[stage], phase, p.err)) break;
    if (nvalid > 0) {
      const uint32_t kbase = smem_u32(sK + stage * C::kKVBytes);
      const uint32_t vbase = smem_u32(sV + stage * C::kKVBytes);
      if (nvalid < KP && (nvalid & 15)) {
        // Rows past the last key of a partly used page may hold anything
        // (including NaN bit patterns); zero them so that P = 0 rows add 0.
        const int jp = (kp * KP + nvalid) >> 4, r0 = nvalid & 15;
        uint8_t* vb = sV + stage * C::kKVBytes;
        const int n16 = (16 - r0) * C::kBoxesPerPage * 8;
        for (int e = lane; e < n16; e += 32) {
          const int hf = e / ((16 - r0) * 8);
          const int rem = e - hf * (16 - r0) * 8;
          const int rr = r0 + rem / 8, cc = rem & 7;
          *reinterpret_cast<uint4*>(vb + (jp * C::kBoxesPerPage + hf) * C::kBoxBytes +
                                    rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }

      // S = Q K^T over this part's keys
      float s[NB][4];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        if constexpr (NB >= 2) {
#pragma unroll
          for (int nbp = 0; nbp < NB / 2; ++nbp) {
            const int j = lane >> 3;
            const int kt = kp * KP + (nbp * 2 + (j >> 1)) * 8 + (lane & 7);
            const int c = ks * 2 + (j & 1);
            uint32_t b00, b01, b10, b11;
            ldmatrix_x4(kbase + kv_off<D>(kt, c), b00, b01, b10, b11);
            mma_bf16_16816(s[2 * nbp], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b00, b01);
            mma_bf16_16816(s[2 * nbp + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b10,
                           b11);
          }
        }
      }

      // scale into the log2 domain, mask keys past the range, online softmax
      float mx[2] = {m_run[0], m_run[1]};
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kt = nb * 8 + 2 * (lane & 3) + (e & 1);
          const float v = s[nb][e] * p.scale_log2;
          s[nb][e] = (kt < nvalid) ? v : -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], s[nb][e]);
        }
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
      }
      float ref[2], alpha[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        ref[hh] = (mx[hh] == -INFINITY) ? 0.f : mx[hh];
        alpha[hh] = exp2f(m_run[hh] - ref[hh]);  // m_run = -inf -> 0
        m_run[hh] = mx[hh];
        l_run[hh] *= alpha[hh];
      }
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o[i][0] *= alpha[0];
        o[i][1] *= alpha[0];
        o[i][2] *= alpha[1];
        o[i][3] *= alpha[1];
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pv = exp2f(s[nb][e] - ref[e >> 1]);
          s[nb][e] = pv;
          l_run[e >> 1] += pv;
        }
      }

      // O += P V, 16 keys (one page) per k-step.  P is split into bf16 hi + lo
      // parts (P = hi + lo to ~2^-17) so that the tensor-core product does not
      // add bf16 rounding of the probabilities to the output.
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        if (kk * 16 < nvalid) {
          uint32_t ah[4], al[4];
          split_bf16x2(s[2 * kk][0], s[2 * kk][1], ah[0], al[0]);
          split_bf16x2(s[2 * kk][2], s[2 * kk][3], ah[1], al[1]);
          split_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1], ah[2], al[2]);
          split_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3], ah[3], al[3]);
#pragma unroll
          for (int dbp = 0; dbp < D / 16; ++dbp) {
            const int j = lane >> 3;
            const int kt = kp * KP + kk * 16 + (j & 1) * 8 + (lane & 7);
            const int c = dbp * 2 + (j >> 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(vbase + kv_off<D>(kt, c), b0, b1, b2, b3);
            mma_bf16_16816(o[2 * dbp], ah[0], ah[1], ah[2], ah[3], b0, b1);
            mma_bf16_16816(o[2 * dbp + 1], ah[0], ah[1], ah[2], ah[3], b2, b3);
            mma_bf16_16816(o[2 * dbp], al[0], al[1], al[2], al[3], b0, b1);
            mma_bf16_16816(o[2 * dbp + 1], al[0], al[1], al[2], al[3], b2, b3);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    if (++stage == kAttnStages) {
      stage = 0;
      phase ^= 1u;
    }
  }

#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 1);
    l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 2);
  }

  if (p.key_parts > 1) {
    // merge the key parts of each row group through the (now idle) stage buffers
    named_bar_sync(1, nwc * 32);
    float* mo = reinterpret_cast<float*>(smem);
    float* mml = mo + (p.key_parts - 1) * p.row_groups * 16 * D;
    if (kp > 0) {
      const int slot = (kp - 1) * p.row_groups + rg;
      float* dst = mo + static_cast<size_t>(slot) * 16 * D;
#pragma unroll
      for (int db = 0; db < D / 8; ++db)
        *reinterpret_cast<float4*>(dst + (db * 32 + lane) * 4) =
            make_float4(o[db][0], o[db][1], o[db][2], o[db][3]);
      *reinterpret_cast<float4*>(mml + (slot * 32 + lane) * 4) =
          make_float4(m_run[0], m_run[1], l_run[0], l_run[1]);
    }
    named_bar_sync(1, nwc * 32);
    if (kp > 0) return;
    for (int j = 1; j < p.key_parts; ++j) {
      const int slot = (j - 1) * p.row_groups + rg;
      const float4 ml = *reinterpret_cast<const float4*>(mml + (slot * 32 + lane) * 4);
      const float mj[2] = {ml.x, ml.y}, lj[2] = {ml.z, ml.w};
      float a_self[2], a_other[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float mm = fmaxf(m_run[hh], mj[hh]);
        const float rf = (mm == -INFINITY) ? 0.f : mm;
        a_self[hh] = exp2f(m_run[hh] - rf);
        a_other[hh] = exp2f(mj[hh] - rf);
        l_run[hh] = l_run[hh] * a_self[hh] + lj[hh] * a_other[hh];
        m_run[hh] = mm;
      }
      const float* src = mo + static_cast<size_t>(slot) * 16 * D;
#pragma unroll
      for (int db = 0; db < D / 8; ++db) {
        const float4 v = *reinterpret_cast<const float4*>(src + (db * 32 + lane) * 4);
        o[db][0] = o[db][0] * a_self[0] + v.x * a_other[0];
        o[db][1] = o[db][1] * a_self[0] + v.y * a_other[0];
        o[db][2] = o[db][2] * a_self[1] + v.z * a_other[1];
        o[db][3] = o[db][3] * a_self[1] + v.w * a_other[1];
      }
    }
  }

#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int r = rg * 16 + (lane >> 2) + hh * 8;
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
            make_float2(m_run[hh], l_run[hh]);
      }
    }
  }
}

// Merge the split partials of requests that needed more than one split:
//   m = max_s m_s,  w_s = 2^(m_s - m),  o = sum_s w_s O_s / sum_s w_s l_s
// One warp per (request, kv head, query row); splits are summed in index order.
template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnParams p) {
  constexpr int PER = D / 32;   // elements of the row per lane
  pdl_trigger();
  pdl_wait();
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.B * p.Hkv * p.R) return;
  const int r = gw % p.R;
  const int h = (gw / p.R) % p.Hkv;
  const int b = gw / (p.R * p.Hkv);
  const int n_keys = p.seq_lens[b] + p.bs;
  const int ns = min((n_keys + p.chunk_keys - 1) / p.chunk_keys, p.max_splits);
  if (ns <= 1) return;
  auto row_of = [&](int s) {
    return ((static_cast<size_t>(s) * p.B + b) * p.Hkv + h) * p.R + r;
  };
  // The (m, l) pairs of the first 32 splits are read lane-parallel and the
  // first kGroup splits' rows are requested at the same time, before the
  // maximum is known, so that a row with up to kGroup splits costs one round
  // trip to memory; more splits follow in groups of kGroup, in index order.
  constexpr int kGroup = 8;
  auto load_row = [&](int s, float* v) {
    const float* src = p.part_o + row_of(s) * D + lane * PER;
    if constexpr (PER == 4) {
      const float4 q = *reinterpret_cast<const float4*>(src);
      v[0] = q.x;
      v[1] = q.y;
      v[2] = q.z;
      v[3] = q.w;
    } else {
      const float2 q = *reinterpret_cast<const float2*>(src);
      v[0] = q.x;
      v[1] = q.y;
    }
  };
  float2 ml0 = make_float2(-INFINITY, 0.f);
  if (lane < ns) ml0 = *reinterpret_cast<const float2*>(p.part_ml + row_of(lane) * 2);
  float v[kGroup][PER];
#pragma unroll
  for (int u = 0; u < kGroup; ++u) {
    if (u < ns) {
      load_row(u, v[u]);
    } else {
#pragma unroll
      for (int e = 0; e < PER; ++e) v[u][e] = 0.f;
    }
  }
  float mmax = ml0.x;
  for (int s = lane + 32; s < ns; s += 32) mmax = fmaxf(mmax, p.part_ml[row_of(s) * 2]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, off));
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float l = 0.f;
  for (int s0 = 0; s0 < ns; s0 += 32) {
    float w = 0.f, wl = 0.f;
    if (s0 + lane < ns) {
      const float2 ml = s0 == 0 ? ml0
                                : *reinterpret_cast<const float2*>(p.part_ml + row_of(s0 + lane) * 2);
      w = exp2f(ml.x - mmax);
      wl = w * ml.y;
    }
    l += wl;
    const int cnt = min(32, ns - s0);
    for (int j = 0; j < cnt; j += kGroup) {
      if (s0 > 0 || j > 0) {
#pragma unroll
        for (int u = 0; u < kGroup; ++u)
          if (j + u < cnt) load_row(s0 + j + u, v[u]);
      }
#pragma unroll
      for (int u = 0; u < kGroup; ++u) {
        const float wsu = __shfl_sync(0xffffffffu, w, (j + u) & 31);
        if (j + u < cnt) {
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[e] += wsu * v[u][e];
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  const float inv = 1.f / l;
  const int i = r / p.G, g = r - (r / p.G) * p.G;
  f16* dst = p.o + (static_cast<size_t>(b * p.bs + i) * p.Hq + h * p.G + g) * D + lane * PER;
  if constexpr (PER == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_f16x2(acc[0] * inv, acc[1] * inv),
                                                pack_f16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_f16x2(acc[0] * inv, acc[1] * inv);
  }
}

}  // namespace dflash
