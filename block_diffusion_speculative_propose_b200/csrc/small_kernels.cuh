// small_kernels.cuh — the light kernels around the GEMMs and attention:
// block build + embedding + first RMSNorm, row RMSNorms, the draft-token
// finalisation, greedy verification, paged-slot mapping and the RoPE table.
#pragma once

#include "dflash_device.cuh"

namespace dflash {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}
// Sum over the block (blockDim.x a multiple of 32, <= 1024); every thread gets it.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = warp_sum(v);
  __syncthreads();  // red may still be read by a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = (lane < (blockDim.x >> 5)) ? red[lane] : 0.f;
  return warp_sum(t);
}

// Block construction ([bonus, mask, ..., mask] per request), embedding with
// the target table, and the first layer's input RMSNorm.
//   x[r, :]   = embed[id_r, :]                       (fp32 residual stream)
//   nrm[r, :] = fp16(x * rsqrt(mean(x^2) + eps) * w)
// Also clears the LM-head argmax keys of the call.
__global__ void __launch_bounds__(256) embed_norm_kernel(
    const int32_t* __restrict__ bonus, int mask_id, const bf16* __restrict__ embed,
    const bf16* __restrict__ w, float* __restrict__ x, f16* __restrict__ nrm,
    unsigned long long* __restrict__ keys, int n_keys, int bs, int H, int V, float eps,
    unsigned* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int r = blockIdx.x;
  const int b = r / bs, i = r - (r / bs) * bs;
  int tok = (i == 0) ? bonus[b] : mask_id;
  if (tok < 0 || tok >= V) {
    if (threadIdx.x == 0) raise_error(err, DFLASH_DEVERR_TOKEN);
    tok = 0;
  }
  if (threadIdx.x == 0 && r < n_keys) keys[r] = 0ull;
  const bf16* e = embed + static_cast<size_t>(tok) * H;
  float* xr = x + static_cast<size_t>(r) * H;
  float ss = 0.f;
  for (int j = threadIdx.x * 8; j < H; j += blockDim.x * 8) {
    const uint4 q = *reinterpret_cast<const uint4*>(e + j);
    const bf16* qb = reinterpret_cast<const bf16*>(&q);
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[k] = bf2f(qb[k]);
      ss += v[k] * v[k];
    }
    *reinterpret_cast<float4*>(xr + j) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(xr + j + 4) = make_float4(v[4], v[5], v[6], v[7]);
  }
  ss = block_sum(ss, red);
  const float rinv = rsqrtf(ss / H + eps);
  f16* nr = nrm + static_cast<size_t>(r) * H;
  for (int j = threadIdx.x * 8; j < H; j += blockDim.x * 8) {
    const uint4 q = *reinterpret_cast<const uint4*>(e + j);
    const uint4 wq = *reinterpret_cast<const uint4*>(w + j);
    const bf16* qb = reinterpret_cast<const bf16*>(&q);
    const bf16* wb = reinterpret_cast<const bf16*>(&wq);
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      ow[k] = pack_f16x2(bf2f(qb[2 * k]) * rinv * bf2f(wb[2 * k]),
                         bf2f(qb[2 * k + 1]) * rinv * bf2f(wb[2 * k + 1]));
    *reinterpret_cast<uint4*>(nr + j) = o;
  }
}

// out[r, :] = fp16(x[src(r), :] * rsqrt(mean(x^2) + eps) * w)  (RMSNorm outputs are
// bounded by sqrt(H) * max|w|, so fp16 holds them with 8x finer rounding than bf16).
// With gather_k > 0, src(r) = (r / gather_k) * bs + 1 + r % gather_k: the block
// slots 1..bs-1 of each request (keep_idx), packed densely.
__global__ void __launch_bounds__(256) rmsnorm_rows_kernel(
    const float* __restrict__ x, const bf16* __restrict__ w, f16* __restrict__ out, int H,
    float eps, int gather_k, int bs) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int r = blockIdx.x;
  const int src = gather_k > 0 ? (r / gather_k) * bs + 1 + (r - (r / gather_k) * gather_k) : r;
  const float* xr = x + static_cast<size_t>(src) * H;
  float ss = 0.f;
  for (int j = threadIdx.x * 8; j < H; j += blockDim.x * 8) {
    const float4 a = *reinterpret_cast<const float4*>(xr + j);
    const float4 c = *reinterpret_cast<const float4*>(xr + j + 4);
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w + c.x * c.x + c.y * c.y + c.z * c.z +
          c.w * c.w;
  }
  ss = block_sum(ss, red);
  const float rinv = rsqrtf(ss / H + eps);
  f16* orow = out + static_cast<size_t>(r) * H;
  for (int j = threadIdx.x * 8; j < H; j += blockDim.x * 8) {
    const float4 a = *reinterpret_cast<const float4*>(xr + j);
    const float4 c = *reinterpret_cast<const float4*>(xr + j + 4);
    const uint4 wq = *reinterpret_cast<const uint4*>(w + j);
    const bf16* wb = reinterpret_cast<const bf16*>(&wq);
    uint4 o;
    o.x = pack_f16x2(a.x * rinv * bf2f(wb[0]), a.y * rinv * bf2f(wb[1]));
    o.y = pack_f16x2(a.z * rinv * bf2f(wb[2]), a.w * rinv * bf2f(wb[3]));
    o.z = pack_f16x2(c.x * rinv * bf2f(wb[4]), c.y * rinv * bf2f(wb[5]));
    o.w = pack_f16x2(c.z * rinv * bf2f(wb[6]), c.w * rinv * bf2f(wb[7]));
    *reinterpret_cast<uint4*>(orow + j) = o;
  }
}

// Tensor-parallel residual add: x[src(r)] += part[src(r)] (the all-reduced sum
// of every rank's row-parallel O or down projection), then out[r] = fp16 of
// RMSNorm(x[src(r)]) * w exactly as rmsnorm_rows_kernel (same src(r) rule).
__global__ void __launch_bounds__(256) add_rmsnorm_rows_kernel(
    float* __restrict__ x, const float* __restrict__ part, const bf16* __restrict__ w,
    f16* __restrict__ out, int H, float eps, int gather_k, int bs) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int r = blockIdx.x;
  const int src = gather_k > 0 ? (r / gather_k) * bs + 1 + (r - (r / gather_k) * gather_k) : r;
  float* xr = x + static_cast<size_t>(src) * H;
  const float* pr = part + static_cast<size_t>(src) * H;
  float ss = 0.f;
  for (int j = threadIdx.x * 4; j < H; j += blockDim.x * 4) {
    float4 a = *reinterpret_cast<const float4*>(xr + j);
    const float4 c = *reinterpret_cast<const float4*>(pr + j);
    a.x += c.x;
    a.y += c.y;
    a.z += c.z;
    a.w += c.w;
    *reinterpret_cast<float4*>(xr + j) = a;
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
  }
  ss = block_sum(ss, red);
  const float rinv = rsqrtf(ss / H + eps);
  f16* orow = out + static_cast<size_t>(r) * H;
  for (int j = threadIdx.x * 4; j < H; j += blockDim.x * 4) {
    const float4 a = *reinterpret_cast<const float4*>(xr + j);
    const uint2 wq = *reinterpret_cast<const uint2*>(w + j);
    const bf16* wb = reinterpret_cast<const bf16*>(&wq);
    uint2 o;
    o.x = pack_f16x2(a.x * rinv * bf2f(wb[0]), a.y * rinv * bf2f(wb[1]));
    o.y = pack_f16x2(a.z * rinv * bf2f(wb[2]), a.w * rinv * bf2f(wb[3]));
    *reinterpret_cast<uint2*>(orow + j) = o;
  }
}

// drafts[b, i] = argmax of LM-head row (b, i); block[b] = [bonus_b, drafts[b]].
__global__ void argmax_finalize_kernel(const unsigned long long* __restrict__ keys,
                                       const int32_t* __restrict__ bonus,
                                       int32_t* __restrict__ drafts,
                                       int32_t* __restrict__ block, int B, int bs) {
  pdl_trigger();
  pdl_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * bs) return;
  const int K = bs - 1;
  const int b = idx / bs, i = idx - (idx / bs) * bs;
  int32_t tok;
  if (i == 0) {
    tok = bonus[b];
  } else {
    tok = static_cast<int32_t>(argmax_key_index(keys[b * K + i - 1]));
    drafts[b * K + i - 1] = tok;
  }
  if (block) block[idx] = tok;
}

// A vocabulary shard's ordered argmax keys as signed 64-bit integers: each key
// with its top bit flipped, so that the signed maximum over shards (an
// all-reduce MAX over int64) is the unsigned maximum — the largest logit, and
// among equal logits the lowest vocabulary id.
__global__ void keys_export_kernel(const unsigned long long* __restrict__ keys, int n,
                                   int64_t* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = static_cast<int64_t>(keys[i] ^ 0x8000000000000000ull);
}

// Drafts from exported keys (their maximum over the shards); block[b] =
// [bonus_b, drafts[b]].  A key naming no vocabulary entry (no shard wrote the
// row, or an id >= vocab) gives -1 and sets DFLASH_DEVERR_INPUT.
__global__ void draft_keys_finalize_kernel(const int64_t* __restrict__ keys,
                                           const int32_t* __restrict__ bonus, int B, int bs,
                                           int vocab, int32_t* __restrict__ drafts,
                                           int32_t* __restrict__ block, unsigned* err) {
  pdl_trigger();
  pdl_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * bs) return;
  const int K = bs - 1;
  const int b = idx / bs, i = idx - (idx / bs) * bs;
  int32_t tok;
  if (i == 0) {
    tok = bonus[b];
  } else {
    const unsigned long long u =
        static_cast<unsigned long long>(keys[b * K + i - 1]) ^ 0x8000000000000000ull;
    const uint32_t id = argmax_key_index(u);
    if (u == 0ull || id >= static_cast<uint32_t>(vocab)) {
      raise_error(err, DFLASH_DEVERR_INPUT);
      tok = -1;
    } else {
      tok = static_cast<int32_t>(id);
    }
    drafts[b * K + i - 1] = tok;
  }
  if (block) block[idx] = tok;
}

// Greedy verification, pass 1: per (row, chunk) ordered argmax key of the fp32
// target logits.  Rows are [B * (K+1)], each V long.
__global__ void __launch_bounds__(256) verify_partial_kernel(
    const float* __restrict__ logits, int V, int chunk_len, int chunks, int rows,
    unsigned long long* __restrict__ part) {
  pdl_trigger();
  pdl_wait();
  __shared__ unsigned long long red[32];
  // grid.y is capped at 65535: CTAs step over the rows
  for (size_t row = blockIdx.y; row < static_cast<size_t>(rows); row += gridDim.y) {
  const int beg = blockIdx.x * chunk_len;
  const int end = min(V, beg + chunk_len);
  const float* src = logits + row * static_cast<size_t>(V);
  // Each thread visits its elements in increasing index order and keeps the
  // first largest (strict compare: NaN never wins, so it counts as -inf; -0
  // ties +0; ties keep the lower index); its result enters the ordered 64-bit
  // key once.  A thread that sees only -inf / NaN reports -inf at its first
  // index, which is what the key order picks among them.
  float bv = -INFINITY;
  int bi = -1;
  auto take = [&](float v, int j) {
    const bool gt = v > bv;
    bv = gt ? v : bv;
    bi = gt ? j : bi;
  };
  if ((V & 3) == 0) {
    // four 16-byte loads in flight per thread (a row is streamed once)
    constexpr int U = 4;
    const int step = blockDim.x * 4;
    int j = beg + threadIdx.x * 4;
    if (j < end) bi = j;
    for (; j + (U - 1) * step < end; j += U * step) {
      float4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = __ldcs(reinterpret_cast<const float4*>(src + j + u * step));
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int jj = j + u * step;
        take(v[u].x, jj);
        take(v[u].y, jj + 1);
        take(v[u].z, jj + 2);
        take(v[u].w, jj + 3);
      }
    }
    for (; j < end; j += step) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(src + j));
      take(v.x, j);
      take(v.y, j + 1);
      take(v.z, j + 2);
      take(v.w, j + 3);
    }
  } else {
    int j = beg + threadIdx.x;
    if (j < end) bi = j;
    for (; j < end; j += blockDim.x) take(__ldcs(src + j), j);
  }
  unsigned long long best = bi >= 0 ? argmax_key(bv, static_cast<uint32_t>(bi)) : 0ull;
  best = warp_max_u64(best);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = best;
  __syncthreads();
  if (warp == 0) {
    unsigned long long t = lane < (blockDim.x >> 5) ? red[lane] : 0ull;
    t = warp_max_u64(t);
    if (lane == 0) part[row * chunks + blockIdx.x] = t;
  }
  __syncthreads();   // red[] is reused by the next row
  }
}

// Pass 2 (one CTA per request, one warp per target row): t_j for j = 0..K,
// longest matching prefix, bonus, and the -1 padded output row.
__global__ void __launch_bounds__(256) verify_final_kernel(
    const unsigned long long* __restrict__ part, int chunks,
    const int32_t* __restrict__ drafts, int K, int32_t* __restrict__ out,
    int32_t* __restrict__ n_acc, int32_t* __restrict__ bonus) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t t[130];
  __shared__ int32_t d[130];
  __shared__ int n_sh;
  const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  for (int j = threadIdx.x; j < K; j += blockDim.x) d[j] = drafts[static_cast<size_t>(b) * K + j];
  for (int j = warp; j <= K; j += nw) {
    const unsigned long long* pr = part + (static_cast<size_t>(b) * (K + 1) + j) * chunks;
    unsigned long long best = 0ull;
    for (int c = lane; c < chunks; c += 32) best = pr[c] > best ? pr[c] : best;
    best = warp_max_u64(best);
    if (lane == 0) t[j] = static_cast<int32_t>(argmax_key_index(best));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    while (n < K && d[n] == t[n]) ++n;
    n_sh = n;
    n_acc[b] = n;
    bonus[b] = t[n];
  }
  __syncthreads();
  const int n = n_sh;
  for (int j = threadIdx.x; j <= K; j += blockDim.x) {
    int32_t v = -1;
    if (j < n) v = d[j];
    else if (j == n) v = t[n];
    out[static_cast<size_t>(b) * (K + 1) + j] = v;
  }
}

// slots[i] = block_table[req * W + min(pos / P, W - 1)] * P + pos % P
__global__ void paged_slots_kernel(const int64_t* __restrict__ pos,
                                   const int64_t* __restrict__ req,
                                   const int32_t* __restrict__ table, int n, int W, int P,
                                   int64_t* __restrict__ slots) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t p = pos[i];
  if (p < 0) {
    slots[i] = -1;
    return;
  }
  int64_t pg = p / P;
  if (pg > W - 1) pg = W - 1;
  const int64_t page = table[req[i] * W + pg];
  slots[i] = page * P + (p - (p / P) * P);
}

// In-place bf16 -> fp16 conversion of weights (exact in fp16's normal range).
// Proposal-input preparation with the async rejection correction: threads
// r < n handle target rows, threads b < B handle requests; nothing is shared
// between threads (each recomputes the few per-request counts it needs).
__device__ __forceinline__ int count_valid(const int32_t* s, int width, int vocab) {
  int c = 0;
  for (int j = 0; j < width; ++j) c += (s[j] != -1 && s[j] < vocab) ? 1 : 0;
  return c;
}

__global__ void prepare_proposal_kernel(
    const int64_t* __restrict__ target_positions, int n, const int32_t* __restrict__ last, int B,
    const int32_t* __restrict__ cur_sampled, int cur_width, const int32_t* __restrict__ cur_num_draft,
    const int32_t* __restrict__ prev_sampled, int prev_width,
    const int32_t* __restrict__ prev_num_draft, const int32_t* __restrict__ table, int W, int P,
    int vocab, int64_t* __restrict__ pos_out, int64_t* __restrict__ slot_out,
    int32_t* __restrict__ seq_out, int32_t* __restrict__ bonus_out, unsigned* err) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  auto prev_rejected = [&](int b) -> int {
    if (!prev_sampled) return 0;
    return 1 + prev_num_draft[b] -
           count_valid(prev_sampled + static_cast<size_t>(b) * prev_width, prev_width, vocab);
  };
  if (t < n) {
    // request of row t: first b with last[b] >= t (binary search)
    int lo = 0, hi = B;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (last[mid] >= t) hi = mid;
      else lo = mid + 1;
    }
    const int64_t p_in = target_positions[t];
    if (lo >= B) {
      pos_out[t] = p_in;      // trailing padding row
      slot_out[t] = -1;
    } else {
      const int64_t p = p_in - prev_rejected(lo);
      pos_out[t] = p;
      if (p < 0) {
        raise_error(err, DFLASH_DEVERR_INPUT);
        slot_out[t] = -1;
      } else {
        const int64_t page_no = min(p / P, static_cast<int64_t>(W - 1));
        const int64_t block = table[static_cast<int64_t>(lo) * W + page_no];
        slot_out[t] = block * P + p % P;
      }
    }
  }
  if (t < B) {
    const int lt = last[t];
    if (lt >= n || lt < 0 || (t > 0 && last[t - 1] >= lt)) {
      raise_error(err, DFLASH_DEVERR_INPUT);
      seq_out[t] = 0;
      bonus_out[t] = -1;
      return;
    }
    const int32_t* cs = cur_sampled + static_cast<size_t>(t) * cur_width;
    const int cur_rej = 1 + cur_num_draft[t] - count_valid(cs, cur_width, vocab);
    const int64_t last_pos = target_positions[lt] - prev_rejected(t);
    seq_out[t] = static_cast<int32_t>(last_pos + 1 - cur_rej);
    int bonus = -1;
    for (int j = 0; j < cur_width; ++j)
      if (cs[j] != -1 && cs[j] < vocab) bonus = cs[j];
    if (bonus == -1) raise_error(err, DFLASH_DEVERR_INPUT);
    bonus_out[t] = bonus;
  }
}

// fp16 range statistics of converted weights: stats[0] = the largest |x| seen
// (float bits, which order like the values for x >= 0; NaN sorts above
// infinity), stats[1] = the number of nonzero values below fp16's smallest
// normal number (2^-14), which fp16 holds only as subnormals.
__device__ __forceinline__ void range_stats_add(unsigned* stats, unsigned amax_bits,
                                                unsigned small) {
  __shared__ unsigned s_max, s_small;
  if (threadIdx.x == 0) {
    s_max = 0u;
    s_small = 0u;
  }
  __syncthreads();
  for (int o = 16; o > 0; o >>= 1) {
    amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, o));
    small += __shfl_xor_sync(0xffffffffu, small, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicMax(&s_max, amax_bits);
    atomicAdd(&s_small, small);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicMax(&stats[0], s_max);
    atomicAdd(&stats[1], s_small);
  }
}

__global__ void bf16_to_f16_kernel(uint16_t* __restrict__ data, size_t n, unsigned* stats) {
  unsigned amax = 0u, small = 0u;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const bf16 v = *reinterpret_cast<const bf16*>(data + i);
    const float f = __bfloat162float(v);
    const unsigned a = __float_as_uint(f) & 0x7fffffffu;
    amax = max(amax, a);
    small += (a != 0u && a < 0x38800000u) ? 1u : 0u;   // 0 < |f| < 2^-14
    const f16 o = __float2half_rn(f);
    data[i] = *reinterpret_cast<const uint16_t*>(&o);
  }
  range_stats_add(stats, amax, small);
}

// Largest |x| of a bf16 vector into stats[2] (float bits, as above).
__global__ void absmax_bf16_kernel(const bf16* __restrict__ x, int n, unsigned* stats) {
  unsigned amax = 0u;
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    amax = max(amax, __float_as_uint(__bfloat162float(x[i])) & 0x7fffffffu);
  for (int o = 16; o > 0; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) atomicMax(&stats[2], amax);
}

// Tile-contiguous GEMM weight layout: the kPackRows x 64 tile (n_tile, k_block)
// of a row-major W [N, K] becomes one contiguous chunk (kPackRows rows of 128
// bytes, in order) at chunk index n_tile * (K / 64) + k_block; rows past N are
// zero.  Every TMA box of the weight stream is then a single contiguous read.
// The source rows are `ld` elements apart (a column slice of a wider matrix
// when ld > K; 16-byte aligned starts).
// With to_f16 the bf16 values are converted to fp16 on the way.
constexpr int kPackRows = 256;

__global__ void pack_tiles_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst,
                                  int N, int K, int ld, size_t units, int to_f16) {
  const int kb_count = K / 64;
  for (size_t u = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; u < units;
       u += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t chunk = u / (kPackRows * 8);
    const int within = static_cast<int>(u - chunk * (kPackRows * 8));
    const int r = within >> 3, j8 = within & 7;
    const int nt = static_cast<int>(chunk / kb_count);
    const int kb = static_cast<int>(chunk - static_cast<size_t>(nt) * kb_count);
    const int row = nt * kPackRows + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row < N)
      v = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(row) * ld + kb * 64 + j8 * 8);
    if (to_f16) {
      uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bf16* b2 = reinterpret_cast<const bf16*>(&w[q]);
        const f16 lo = __float2half_rn(__bfloat162float(b2[0]));
        const f16 hi = __float2half_rn(__bfloat162float(b2[1]));
        w[q] = static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&lo)) |
               (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&hi)) << 16);
      }
    }
    *reinterpret_cast<uint4*>(dst + u * 8) = v;
  }
}

// cos / sin of pos * theta^(-2j/D), evaluated in double, stored as fp32 pairs.
__global__ void rope_table_kernel(float2* __restrict__ table, int max_pos, int half,
                                  double theta) {
  const int pos = blockIdx.x;
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    const double inv = pow(theta, -2.0 * j / (2.0 * half));
    const double a = static_cast<double>(pos) * inv;
    table[static_cast<size_t>(pos) * half + j] =
        make_float2(static_cast<float>(cos(a)), static_cast<float>(sin(a)));
  }
}

// Diagnostics: one bounded wait that runs out.  Thread 0 initialises an
// mbarrier that expects one arrival and waits for its first phase with the
// pipelines' own bounded wait; nothing ever arrives, so the wait gives up after
// the device's wait limit and sets DFLASH_DEVERR_TIMEOUT in *err.  No fault, no
// trap: the kernel then returns normally.
__global__ void wait_timeout_selftest_kernel(unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait(&bar, 0, err);
  }
}

}  // namespace dflash
