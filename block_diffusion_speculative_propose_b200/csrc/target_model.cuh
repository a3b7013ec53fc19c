// target_model.cuh — a small Qwen3-style causal target model on the GPU, with
// the auxiliary hidden-state capture that DFlash consumes ("DFlash
// Speculative Decoding in the vLLM Neuron Framework", §Target Auxiliary Hidden
// State Extraction): during the forward, the pre-layer residual states at the
// requested capture layers are written, concatenated in request order, as the
// bf16 [n, n_capture * hidden] input of the context-KV injection.
//
// It exists so that the whole speculative loop (target forward -> greedy
// verification -> injection -> proposal) runs on the device and can be checked
// for losslessness against plain greedy decoding of the same target.  Its
// design goal is therefore exact reproducibility, not speed: every output
// element of every kernel is reduced in one fixed order that does not depend on
// how many rows a call processes, so a token at a given position gets
// bit-identical logits whether it is decoded alone or inside a block of
// verified rows.  fp32 weights and activations throughout.
//
// One sequence per model instance; its K/V cache is [n_layers][max_len][Hkv][d]
// fp32, owned by the instance.  A forward over tokens at positions
// [start, start + n) writes their K/V and attends causally over [0, pos].
#pragma once

#include "dflash_device.cuh"

namespace dflash {

struct TargetDims {
  int H, Hq, Hkv, D, I, V, max_len;
  float eps, theta;
};

// x[r] = embed[tokens[r]] (fp32 rows); a token outside [0, V) gives a zero row
// and sets DFLASH_DEVERR_TOKEN.
__global__ void target_embed_kernel(const int32_t* __restrict__ tokens, const float* __restrict__ embed,
                                    int H, int V, float* __restrict__ x, unsigned* err) {
  const int r = blockIdx.x;
  const int tok = tokens[r];
  const bool ok = tok >= 0 && tok < V;
  if (!ok && threadIdx.x == 0) raise_error(err, DFLASH_DEVERR_TOKEN);
  for (int i = threadIdx.x; i < H; i += blockDim.x)
    x[static_cast<size_t>(r) * H + i] = ok ? embed[static_cast<size_t>(tok) * H + i] : 0.f;
}

// Fixed-order block reduction of 256 threads (tree over the thread index).
__device__ __forceinline__ float block_sum_fixed(float v, float* red) {
  red[threadIdx.x] = v;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  const float out = red[0];
  __syncthreads();
  return out;
}

// y[r] = x[r] / sqrt(mean(x[r]^2) + eps) * w   (256 threads per row)
__global__ void __launch_bounds__(256) target_rmsnorm_kernel(const float* __restrict__ x,
                                                             const float* __restrict__ w, int H,
                                                             float eps, float* __restrict__ y) {
  __shared__ float red[256];
  const size_t r = blockIdx.x;
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += blockDim.x) {
    const float v = x[r * H + i];
    ss += v * v;
  }
  ss = block_sum_fixed(ss, red);
  const float inv = rsqrtf(ss / H + eps);
  for (int i = threadIdx.x; i < H; i += blockDim.x) y[r * H + i] = x[r * H + i] * inv * w[i];
}

// out[r][j] (+)= sum_k a[r][k] * W[j][k]; one warp per output element, lanes
// stride k, then a fixed butterfly.  accumulate: out += result (residual add).
__global__ void __launch_bounds__(256) target_linear_kernel(const float* __restrict__ a,
                                                            const float* __restrict__ W, int N,
                                                            int K, float* __restrict__ out,
                                                            int accumulate) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + warp;
  const size_t r = blockIdx.y;
  if (j >= N) return;
  const float* ar = a + r * K;
  const float* wr = W + static_cast<size_t>(j) * K;
  float s = 0.f;
  for (int k = lane; k < K; k += 32) s = fmaf(ar[k], wr[k], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    float* dst = out + r * N + j;
    *dst = accumulate ? *dst + s : s;
  }
}

// h[r][i] = silu(gu[r][i]) * gu[r][I + i]   (gate | up stacked in one row)
__global__ void target_swiglu_kernel(const float* __restrict__ gu, int I, int rows,
                                     float* __restrict__ h) {
  const size_t n = static_cast<size_t>(rows) * I;
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = e / I, i = e - r * I;
    const float g = gu[r * 2 * I + i], u = gu[r * 2 * I + I + i];
    h[e] = g / (1.f + expf(-g)) * u;
  }
}

// Rotate-half RoPE of one head vector held by one warp (d/2 pairs, lane
// strided), angle pos * theta^(-2i/d) evaluated in double precision.
__device__ __forceinline__ void target_rope_warp(float* v, int D, int pos, float theta) {
  const int half = D / 2;
  for (int i = threadIdx.x & 31; i < half; i += 32) {
    const double ang = static_cast<double>(pos) * pow(static_cast<double>(theta), -2.0 * i / D);
    double sn, cs;
    sincos(ang, &sn, &cs);
    const float c = static_cast<float>(cs), s = static_cast<float>(sn);
    const float x1 = v[i], x2 = v[i + half];
    v[i] = x1 * c - x2 * s;
    v[i + half] = x2 * c + x1 * s;
  }
}

// Per row r and head: q/k RMSNorm over d (fixed-order warp sum), RoPE at
// position start + r; q to qout, k and v into the layer's cache at that
// position.  qkv row layout: [q (Hq*D) | k (Hkv*D) | v (Hkv*D)].  One warp per
// (row, head), heads 0..Hq-1 are q, Hq..Hq+Hkv-1 are k (v copied alongside).
__global__ void __launch_bounds__(256) target_qkv_kernel(const float* __restrict__ qkv, int rows,
                                                         int start, TargetDims d,
                                                         const float* __restrict__ qn,
                                                         const float* __restrict__ kn,
                                                         float* __restrict__ qout,
                                                         float* __restrict__ kcache,
                                                         float* __restrict__ vcache,
                                                         unsigned* err) {
  __shared__ float buf[8][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x * 8 + warp;
  const int heads = d.Hq + d.Hkv;
  if (item >= rows * heads) return;
  const int r = item / heads, hh = item - r * heads;
  const int pos = start + r;
  const bool is_q = hh < d.Hq;
  const float* src = qkv + static_cast<size_t>(r) * (d.Hq + 2 * d.Hkv) * d.D + hh * d.D;
  float* v = buf[warp];
  float ss = 0.f;
  for (int i = lane; i < d.D; i += 32) {
    v[i] = src[i];
    ss += v[i] * v[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = rsqrtf(ss / d.D + d.eps);
  const float* w = is_q ? qn : kn;
  for (int i = lane; i < d.D; i += 32) v[i] = v[i] * inv * w[i];
  __syncwarp();
  target_rope_warp(v, d.D, pos, d.theta);
  __syncwarp();
  if (is_q) {
    float* dst = qout + (static_cast<size_t>(r) * d.Hq + hh) * d.D;
    for (int i = lane; i < d.D; i += 32) dst[i] = v[i];
    return;
  }
  if (pos < 0 || pos >= d.max_len) {
    if (lane == 0) raise_error(err, DFLASH_DEVERR_POSITION);
    return;
  }
  const int kh = hh - d.Hq;
  const size_t slot = (static_cast<size_t>(pos) * d.Hkv + kh) * d.D;
  const float* vsrc = src + d.Hkv * d.D;   // the v head of the same kv head
  for (int i = lane; i < d.D; i += 32) {
    kcache[slot + i] = v[i];
    vcache[slot + i] = vsrc[i];
  }
}

// Causal attention: one warp per (row, q head) over keys [0, start + r], in
// key order, online softmax in fp32, scale 1/sqrt(d).  Each lane holds d/32
// output dims.
__global__ void __launch_bounds__(256) target_attention_kernel(const float* __restrict__ q, int rows,
                                                               int start, TargetDims d,
                                                               const float* __restrict__ kcache,
                                                               const float* __restrict__ vcache,
                                                               float* __restrict__ o) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x * 8 + warp;
  if (item >= rows * d.Hq) return;
  const int r = item / d.Hq, h = item - r * d.Hq;
  const int kvh = h / (d.Hq / d.Hkv);
  const int pos = start + r;
  if (pos < 0 || pos >= d.max_len) return;   // flagged by target_qkv_kernel
  const float* qr = q + (static_cast<size_t>(r) * d.Hq + h) * d.D;
  const float scale = rsqrtf(static_cast<float>(d.D));
  constexpr int kMaxPer = 4;                  // d <= 128
  float acc[kMaxPer] = {0.f, 0.f, 0.f, 0.f};
  float m = -INFINITY, l = 0.f;
  const int per = d.D / 32;
  for (int j = 0; j <= pos; ++j) {
    const float* kr = kcache + (static_cast<size_t>(j) * d.Hkv + kvh) * d.D;
    float s = 0.f;
    for (int i = lane; i < d.D; i += 32) s = fmaf(qr[i], kr[i], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    s *= scale;
    const float mn = fmaxf(m, s);
    const float a = expf(m - mn), p = expf(s - mn);
    l = l * a + p;
    const float* vr = vcache + (static_cast<size_t>(j) * d.Hkv + kvh) * d.D;
    for (int t = 0; t < per; ++t) acc[t] = acc[t] * a + p * vr[lane + 32 * t];
    m = mn;
  }
  float* dst = o + (static_cast<size_t>(r) * d.Hq + h) * d.D;
  for (int t = 0; t < per; ++t) dst[lane + 32 * t] = acc[t] / l;
}

// aux[r][c * H + i] = bf16(x[r][i]): the residual state at capture slot c.
__global__ void target_capture_kernel(const float* __restrict__ x, int rows, int H, int n_capture,
                                      int c, bf16* __restrict__ aux) {
  const size_t n = static_cast<size_t>(rows) * H;
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = e / H, i = e - r * H;
    aux[r * static_cast<size_t>(n_capture) * H + static_cast<size_t>(c) * H + i] =
        __float2bfloat16_rn(x[e]);
  }
}

}  // namespace dflash
