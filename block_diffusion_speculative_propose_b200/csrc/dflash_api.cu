// dflash_api.cu — the C ABI declared in include/dflash.h: argument checking,
// handle / weight packing, launch planning (GEMM tiles and split-K, attention
// key splits), TMA descriptor construction and the launch sequences of
// inject / propose / verify.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <tuple>
#include <vector>

#include "attention.cuh"
#include "attention_tc.cuh"
#include "attention_tc2.cuh"
#include "dflash.h"
#include "gemm_tcgen05.cuh"
#include "gemm_pair.cuh"
#include "small_kernels.cuh"
#include "target_model.cuh"

using namespace dflash;

namespace {

constexpr int kCounterSlots = 1 << 16;
constexpr float kFp16Max = 65504.f;            // largest finite fp16
constexpr double kFp16SubnormalLimit = 0.01;   // fraction of fp16-subnormal weights refused
constexpr size_t kAlign = 256;

size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }
int cdiv(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------
// driver entry point for tensor-map encoding (no link-time libcuda dependency)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D view of 16-bit elements (bf16, or fp16 when f16) [rows][cols] (row pitch
// cols * 2 bytes), box [box_rows][64], 128-byte swizzle.  Out-of-range box
// rows read as zeros.
bool make_tmap(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols,
               uint32_t box_rows, bool f16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(ptr), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// GEMM planning
// ---------------------------------------------------------------------------
struct GemmPlan {
  int BN = 0, m_tiles = 0, n_tiles = 0, k_blocks = 0, tiles = 0, stream_k = 0, cluster_s = 1, ipc = 0,
      total_iters = 0, nacc = 1, nbuf = 2, tmem_cols = 32, grid = 0, a_rows = 128, stages = 1,
      smem = 0, slot_rows = 0;
  size_t partial_bytes = 0;
};

// A box / slot rows: all 128 once there is more than one M tile, else M
// rounded up to 16 (multiples of 8 rows keep every slot 1024-byte aligned).
int gemm_a_rows(int M) { return M >= kGemmBM ? kGemmBM : std::max(16, (M + 15) / 16 * 16); }

// Few-row (staged) GEMMs keep 4 stages in flight: measured on the Qwen3-8B
// draft step, 4 stages stream the weights faster than 5 or 6 (and 2 or 3).
constexpr int kGemmStagedStages = 4;

int gemm_stages(int a_rows, int bn) {
  int st = gemm_staged(a_rows) ? kGemmStagedStages : kGemmMaxStages;
  while (st > 2 && gemm_smem_bytes(a_rows, bn, st) > kGemmSmemLimit) --st;
  return st;
}

// Tile width, accumulator chains and schedule.  BN = 256.  One M tile (the
// weight-streaming regime, M <= 128): two accumulator chains in a single TMEM
// buffer, and stream-K (the (tile, k-block) iterations split evenly over the
// SMs) unless whole tiles already fill >= 90% of the last round.  Several M
// tiles (tensor-bound): 256-wide tiles, or 128-wide ones when only those fill
// >= 75% of the last round; double-buffered accumulator, whole tiles
// round-robin; stream-K only when the tiles cannot occupy half of the SMs.  force_bn /
// force_splits (0 = automatic) pin the tile width and the schedule: 1 = whole
// tiles, n >= 2 = stream-K with ceil(k_blocks / n) iterations per CTA.
//
// Few rows (the staged epilogue, M <= 32) and fewer tiles than SMs: cluster
// split-K with the largest cluster size S <= 8 (and <= the k-blocks) for which
// every tile's cluster is resident at once (cluster_cap[S] = clusters of S CTAs
// that fit on the GPU, 0 = unknown); with no such S, whole tiles when they
// occupy at least half of the SMs, else stream-K.
GemmPlan plan_gemm(int M, int N, int K, int group, int num_sms, int force_bn = 0,
                   int force_splits = 0, const int* cluster_cap = nullptr) {
  GemmPlan pl;
  pl.k_blocks = K / kGemmBK;
  pl.m_tiles = cdiv(M, kGemmBM);
  pl.BN = force_bn ? force_bn : 256;
  if (!force_bn && pl.m_tiles > 1 && group <= 128) {
    // several M tiles (tensor-bound): 128-wide tiles when only they fill the
    // SMs (e.g. 4 x 32 tiles of a 4096-wide output at 512 rows)
    auto util = [&](int bn) {
      const int t = pl.m_tiles * cdiv(N, bn);
      return static_cast<double>(t) / (static_cast<double>(cdiv(t, num_sms)) * num_sms);
    };
    if (util(256) < 0.75 && util(128) >= 0.75) pl.BN = 128;
  }
  if (pl.BN < group || pl.BN % group) pl.BN = 256;
  const bool one_m_tile = pl.m_tiles == 1;
  if (M <= kGemmStagedRows) {
    // staged epilogue: the accumulator is copied out at once (one buffer); the
    // weight stream, not the MMA chain, paces these tiles (one chain)
    pl.nacc = 1;
    pl.nbuf = 1;
  } else if (one_m_tile) {
    pl.nacc = pl.BN >= 256 ? 2 : 4;
    pl.nbuf = (2 * pl.nacc * pl.BN <= 512) ? 2 : 1;
  } else {
    pl.nacc = pl.BN >= 256 ? 1 : pl.BN >= 128 ? 2 : 4;
    pl.nbuf = 2;
  }
  pl.tmem_cols = 32;
  while (pl.tmem_cols < pl.nbuf * pl.nacc * pl.BN) pl.tmem_cols *= 2;
  pl.n_tiles = cdiv(N, pl.BN);
  pl.tiles = pl.m_tiles * pl.n_tiles;
  const int rounds = cdiv(pl.tiles, num_sms);
  const double fill = static_cast<double>(pl.tiles) / (static_cast<double>(rounds) * num_sms);
  bool sk = one_m_tile ? fill < 0.9 : 2 * pl.tiles < num_sms;
  if (force_splits == 1) sk = false;
  if (force_splits >= 2) sk = true;
  if (sk && pl.tiles > kCounterSlots - 2) sk = false;   // the last 2 slots: chain arrivals
  pl.total_iters = pl.tiles * pl.k_blocks;
  pl.a_rows = gemm_a_rows(M);
  if (!force_splits && cluster_cap && gemm_staged(pl.a_rows) && pl.tiles <= num_sms) {
    int best = 1;
    for (int S = 2; S <= std::min(8, pl.k_blocks); ++S)
      if (cluster_cap[S] >= pl.tiles && pl.tiles * S <= num_sms) best = S;
    if (best > 1) {
      pl.cluster_s = best;
      pl.stream_k = 0;
      pl.ipc = cdiv(pl.k_blocks, best);
      pl.grid = pl.tiles * best;
      pl.slot_rows = std::min(M, kGemmBM);
      pl.partial_bytes = 0;
      pl.stages = gemm_stages(pl.a_rows, pl.BN);
      pl.smem = gemm_smem_bytes(pl.a_rows, pl.BN, pl.stages);
      return pl;
    }
    if (2 * pl.tiles >= num_sms) sk = false;
  }
  if (sk) {
    pl.stream_k = 1;
    if (force_splits >= 2) {
      pl.ipc = cdiv(pl.k_blocks, force_splits);
    } else {
      pl.ipc = std::max(cdiv(pl.total_iters, num_sms), std::min(pl.k_blocks, 4));
    }
    pl.grid = cdiv(pl.total_iters, pl.ipc);
    pl.slot_rows = std::min(M, kGemmBM);
    pl.partial_bytes = static_cast<size_t>(pl.grid) * 2 * pl.slot_rows * pl.BN * 4;
  } else {
    pl.stream_k = 0;
    pl.ipc = pl.k_blocks;
    pl.grid = std::min(pl.tiles, num_sms);
    pl.slot_rows = std::min(M, kGemmBM);
    pl.partial_bytes = 0;
  }
  pl.a_rows = gemm_a_rows(M);
  pl.stages = gemm_stages(pl.a_rows, pl.BN);
  pl.smem = gemm_smem_bytes(pl.a_rows, pl.BN, pl.stages);
  return pl;
}

// Upper bound of GemmPlan::partial_bytes over every automatic plan with M
// rows: stream-K never uses more CTAs than SMs, each CTA owns two slots of
// min(M, 128) x 256 fp32.  Monotonic in M, so it also bounds smaller calls.
size_t gemm_partial_bound(int M, int num_sms) {
  return static_cast<size_t>(num_sms) * 2 * std::min(M, kGemmBM) * 256 * 4;
}

// ---------------------------------------------------------------------------
// attention planning
// ---------------------------------------------------------------------------
// Requests per attention launch: the request index is a grid dimension (y for
// the two-CTA kernel, z for the others), at most 65535.
constexpr int kMaxAttnRequests = 65535;

struct AttnPlan {
  int chunk_keys = 0, max_splits = 0, R = 0, row_groups = 0, key_parts = 0, nwc = 0;
  bool tc = false;   // tcgen05 kernel (kv groups of up to 64 query rows)
  int kt = 128;      // tcgen05 kernel: keys per tile
  int st = 2;        // tcgen05 kernel: K/V ring depth (64-key tiles: 2 -> two CTAs per SM)
  bool persist = false;  // six-deep ring: persistent CTAs (one per SM) walk the items
  bool cluster = false;  // tcgen05 kernel, splits of a (request, kv head) combined in a cluster
  bool tc2 = false;      // head_dim 128: two CTAs per SM, P V transposed (attention_tc2.cuh)
  size_t part_o_bytes = 0, part_ml_bytes = 0;
};

// forced_ring: K/V ring depth of the 64-key tcgen05 kernel (2 or 6), or 0 to
// let the planner decide; persist: the six-deep ring as persistent CTAs.
AttnPlan plan_attention(int B, int Hkv, int W, int P, int bs, int G, int D, int num_sms,
                        bool allow_cluster, int forced_ring, bool persist = false,
                        int tc2_keys = 64) {
  AttnPlan a;
  const int keys_max = W * P;
  const double est = static_cast<double>(B) * Hkv * keys_max;
  a.R = bs * G;
  a.tc = a.R <= kTcM;
  a.kt = kTcKeysSmall;   // 64-key tiles (the ring depth is chosen below)
  const int tile = a.tc ? a.kt : kAttnTileKeys;
  int chunk = static_cast<int>(std::ceil(est / (4.0 * num_sms)));
  chunk = (chunk + tile - 1) / tile * tile;
  chunk = std::max(128, std::min(8192, chunk));
  a.chunk_keys = chunk;
  a.max_splits = cdiv(keys_max, chunk);
  // Ring depth: a split of at least 2 x 6 tiles keeps a six-deep ring busy, and
  // one CTA per SM with six 64-key tiles in flight then beats two CTAs with two
  // each.  Measured on the Qwen3-8B shape: batch 32, contexts U[512, 8192]
  // (56-tile splits): 234 -> 191 us per layer; batch 32 x 8192: 366 -> 358 us;
  // batch 128 x 4096: 586 -> 604 us; short splits (batch 2-4, 2-4 tiles) lose
  // 25-30%, so they keep the two-CTA ring.
  a.st = (chunk / kTcKeysSmall >= 2 * kTcDeepStages) ? kTcDeepStages : kTcStages;
  if (forced_ring == kTcStages || forced_ring == kTcDeepStages) a.st = forced_ring;
  a.persist = persist && a.tc && a.st == kTcDeepStages;
  // head_dim 128 (every configuration of the pages' models): unless a ring
  // depth, the persistent or the cluster variant is asked for, the kernel
  // with two CTAs per SM and P V transposed; its splits are sized for 8
  // CTAs per SM (two resident at a time) so that mixed context lengths
  // balance over several waves
  if (a.tc && D == 128 && forced_ring == 0 && !persist && !allow_cluster) {
    a.tc2 = true;
    a.kt = tc2_keys;
    a.st = tc2_keys == 64 ? Tc2Cfg<64>::ST : Tc2Cfg<32>::ST;
    chunk = static_cast<int>(std::ceil(est / (8.0 * num_sms)));
    chunk = (chunk + tile - 1) / tile * tile;
    chunk = std::max(128, std::min(8192, chunk));
    a.chunk_keys = chunk;
    a.max_splits = cdiv(keys_max, chunk);
  }
  a.row_groups = cdiv(a.R, 16);
  a.key_parts = 1;
  while (a.key_parts < 4 && a.row_groups * a.key_parts * 2 <= kAttnMaxComputeWarps)
    a.key_parts *= 2;
  a.nwc = a.row_groups * a.key_parts;
  a.part_o_bytes =
      a.max_splits > 1 ? static_cast<size_t>(a.max_splits) * B * Hkv * a.R * D * 4 : 0;
  a.part_ml_bytes =
      a.max_splits > 1 ? static_cast<size_t>(a.max_splits) * B * Hkv * a.R * 2 * 4 : 0;
  // Opt-in: with few (request, kv head) pairs, combine the key splits inside a
  // cluster of up to 8 CTAs (128-key tiles) instead of through global partials
  // and a second kernel.  Measured slower than the default (64-key tiles, two
  // CTAs per SM, combine kernel) at batch 1-4 of the Qwen3-8B shape
  // (batch 1, context 2048: 18.2 vs 14.6 us per layer).
  if (allow_cluster && a.tc && 2 * B * Hkv <= num_sms) {
    const int S = std::min(8, num_sms / (B * Hkv));
    if (S >= 2) {
      const int chunk = cdiv(cdiv(keys_max, S), kTcKeys) * kTcKeys;
      const int splits = cdiv(keys_max, chunk);
      if (splits >= 2) {
        a.cluster = true;
        a.kt = kTcKeys;      // few requests: 128-key tiles, more keys in flight per CTA
        a.chunk_keys = chunk;
        a.max_splits = splits;
        a.part_o_bytes = 0;
        a.part_ml_bytes = 0;
      }
    }
  }
  return a;
}

// ---------------------------------------------------------------------------
// error helpers
// ---------------------------------------------------------------------------
#define DF_CUDA(expr)                                   \
  do {                                                  \
    if ((expr) != cudaSuccess) return DFLASH_ERR_CUDA;  \
  } while (0)

}  // namespace

// Programmatic dependent launch unless the environment sets DFLASH_PDL=0
// (read once per process).
bool pdl_default() {
  static const bool on = [] {
    const char* e = std::getenv("DFLASH_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

// ---------------------------------------------------------------------------
// handle
// ---------------------------------------------------------------------------
struct dflash_handle {
  dflash_config cfg{};
  std::vector<int> target_layer_ids;
  int device = 0;
  int num_sms = 148;
  // aliased caller weights (embedding table and norm weights)
  const bf16 *hidden_norm_w = nullptr, *embed = nullptr, *final_norm_w = nullptr;
  std::vector<const bf16*> in_norm_w, post_norm_w, q_norm_w, k_norm_w;
  // GEMM weights: copies owned by the handle, in the tile-contiguous layout of
  // pack_tiles_kernel; the ones multiplied against fp16 operands are held as
  // fp16 (bf16 -> fp16 is exact in fp16's normal range)
  std::vector<f16*> wqkv, wgu, wo;  // [Wq; Wk; Wv], gate/up interleaved by 16 rows, Wo
  std::vector<bf16*> wdown;         // W_down (bf16: multiplied against the bf16 MLP hidden)
  bf16* fcw = nullptr;              // fc (bf16: multiplied against the bf16 target states)
  f16* wkv = nullptr;               // all layers' [Wk; Wv], [L * 2 * Hkv * D, H]
  f16* lm_head16 = nullptr;         // [vocab_count, H]: rows [vocab_start, +vocab_count)
  // vocabulary shard of the LM head (tensor-parallel proposal); the whole
  // vocabulary unless created by dflash_create_vocab_shard
  int vocab_start = 0, vocab_count = 0;
  // tensor-parallel shard (dflash_create_tp_shard): rank and group size; the
  // cfg above then holds this shard's head and MLP-feature counts
  int tp_rank = 0, tp_size = 1;
  bf16* knorm_all = nullptr;  // [L, D]
  float2* rope = nullptr;   // [max_position, D/2]
  unsigned* dev_err = nullptr;
  unsigned* counters = nullptr;
  // fp16 range of the weights stored in fp16 (checked by dflash_create)
  unsigned* range_stats = nullptr;
  float fp16_weight_absmax = 0.f;
  double fp16_subnormal_fraction = 0.0;
  double norm_output_bound = 0.0;
  std::mutex mu;
  std::map<std::tuple<const void*, uint64_t, uint64_t, uint32_t, bool>, CUtensorMap> tmaps;
  std::map<std::pair<const void*, int>, std::array<int, 9>> cluster_caps;
  // launch accounting and optional per-launch event profiling (diagnostics)
  unsigned long long launches = 0;
  bool prof_on = false;
  // hot-path kernels are launched with programmatic dependent launch (the
  // environment variable DFLASH_PDL=0 turns it off)
  bool pdl = pdl_default();
  // few-row gate/up + down as one chain launch: opt-in (DFLASH_CHAIN=1 when the
  // handle is created).  Measured on the batch-1 Qwen3-8B-shaped step it is
  // 1-2% slower than two launches, whose down GEMM already prefetches on the
  // SMs gate/up leaves free and reduces through clusters.
  bool chain = [] {
    const char* e = std::getenv("DFLASH_CHAIN");
    return e && e[0] == '1';
  }();
  // cluster-combined attention splits for few requests: opt-in
  // (DFLASH_ATTN_CLUSTER=1 when the handle is created)
  bool attn_cluster = [] {
    const char* e = std::getenv("DFLASH_ATTN_CLUSTER");
    return e && e[0] == '1';
  }();
  // K/V ring depth of the 64-key attention kernel forced by DFLASH_ATTN_STAGES
  // (2 or 6) when the handle is created; 0 lets the planner decide
  int attn_ring = [] {
    const char* e = std::getenv("DFLASH_ATTN_STAGES");
    return e ? std::atoi(e) : 0;
  }();
  // six-deep-ring attention as persistent CTAs: opt-in (DFLASH_ATTN_PERSIST=1
  // when the handle is created)
  bool attn_persist = [] {
    const char* e = std::getenv("DFLASH_ATTN_PERSIST");
    return e && e[0] == '1';
  }();
  // keys per tile of the two-CTA-per-SM head_dim-128 kernel (DFLASH_ATTN_TILE
  // = 32 or 64 when the handle is created; 64 otherwise: measured at 128
  // requests x 8k-32k keys, 64-key tiles stream 4.2 TB/s, 32-key ones 3.7)
  int attn_tile = [] {
    const char* e = std::getenv("DFLASH_ATTN_TILE");
    return (e && std::atoi(e) == 32) ? 32 : 64;
  }();
  // whole-tile GEMMs over several 128-row M tiles run on CTA pairs (one MMA of
  // 256 x 256 over two SMs, gemm_pair.cuh) unless DFLASH_GEMM_PAIR=0 when the
  // handle is created
  bool gemm_pair = [] {
    const char* e = std::getenv("DFLASH_GEMM_PAIR");
    return !(e && e[0] == '0');
  }();
  // few wide pair tiles with a long K split over two pairs (a cluster of four)
  // unless DFLASH_GEMM_SPLIT=0 when the handle is created
  bool gemm_split = [] {
    const char* e = std::getenv("DFLASH_GEMM_SPLIT");
    return !(e && e[0] == '0');
  }();
  // two-CTA clusters of each pair-GEMM instantiation that can be resident at
  // once (occupancy query, per kernel)
  std::map<const void*, int> pair_clusters;
  std::vector<cudaEvent_t> prof_events;
  size_t prof_next = 0;
  std::vector<int> prof_kind;

  bool tmap(CUtensorMap* out, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
            bool f16 = false) {
    std::lock_guard<std::mutex> lk(mu);
    auto key = std::make_tuple(ptr, rows, cols, box_rows, f16);
    auto it = tmaps.find(key);
    if (it != tmaps.end()) {
      *out = it->second;
      return true;
    }
    if (tmaps.size() > 8192) tmaps.clear();
    if (!make_tmap(out, ptr, rows, cols, box_rows, f16)) return false;
    tmaps.emplace(key, *out);
    return true;
  }
};

namespace {

void free_handle(dflash_handle* h) {
  if (!h) return;
  for (auto e : h->prof_events) cudaEventDestroy(e);
  for (auto p : h->wqkv) cudaFree(p);
  for (auto p : h->wgu) cudaFree(p);
  for (auto p : h->wo) cudaFree(p);
  for (auto p : h->wdown) cudaFree(p);
  cudaFree(h->fcw);
  cudaFree(h->wkv);
  cudaFree(h->lm_head16);
  cudaFree(h->knorm_all);
  cudaFree(h->rope);
  cudaFree(h->dev_err);
  cudaFree(h->counters);
  cudaFree(h->range_stats);
  delete h;
}

// Counts every kernel launch a handle's call makes and, while profiling is on,
// brackets it with a pair of events recorded on the launching stream.
struct LaunchScope {
  dflash_handle* h;
  cudaStream_t st;
  cudaEvent_t stop = nullptr;
  LaunchScope(dflash_handle* h_, int kind, cudaStream_t st_) : h(h_), st(st_) {
    ++h->launches;
    if (h->prof_on && h->prof_next + 2 <= h->prof_events.size()) {
      cudaEvent_t a = h->prof_events[h->prof_next];
      stop = h->prof_events[h->prof_next + 1];
      h->prof_next += 2;
      h->prof_kind.push_back(kind);
      cudaEventRecord(a, st);
    }
  }
  ~LaunchScope() {
    if (stop) cudaEventRecord(stop, st);
  }
};

// Launch of a hot-path kernel; with `pdl` the launch may overlap the tail of
// the previous kernel in the stream (every such kernel calls pdl_wait() before
// it touches memory that an earlier kernel writes or a later one overwrites).
// `cluster` > 1 launches thread-block clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
void launch_kc(bool pdl, int cluster, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
               cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
void launch_k(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
              cudaStream_t st, Args&&... args) {
  launch_kc(pdl, 1, kern, grid, block, smem, st, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// GEMM launch
// ---------------------------------------------------------------------------
template <int BN, class Epi>
cudaError_t set_gemm_attr() {
  return cudaFuncSetAttribute(gemm_tcgen05_kernel<BN, Epi>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemLimit);
}

template <class Epi>
cudaError_t set_gemm_attrs_all() {
  cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel<256, 1, Epi>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kGemmSmemLimit);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(gemm_pair_kernel<256, 2, Epi>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemLimit)) !=
      cudaSuccess)
    return e;
  if constexpr (128 % Epi::kGroup == 0)
    if ((e = cudaFuncSetAttribute(gemm_pair_kernel<128, 1, Epi>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kGemmSmemLimit)) != cudaSuccess)
      return e;
  if constexpr (256 % Epi::kGroup == 0)
    if ((e = set_gemm_attr<256, Epi>()) != cudaSuccess) return e;
  if constexpr (128 % Epi::kGroup == 0)
    if ((e = set_gemm_attr<128, Epi>()) != cudaSuccess) return e;
  if constexpr (Epi::kGroup <= 64)
    if ((e = set_gemm_attr<64, Epi>()) != cudaSuccess) return e;
  if constexpr (Epi::kGroup <= 32)
    if ((e = set_gemm_attr<32, Epi>()) != cudaSuccess) return e;
  return e;
}

template <int BN, class Epi>
void launch_gemm_bn(const dflash_handle* h, const CUtensorMap& ta, const CUtensorMap& tw,
                    const GemmParams& gp, const Epi& epi, int grid, int smem, cudaStream_t st) {
  launch_kc(h->pdl, gp.cluster_s, gemm_tcgen05_kernel<BN, Epi>, dim3(grid), dim3(kGemmThreads),
            smem, st, ta, tw, gp, epi);
}

// cap[S] = clusters of S CTAs (S = 2..8) of this GEMM instantiation that can be
// resident at once with `smem` bytes each; cached per handle.  nullptr if the
// occupancy query fails (cluster split-K is then not used).
template <int BN, class Epi>
const int* gemm_cluster_caps_bn(dflash_handle* h, int smem) {
  const void* key = reinterpret_cast<const void*>(gemm_tcgen05_kernel<BN, Epi>);
  std::lock_guard<std::mutex> lk(h->mu);
  auto it = h->cluster_caps.find(std::make_pair(key, smem));
  if (it != h->cluster_caps.end()) return it->second.data();
  std::array<int, 9> cap{};
  for (int S = 2; S <= 8; ++S) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S);
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tcgen05_kernel<BN, Epi>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    cap[S] = n;
  }
  return h->cluster_caps.emplace(std::make_pair(key, smem), cap).first->second.data();
}

template <class Epi>
const int* gemm_cluster_caps(dflash_handle* h, int bn, int smem) {
  switch (bn) {
    case 256:
      if constexpr (256 % Epi::kGroup == 0) return gemm_cluster_caps_bn<256, Epi>(h, smem);
      break;
    case 128:
      if constexpr (128 % Epi::kGroup == 0) return gemm_cluster_caps_bn<128, Epi>(h, smem);
      break;
    case 64:
      if constexpr (Epi::kGroup <= 64) return gemm_cluster_caps_bn<64, Epi>(h, smem);
      break;
    case 32:
      if constexpr (Epi::kGroup <= 32) return gemm_cluster_caps_bn<32, Epi>(h, smem);
      break;
  }
  return nullptr;
}

// Tile width of the CTA-pair kernel for a plan over several 128-row M tiles
// (not the staged few-row epilogue, no cluster split-K), or 0 to keep the
// one-SM plan.  256-wide pair tiles read half the operand bytes per MMA cycle
// that a one-SM 128 x 256 tile does; 256 x 128 pair tiles read as many as the
// one-SM tile (about 3/4 of the wide pair's rate, as measured on the draft
// GEMMs) but are twice as many, so they are taken only when that fills the
// SMs enough better (e.g. the O and down projections of 512 rows: 32 wide
// pair tiles for 74 pairs of SMs, or 64 narrow ones).  A one-SM stream-K
// plan (too few whole tiles) is replaced only when the pair tiles fill at
// least half of the SMs.
// A third option for few wide tiles with a long K (>= 96 k-blocks, so that
// each half still amortises the reduction): split K over two pairs (a cluster
// of four, one tile per cluster; the second pair's partial reduced through
// distributed shared memory), taken when the tiles fit one round as split
// units and that fills the SMs enough better (0.85 of the wide rate for the
// reduction).  Measured at 512 rows: down (K = 12288, 32 wide tiles -> 64
// pairs) 0.48 -> 0.61 of the sustained bf16 figure, fc 0.29 -> 0.44; O
// (K = 4096) lost 0.33 -> 0.31, hence the K floor.
struct PairChoice {
  int bn = 0, ks = 1;   // bn = 0: keep the one-SM plan
};
PairChoice gemm_pair_choice(const GemmPlan& pl, int M, int N, int group, int num_sms,
                            int split_cap) {
  PairChoice c;
  if (pl.cluster_s != 1 || gemm_staged(pl.a_rows) || pl.m_tiles < 2) return c;
  const int ncl = std::max(1, num_sms / 2);
  auto fill = [&](int bn) {
    const int tiles = cdiv(M, 2 * kPairRows) * cdiv(N, bn);
    return static_cast<double>(tiles) / (static_cast<double>(cdiv(tiles, ncl)) * ncl);
  };
  const int wide_tiles = cdiv(M, 2 * kPairRows) * cdiv(N, 256);
  const double wide = fill(256), narrow = 0.75 * fill(128);
  const double split = (pl.k_blocks >= 96 && wide_tiles <= split_cap)
                           ? 0.85 * static_cast<double>(2 * wide_tiles) / ncl : 0.0;
  const double best = std::max(wide, std::max(narrow, split));
  if (pl.stream_k && best < 0.5) return c;
  if (split > wide + 0.05 && split >= narrow) {
    c.bn = 256;
    c.ks = 2;
  } else {
    c.bn = (group <= 128 && narrow > wide + 0.05) ? 128 : 256;
  }
  return c;
}

// Clusters of 2 KS CTAs of gemm_pair_kernel<BN, KS, Epi> with `smem` bytes each
// that fit on the GPU at once (cached per handle); 0 if the query fails.
template <int BN, int KS, class Epi>
int gemm_pair_capacity(dflash_handle* h, int smem) {
  const void* key = reinterpret_cast<const void*>(gemm_pair_kernel<BN, KS, Epi>);
  std::lock_guard<std::mutex> lk(h->mu);
  auto it = h->pair_clusters.find(key);
  if (it != h->pair_clusters.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2 * KS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2 * KS);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<BN, KS, Epi>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  h->pair_clusters.emplace(key, n);
  return n;
}

// The plan `pl` on CTA pairs: 256 x BN tiles, one cluster of two CTAs per
// pair of SMs walking them; W boxes of BN / 2 rows (each CTA loads its half of
// a tile's W rows).
template <int BN, int KS, class Epi>
dflash_status run_gemm_pair(dflash_handle* h, int kind, bool f16, bool w_packed, const void* A,
                            int M, int K, const void* Wt, int N, const Epi& epi,
                            const GemmPlan& pl, cudaStream_t st) {
  using PC = PairCfg<BN>;
  const int stages = PC::kStages;
  const int smem = PC::kSmem;
  CUtensorMap ta, tw;
  if (!h->tmap(&ta, A, M, K, kPairRows, f16)) return DFLASH_ERR_CUDA;
  if (w_packed) {
    if (!h->tmap(&tw, Wt, static_cast<uint64_t>(cdiv(N, kPackRows)) * pl.k_blocks * kPackRows,
                 kGemmBK, PC::kWRows, f16))
      return DFLASH_ERR_CUDA;
  } else if (!h->tmap(&tw, Wt, N, K, PC::kWRows, f16)) {
    return DFLASH_ERR_CUDA;
  }
  GemmParams gp{};
  gp.M = M;
  gp.N = N;
  gp.K = K;
  gp.m_tiles = cdiv(M, 2 * kPairRows);
  gp.n_tiles = cdiv(N, BN);
  gp.k_blocks = pl.k_blocks;
  gp.tiles = gp.m_tiles * gp.n_tiles;
  gp.stream_k = 0;
  gp.cluster_s = 2 * KS;
  gp.ipc = pl.k_blocks;
  gp.total_iters = gp.tiles * pl.k_blocks;
  gp.nacc = 1;
  gp.nbuf = 2;
  gp.tmem_cols = PC::kTmemCols;
  gp.a_rows = kPairRows;
  gp.stages = stages;
  gp.f16 = f16 ? 1 : 0;
  gp.w_packed = w_packed ? 1 : 0;
  gp.slot_rows = 0;
  gp.partials = nullptr;
  gp.counters = h->counters;
  gp.err = h->dev_err;
  int clusters = gemm_pair_capacity<BN, KS, Epi>(h, smem);
  if (clusters <= 0) clusters = h->num_sms / (2 * KS);
  clusters = std::max(1, std::min(clusters, gp.tiles));
  if (KS == 2) clusters = gp.tiles;   // one tile per cluster (the planner keeps it to one round)
  LaunchScope scope(h, kind, st);
  launch_kc(h->pdl, 2 * KS, gemm_pair_kernel<BN, KS, Epi>, dim3(2 * KS * clusters),
            dim3(kGemmThreads), smem, st,
            ta, tw, gp, epi);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

// D = A[M, K] * W[N, K]^T with epilogue `epi`.  `partials` must hold
// plan.partial_bytes.
template <class Epi>
dflash_status run_gemm(dflash_handle* h, int kind, bool f16, bool w_packed, const void* A, int M,
                       int K,
                       const void* Wt, int N, const Epi& epi, float* partials,
                       size_t partial_cap, cudaStream_t st, int force_bn = 0,
                       int force_splits = 0) {
  if (M <= 0) return DFLASH_OK;
  if (force_bn && ((force_bn != 32 && force_bn != 64 && force_bn != 128 && force_bn != 256) ||
                   force_bn % Epi::kGroup))
    return DFLASH_ERR_INVALID_ARG;
  if (force_splits < 0 || force_splits > K / kGemmBK) return DFLASH_ERR_INVALID_ARG;
  GemmPlan pl = plan_gemm(M, N, K, Epi::kGroup, h->num_sms, force_bn, force_splits);
  if (gemm_staged(pl.a_rows) && pl.tiles <= h->num_sms && !force_splits) {
    const int* cap = gemm_cluster_caps<Epi>(h, pl.BN, pl.smem);
    if (cap) pl = plan_gemm(M, N, K, Epi::kGroup, h->num_sms, force_bn, force_splits, cap);
  }
  if (pl.stream_k && pl.tiles > kCounterSlots - 2) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if (pl.partial_bytes > partial_cap) return DFLASH_ERR_WORKSPACE;
  if (h->gemm_pair && !force_bn && !force_splits) {
    const int cap = h->gemm_split ? gemm_pair_capacity<256, 2, Epi>(h, PairCfg<256>::kSmem) : 0;
    const PairChoice pc = gemm_pair_choice(pl, M, N, Epi::kGroup, h->num_sms, cap);
    if (pc.bn == 256 && pc.ks == 2)
      return run_gemm_pair<256, 2>(h, kind, f16, w_packed, A, M, K, Wt, N, epi, pl, st);
    if (pc.bn == 256)
      return run_gemm_pair<256, 1>(h, kind, f16, w_packed, A, M, K, Wt, N, epi, pl, st);
    if constexpr (128 % Epi::kGroup == 0)
      if (pc.bn == 128)
        return run_gemm_pair<128, 1>(h, kind, f16, w_packed, A, M, K, Wt, N, epi, pl, st);
  }
  CUtensorMap ta, tw;
  if (!h->tmap(&ta, A, M, K, pl.a_rows, f16)) return DFLASH_ERR_CUDA;
  if (w_packed) {
    if (!h->tmap(&tw, Wt, static_cast<uint64_t>(cdiv(N, kPackRows)) * pl.k_blocks * kPackRows,
                 kGemmBK, pl.BN, f16))
      return DFLASH_ERR_CUDA;
  } else if (!h->tmap(&tw, Wt, N, K, pl.BN, f16)) {
    return DFLASH_ERR_CUDA;
  }
  GemmParams gp{};
  gp.M = M;
  gp.N = N;
  gp.K = K;
  gp.m_tiles = pl.m_tiles;
  gp.n_tiles = pl.n_tiles;
  gp.k_blocks = pl.k_blocks;
  gp.tiles = pl.tiles;
  gp.stream_k = pl.stream_k;
  gp.cluster_s = pl.cluster_s;
  gp.ipc = pl.ipc;
  gp.total_iters = pl.total_iters;
  gp.nacc = pl.nacc;
  gp.nbuf = pl.nbuf;
  gp.tmem_cols = pl.tmem_cols;
  gp.a_rows = pl.a_rows;
  gp.stages = pl.stages;
  gp.f16 = f16 ? 1 : 0;
  gp.w_packed = w_packed ? 1 : 0;
  gp.slot_rows = pl.slot_rows;
  gp.partials = partials;
  gp.counters = h->counters;
  gp.err = h->dev_err;
  LaunchScope scope(h, kind, st);
  switch (pl.BN) {
    case 256:
      if constexpr (256 % Epi::kGroup == 0) launch_gemm_bn<256>(h, ta, tw, gp, epi, pl.grid, pl.smem, st);
      break;
    case 128:
      if constexpr (128 % Epi::kGroup == 0) launch_gemm_bn<128>(h, ta, tw, gp, epi, pl.grid, pl.smem, st);
      break;
    case 64:
      if constexpr (Epi::kGroup <= 64) launch_gemm_bn<64>(h, ta, tw, gp, epi, pl.grid, pl.smem, st);
      break;
    case 32:
      if constexpr (Epi::kGroup <= 32) launch_gemm_bn<32>(h, ta, tw, gp, epi, pl.grid, pl.smem, st);
      break;
    default:
      return DFLASH_ERR_UNSUPPORTED_SHAPE;
  }
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

// Phase parameters of one GEMM of a chain launch (packed weights).
template <class Epi>
bool chain_phase(dflash_handle* h, const GemmPlan& pl, bool f16, const void* A, int M, int K,
                 const void* Wt, int N, float* partials, unsigned* counters, CUtensorMap* ta,
                 CUtensorMap* tw, GemmParams* gp) {
  if (!h->tmap(ta, A, M, K, pl.a_rows, f16)) return false;
  if (!h->tmap(tw, Wt, static_cast<uint64_t>(cdiv(N, kPackRows)) * pl.k_blocks * kPackRows,
               kGemmBK, pl.BN, f16))
    return false;
  *gp = GemmParams{};
  gp->M = M;
  gp->N = N;
  gp->K = K;
  gp->m_tiles = pl.m_tiles;
  gp->n_tiles = pl.n_tiles;
  gp->k_blocks = pl.k_blocks;
  gp->tiles = pl.tiles;
  gp->stream_k = pl.stream_k;
  gp->cluster_s = 1;
  gp->ipc = pl.ipc;
  gp->total_iters = pl.total_iters;
  gp->nacc = pl.nacc;
  gp->nbuf = pl.nbuf;
  gp->tmem_cols = pl.tmem_cols;
  gp->a_rows = pl.a_rows;
  gp->stages = pl.stages;
  gp->f16 = f16 ? 1 : 0;
  gp->w_packed = 1;
  gp->slot_rows = pl.slot_rows;
  gp->partials = partials;
  gp->counters = counters;
  gp->err = h->dev_err;
  return true;
}

// True when two few-row GEMMs (packed weights) can run as one chain launch:
// the staged epilogue on both sides with the same tile shape and ring.
bool chain_ok(int M, int num_sms) {
  return gemm_staged(gemm_a_rows(M)) && M > 0 && num_sms > 0;
}

// Phase 1: D1 = A1 W1^T with epilogue e1 (whole tiles, one per CTA, when they
// occupy at least half of the SMs; else stream-K); phase 2: D2 = A2 W2^T with
// e2 (stream-K), A2 written by phase 1.  One launch of one CTA per SM.
template <class Epi1, class Epi2>
dflash_status run_gemm_chain(dflash_handle* h, int kind, bool f16_1, const void* A1, int M,
                             int K1, const void* W1, int N1, const Epi1& e1, bool f16_2,
                             const void* A2, int K2, const void* W2, int N2, const Epi2& e2,
                             float* partials, size_t partial_cap, cudaStream_t st) {
  if (!chain_ok(M, h->num_sms)) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  const int t1 = cdiv(N1, kPackRows);
  GemmPlan pl1 = plan_gemm(M, N1, K1, Epi1::kGroup, h->num_sms, kPackRows,
                           2 * t1 >= h->num_sms && t1 <= h->num_sms ? 1 : 0);
  GemmPlan pl2 = plan_gemm(M, N2, K2, Epi2::kGroup, h->num_sms, kPackRows, 0);
  if (pl1.a_rows != pl2.a_rows || pl1.stages != pl2.stages || pl1.tmem_cols != pl2.tmem_cols ||
      pl1.BN != 256 || pl2.BN != 256 || pl1.nbuf != 1 || pl2.nbuf != 1)
    return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if (pl1.stream_k && pl2.stream_k &&
      static_cast<size_t>(pl1.tiles) + pl2.tiles > static_cast<size_t>(kCounterSlots - 2))
    return DFLASH_ERR_UNSUPPORTED_SHAPE;
  const int grid = h->num_sms;
  const size_t part = static_cast<size_t>(grid) * 2 * std::min(M, kGemmBM) * 256 * 4;
  if ((pl1.stream_k || pl2.stream_k) && part > partial_cap) return DFLASH_ERR_WORKSPACE;
  CUtensorMap ta1, tw1, ta2, tw2;
  GemmParams g1, g2;
  if (!chain_phase<Epi1>(h, pl1, f16_1, A1, M, K1, W1, N1, partials, h->counters, &ta1, &tw1,
                         &g1) ||
      !chain_phase<Epi2>(h, pl2, f16_2, A2, M, K2, W2, N2, partials,
                         h->counters + (pl1.stream_k ? pl1.tiles : 0), &ta2, &tw2, &g2))
    return DFLASH_ERR_CUDA;
  unsigned* dep = h->counters + kCounterSlots - 2;
  // every CTA waits for all the others' phase-1 stores: the grid must be
  // co-resident, which a cooperative launch guarantees (or refuses)
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemm_chain_kernel<256, Epi1, Epi2>,
                                                    kGemmThreads, pl1.smem) != cudaSuccess ||
      per_sm < 1)
    return DFLASH_ERR_UNSUPPORTED_SHAPE;
  LaunchScope scope(h, kind, st);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = pl1.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, gemm_chain_kernel<256, Epi1, Epi2>, ta1, tw1, g1, e1, ta2, tw2, g2, e2,
                     dep);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// attention launch
// ---------------------------------------------------------------------------
template <int D>
cudaError_t set_attn_attrs() {
  const int bytes = AttnCfg<D>::smem_bytes(kAttnMaxComputeWarps);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(attn_block_kernel<D, 64>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(attn_block_kernel<D, 32>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(attn_block_kernel<D, 16>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(attn_block_tc_kernel<D, kTcKeysSmall>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                TcAttnCfg<D, kTcKeysSmall>::kSmem)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(attn_block_tc_kernel<D, kTcKeysSmall, kTcDeepStages>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                TcAttnCfg<D, kTcKeysSmall, kTcDeepStages>::kSmem)) != cudaSuccess)
    return e;
  if constexpr (D == 128) {
    if ((e = cudaFuncSetAttribute(attn_block_tc2_kernel<64>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  Tc2Cfg<64>::kSmem)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(attn_block_tc2_kernel<32>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  Tc2Cfg<32>::kSmem)) != cudaSuccess)
      return e;
  }
  if ((e = cudaFuncSetAttribute(attn_block_tc_persistent_kernel<D, kTcDeepStages>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                TcAttnCfg<D, kTcKeysSmall, kTcDeepStages>::kSmem)) != cudaSuccess)
    return e;
  return cudaFuncSetAttribute(attn_block_tc_kernel<D, kTcKeys>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              TcAttnCfg<D, kTcKeys>::kSmem);
}

template <int D>
dflash_status run_attention(dflash_handle* h, const AttnPlan& ap, AttnParams prm,
                            const void* kc, const void* vc, int num_pages, cudaStream_t st) {
  const dflash_config& c = h->cfg;
  CUtensorMap tk, tv;
  const uint64_t rows = static_cast<uint64_t>(num_pages) * c.n_kv_heads * c.page_size;
  // box: 16 rows (one page of one head) x 64 columns
  if (!h->tmap(&tk, kc, rows, D, 16)) return DFLASH_ERR_CUDA;
  if (!h->tmap(&tv, vc, rows, D, 16)) return DFLASH_ERR_CUDA;
  dim3 grid(ap.max_splits, c.n_kv_heads, prm.B);
  const int threads = 32 * (ap.nwc + 1);
  const int smem = AttnCfg<D>::smem_bytes(ap.nwc);
  prm.row_groups = ap.row_groups;
  prm.key_parts = ap.key_parts;
  prm.cluster = ap.cluster ? 1 : 0;
  if (ap.tc2) {
    LaunchScope scope(h, DFLASH_KERNEL_ATTENTION, st);
    if constexpr (D == 128) {
      // split-major: every request's first splits are dispatched first and the
      // partial last splits fill the tail
      const dim3 grid2(c.n_kv_heads, prm.B, ap.max_splits);
      if (ap.kt == 64)
        launch_k(h->pdl, attn_block_tc2_kernel<64>, grid2, dim3(kTcThreads), Tc2Cfg<64>::kSmem,
                 st, tk, tv, prm);
      else
        launch_k(h->pdl, attn_block_tc2_kernel<32>, grid2, dim3(kTcThreads), Tc2Cfg<32>::kSmem,
                 st, tk, tv, prm);
    }
  } else if (ap.tc) {
    LaunchScope scope(h, DFLASH_KERNEL_ATTENTION, st);
    if (ap.kt == kTcKeysSmall && ap.persist) {
      const int items = ap.max_splits * c.n_kv_heads * prm.B;
      launch_k(h->pdl, attn_block_tc_persistent_kernel<D, kTcDeepStages>,
               dim3(std::min(items, h->num_sms)), dim3(kTcThreads),
               TcAttnCfg<D, kTcKeysSmall, kTcDeepStages>::kSmem, st, tk, tv, prm);
    } else if (ap.kt == kTcKeysSmall && ap.st == kTcDeepStages)
      launch_kc(h->pdl, ap.cluster ? ap.max_splits : 1,
                attn_block_tc_kernel<D, kTcKeysSmall, kTcDeepStages>, grid, dim3(kTcThreads),
                TcAttnCfg<D, kTcKeysSmall, kTcDeepStages>::kSmem, st, tk, tv, prm);
    else if (ap.kt == kTcKeysSmall)
      launch_kc(h->pdl, ap.cluster ? ap.max_splits : 1, attn_block_tc_kernel<D, kTcKeysSmall>,
                grid, dim3(kTcThreads), TcAttnCfg<D, kTcKeysSmall>::kSmem, st, tk, tv, prm);
    else
      launch_kc(h->pdl, ap.cluster ? ap.max_splits : 1, attn_block_tc_kernel<D, kTcKeys>, grid,
                dim3(kTcThreads), TcAttnCfg<D, kTcKeys>::kSmem, st, tk, tv, prm);
  } else {
    LaunchScope scope(h, DFLASH_KERNEL_ATTENTION, st);
    if (ap.key_parts == 1)
      launch_k(h->pdl, attn_block_kernel<D, 64>, grid, dim3(threads), smem, st, tk, tv, prm);
    else if (ap.key_parts == 2)
      launch_k(h->pdl, attn_block_kernel<D, 32>, grid, dim3(threads), smem, st, tk, tv, prm);
    else
      launch_k(h->pdl, attn_block_kernel<D, 16>, grid, dim3(threads), smem, st, tk, tv, prm);
  }
  if (ap.max_splits > 1 && !ap.cluster) {
    LaunchScope scope(h, DFLASH_KERNEL_ATTN_COMBINE, st);
    const int rows = prm.B * c.n_kv_heads * prm.R;
    launch_k(h->pdl, attn_combine_kernel<D>, dim3(cdiv(rows, 8)), dim3(256), 0, st, prm);
  }
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// workspace layouts
// ---------------------------------------------------------------------------
struct InjectWs {
  size_t fcx = 0, ctx = 0, partial = 0, total = 0, partial_cap = 0;
};
InjectWs inject_layout(const dflash_handle* h, int n) {
  const dflash_config& c = h->cfg;
  InjectWs w;
  size_t off = 0;
  w.fcx = off;
  off += align_up(static_cast<size_t>(n) * c.hidden * 4);
  w.ctx = off;
  off += align_up(static_cast<size_t>(n) * c.hidden * 2);
  const size_t cap = gemm_partial_bound(n, h->num_sms);
  w.partial = off;
  w.partial_cap = cap;
  off += align_up(cap);
  w.total = off;
  return w;
}

struct ProposeWs {
  size_t x = 0, nrm = 0, q = 0, o = 0, hm = 0, frows = 0, keys = 0, part_o = 0, part_ml = 0,
         partial = 0, total = 0, partial_cap = 0, part_o_cap = 0, part_ml_cap = 0, xpart = 0;
};
size_t propose_partial_need(const dflash_handle* h, int B) {
  return gemm_partial_bound(B * h->cfg.block_size, h->num_sms);
}
ProposeWs propose_layout(const dflash_handle* h, int B, int W) {
  const dflash_config& c = h->cfg;
  const int bs = c.block_size, K = bs - 1, M = B * bs, MK = B * K;
  const int D = c.head_dim, Hq = c.n_q_heads, Hkv = c.n_kv_heads, H = c.hidden;
  ProposeWs w;
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes);
    return at;
  };
  w.x = take(static_cast<size_t>(M) * H * 4);
  w.nrm = take(static_cast<size_t>(M) * H * 2);
  w.q = take(static_cast<size_t>(M) * Hq * D * 2);
  w.o = take(static_cast<size_t>(M) * Hq * D * 2);
  w.hm = take(static_cast<size_t>(M) * c.intermediate * 2);
  w.frows = take(static_cast<size_t>(MK) * H * 2);
  w.keys = take(static_cast<size_t>(MK) * 8);
  size_t po = 0, pm = 0, pc = 0;
  // the attention split plan is not monotonic in the batch: cover every size
  for (int bb = 1; bb <= B; ++bb) {
    const AttnPlan ap = plan_attention(bb, Hkv, W, c.page_size, bs, Hq / Hkv, D, h->num_sms,
                                       h->attn_cluster, h->attn_ring,
                                     h->attn_persist, h->attn_tile);
    po = std::max(po, ap.part_o_bytes);
    pm = std::max(pm, ap.part_ml_bytes);
  }
  pc = propose_partial_need(h, B);
  w.part_o = take(po);
  w.part_ml = take(pm);
  w.part_o_cap = po;
  w.part_ml_cap = pm;
  w.partial = take(pc);
  w.partial_cap = pc;
  // tensor-parallel shard: this rank's partial sums of the O / down
  // projections, all-reduced in place by the caller's exchange hook
  if (h->tp_size > 1) w.xpart = take(static_cast<size_t>(M) * H * 4);
  w.total = off;
  return w;
}

template <class T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

// Makes `dev` current for this library's runtime (a no-op when it already is,
// so calls stay cheap and legal inside stream capture).
cudaError_t use_device(int dev) {
  int cur = -1;
  if (cudaGetDevice(&cur) == cudaSuccess && cur == dev) return cudaSuccess;
  return cudaSetDevice(dev);
}

// Handle-free calls run on the device of their stream (or, on the legacy
// default stream, of their output buffer).
// Under stream capture the device is not queried (a stream query would
// invalidate a global-mode capture); the current device is used as is.
dflash_status set_device_for(cudaStream_t st, const void* p) {
  int dev = -1;
  if (st != nullptr) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
      cudaGetLastError();
      return DFLASH_ERR_INVALID_ARG;
    }
    if (cs != cudaStreamCaptureStatusNone) return DFLASH_OK;
    if (cudaStreamGetDevice(st, &dev) != cudaSuccess) {
      cudaGetLastError();
      return DFLASH_ERR_INVALID_ARG;
    }
  } else {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess || a.type != cudaMemoryTypeDevice) {
      cudaGetLastError();
      return DFLASH_ERR_INVALID_ARG;
    }
    dev = a.device;
  }
  DF_CUDA(use_device(dev));
  return DFLASH_OK;
}

}  // namespace

namespace {
struct VerifyPlan {
  int chunks = 1, chunk_len = 0;
  size_t bytes = 0;
};
VerifyPlan plan_verify(int B, int K, int V) {
  VerifyPlan v;
  const int rows = B * (K + 1);
  int chunks = std::max(1, cdiv(4 * 148, std::max(rows, 1)));
  chunks = std::min(chunks, std::max(1, V / 4096));
  int len = cdiv(V, chunks);
  len = (len + 3) / 4 * 4;
  v.chunk_len = len;
  v.chunks = cdiv(V, len);
  v.bytes = align_up(static_cast<size_t>(rows) * v.chunks * 8);
  return v;
}
}  // namespace

namespace {
template <int D>
dflash_status propose_layers(dflash_handle* h, const ProposeWs& lw, void* ws,
                             const int32_t* seq_lens, const int32_t* block_table, int B, int W,
                             void* const* k_cache, void* const* v_cache, int num_pages,
                             cudaStream_t st, dflash_allreduce_fn exchange, void* user) {
  const dflash_config& c = h->cfg;
  const int bs = c.block_size, M = B * bs, H = c.hidden, Hq = c.n_q_heads, Hkv = c.n_kv_heads,
            I = c.intermediate, K = bs - 1;
  float* x = at<float>(ws, lw.x);
  f16* nrm = at<f16>(ws, lw.nrm);
  bf16* q = at<bf16>(ws, lw.q);
  f16* o = at<f16>(ws, lw.o);
  bf16* hm = at<bf16>(ws, lw.hm);
  f16* frows = at<f16>(ws, lw.frows);
  float* partial = at<float>(ws, lw.partial);
  const AttnPlan ap = plan_attention(B, Hkv, W, c.page_size, bs, Hq / Hkv, D, h->num_sms,
                                     h->attn_cluster, h->attn_ring,
                                     h->attn_persist, h->attn_tile);
  if (ap.part_o_bytes > lw.part_o_cap || ap.part_ml_bytes > lw.part_ml_cap)
    return DFLASH_ERR_WORKSPACE;
  AttnParams prm;
  prm.q = q;
  prm.o = o;
  prm.part_o = at<float>(ws, lw.part_o);
  prm.part_ml = at<float>(ws, lw.part_ml);
  prm.seq_lens = seq_lens;
  prm.block_table = block_table;
  prm.B = B;
  prm.W = W;
  prm.bs = bs;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.R = ap.R;
  prm.num_pages = num_pages;
  prm.chunk_keys = ap.chunk_keys;
  prm.max_splits = ap.max_splits;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  prm.err = h->dev_err;

  for (int l = 0; l < c.n_layers; ++l) {
    // QKV projection with q/k norm, RoPE and the block's paged K/V write
    EpiQKV<D> eq;
    eq.q = q;
    eq.q_norm_w = h->q_norm_w[l];
    eq.k_norm_w = h->k_norm_w[l];
    eq.rope = h->rope;
    eq.k_cache = static_cast<bf16*>(k_cache[l]);
    eq.v_cache = static_cast<bf16*>(v_cache[l]);
    eq.seq_lens = seq_lens;
    eq.block_table = block_table;
    eq.max_pos = c.max_position;
    eq.W = W;
    eq.bs = bs;
    eq.Hq = Hq;
    eq.Hkv = Hkv;
    eq.P = c.page_size;
    eq.num_pages = num_pages;
    eq.eps = c.rms_eps;
    eq.err = h->dev_err;
    dflash_status s = run_gemm(h, DFLASH_KERNEL_GEMM_QKV, true, true, nrm, M, H, h->wqkv[l],
                               (Hq + 2 * Hkv) * D, eq, partial, lw.partial_cap, st);
    if (s != DFLASH_OK) return s;
    // non-causal block attention over context + block
    s = run_attention<D>(h, ap, prm, k_cache[l], v_cache[l], num_pages, st);
    if (s != DFLASH_OK) return s;
    if (h->tp_size > 1) {
      // tensor-parallel shard: Wo and W_down are row-parallel, so this rank
      // forms partial sums of both projections over its heads / features;
      // the caller's hook sums them over the ranks (an all-reduce) before
      // each residual add
      float* xpart = at<float>(ws, lw.xpart);
      EpiStoreF32 es{xpart, H};
      s = run_gemm(h, DFLASH_KERNEL_GEMM_O, true, true, o, M, Hq * D, h->wo[l], H, es, partial,
                   lw.partial_cap, st);
      if (s != DFLASH_OK) return s;
      if (exchange(xpart, static_cast<size_t>(M) * H, st, user) != 0) return DFLASH_ERR_EXCHANGE;
      {
        LaunchScope scope(h, DFLASH_KERNEL_RMSNORM, st);
        launch_k(h->pdl, add_rmsnorm_rows_kernel, dim3(M), dim3(256), 0, st, x,
                 static_cast<const float*>(xpart), h->post_norm_w[l], nrm, H, c.rms_eps, 0, bs);
      }
      if (cudaGetLastError() != cudaSuccess) return DFLASH_ERR_CUDA;
      EpiSwiGLU eg{hm, I};
      s = run_gemm(h, DFLASH_KERNEL_GEMM_GATE_UP, true, true, nrm, M, H, h->wgu[l], 2 * I, eg,
                   partial, lw.partial_cap, st);
      if (s != DFLASH_OK) return s;
      s = run_gemm(h, DFLASH_KERNEL_GEMM_DOWN, false, true, hm, M, I, h->wdown[l], H, es,
                   partial, lw.partial_cap, st);
      if (s != DFLASH_OK) return s;
      if (exchange(xpart, static_cast<size_t>(M) * H, st, user) != 0) return DFLASH_ERR_EXCHANGE;
      LaunchScope scope(h, DFLASH_KERNEL_RMSNORM, st);
      if (l + 1 < c.n_layers)
        launch_k(h->pdl, add_rmsnorm_rows_kernel, dim3(M), dim3(256), 0, st, x,
                 static_cast<const float*>(xpart), h->in_norm_w[l + 1], nrm, H, c.rms_eps, 0, bs);
      else
        launch_k(h->pdl, add_rmsnorm_rows_kernel, dim3(B * K), dim3(256), 0, st, x,
                 static_cast<const float*>(xpart), h->final_norm_w, frows, H, c.rms_eps, K, bs);
      if (cudaGetLastError() != cudaSuccess) return DFLASH_ERR_CUDA;
      continue;
    }
    // x += Wo o
    EpiResidAdd er{x, H};
    s = run_gemm(h, DFLASH_KERNEL_GEMM_O, true, true, o, M, Hq * D, h->wo[l], H, er, partial,
                 lw.partial_cap, st);
    if (s != DFLASH_OK) return s;
    {
      LaunchScope scope(h, DFLASH_KERNEL_RMSNORM, st);
      launch_k(h->pdl, rmsnorm_rows_kernel, dim3(M), dim3(256), 0, st, x, h->post_norm_w[l], nrm, H,
               c.rms_eps, 0, bs);
    }
    if (cudaGetLastError() != cudaSuccess) return DFLASH_ERR_CUDA;
    // h = silu(gate) * up; x += Wd h — one launch for few rows
    EpiSwiGLU eg{hm, I};
    if (h->chain && chain_ok(M, h->num_sms)) {
      s = run_gemm_chain(h, DFLASH_KERNEL_GEMM_MLP, true, nrm, M, H, h->wgu[l], 2 * I, eg, false,
                         hm, I, h->wdown[l], H, er, partial, lw.partial_cap, st);
      if (s != DFLASH_OK) return s;
    } else {
      s = run_gemm(h, DFLASH_KERNEL_GEMM_GATE_UP, true, true, nrm, M, H, h->wgu[l], 2 * I, eg,
                   partial, lw.partial_cap, st);
      if (s != DFLASH_OK) return s;
      s = run_gemm(h, DFLASH_KERNEL_GEMM_DOWN, false, true, hm, M, I, h->wdown[l], H, er, partial,
                   lw.partial_cap, st);
      if (s != DFLASH_OK) return s;
    }
    LaunchScope scope(h, DFLASH_KERNEL_RMSNORM, st);
    if (l + 1 < c.n_layers) {
      launch_k(h->pdl, rmsnorm_rows_kernel, dim3(M), dim3(256), 0, st, x, h->in_norm_w[l + 1], nrm,
               H, c.rms_eps, 0, bs);
    } else {
      // final norm on the kept rows (block slots 1..bs-1) only
      launch_k(h->pdl, rmsnorm_rows_kernel, dim3(B * K), dim3(256), 0, st, x, h->final_norm_w,
               frows, H, c.rms_eps, K, bs);
    }
    if (cudaGetLastError() != cudaSuccess) return DFLASH_ERR_CUDA;
  }
  return DFLASH_OK;
}
}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
namespace {
dflash_status create_handle(const dflash_config* cfg, const dflash_weights* w, int device,
                            int vocab_start, int vocab_count, int tp_rank, int tp_size,
                            dflash_handle** out);
}  // namespace

extern "C" {

const char* dflash_status_string(dflash_status s) {
  switch (s) {
    case DFLASH_OK: return "DFLASH_OK";
    case DFLASH_ERR_INVALID_ARG: return "DFLASH_ERR_INVALID_ARG";
    case DFLASH_ERR_CUDA: return "DFLASH_ERR_CUDA";
    case DFLASH_ERR_WORKSPACE: return "DFLASH_ERR_WORKSPACE";
    case DFLASH_ERR_UNSUPPORTED_SHAPE: return "DFLASH_ERR_UNSUPPORTED_SHAPE";
    case DFLASH_ERR_DEVICE_BOUNDS: return "DFLASH_ERR_DEVICE_BOUNDS";
    case DFLASH_ERR_UNIMPLEMENTED: return "DFLASH_ERR_UNIMPLEMENTED";
    case DFLASH_ERR_DEVICE_TIMEOUT: return "DFLASH_ERR_DEVICE_TIMEOUT";
    case DFLASH_ERR_RANGE: return "DFLASH_ERR_RANGE";
    case DFLASH_ERR_EXCHANGE: return "DFLASH_ERR_EXCHANGE";
  }
  return "DFLASH_ERR_UNKNOWN";
}

const char* dflash_version(void) { return "dflash-b200 0.1 (sm_100a)"; }

dflash_status dflash_set_wait_limit(int device, long long cycles) {
  if (cycles <= 0) return DFLASH_ERR_INVALID_ARG;
  DF_CUDA(use_device(device));
  DF_CUDA(cudaMemcpyToSymbol(g_wait_limit_cycles, &cycles, sizeof(cycles)));
  return DFLASH_OK;
}

dflash_status dflash_selftest_wait_timeout(dflash_handle* h, void* stream) {
  if (!h) return DFLASH_ERR_INVALID_ARG;
  DF_CUDA(use_device(h->device));
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(h->dev_err);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

dflash_status dflash_create(const dflash_config* cfg, const dflash_weights* w, int device,
                            dflash_handle** out) {
  return dflash_create_vocab_shard(cfg, w, device, 0, cfg ? cfg->vocab : 0, out);
}

dflash_status dflash_create_vocab_shard(const dflash_config* cfg, const dflash_weights* w,
                                        int device, int vocab_start, int vocab_count,
                                        dflash_handle** out) {
  return create_handle(cfg, w, device, vocab_start, vocab_count, 0, 1, out);
}

dflash_status dflash_create_tp_shard(const dflash_config* cfg, const dflash_weights* w,
                                     int device, int tp_rank, int tp_size, int vocab_start,
                                     int vocab_count, dflash_handle** out) {
  if (tp_size < 1 || tp_rank < 0 || tp_rank >= tp_size) {
    if (out) *out = nullptr;
    return DFLASH_ERR_INVALID_ARG;
  }
  return create_handle(cfg, w, device, vocab_start, vocab_count, tp_rank, tp_size, out);
}

}  // extern "C"

namespace {
// A handle over the whole model (tp_size 1) or over tensor-parallel rank
// tp_rank's slice of it: kv heads [r Hkv/S, (r+1) Hkv/S) with their query
// heads, MLP features [r I/S, (r+1) I/S), the matching columns of Wo and
// W_down, and the LM-head vocabulary rows [vocab_start, + vocab_count).
dflash_status create_handle(const dflash_config* cfg, const dflash_weights* w, int device,
                            int vocab_start, int vocab_count, int tp_rank, int tp_size,
                            dflash_handle** out) {
  if (!out) return DFLASH_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || !w) return DFLASH_ERR_INVALID_ARG;
  const dflash_config& c = *cfg;
  if (vocab_start < 0 || vocab_count <= 0 || vocab_count > c.vocab - vocab_start)
    return DFLASH_ERR_INVALID_ARG;
  if (vocab_start % 32 || vocab_count % 32) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if (c.hidden <= 0 || c.n_layers <= 0 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 ||
      c.head_dim <= 0 || c.intermediate <= 0 || c.vocab <= 0 || c.n_target_layers <= 0 ||
      c.block_size <= 0 || c.page_size <= 0 || c.max_position <= 0 || !(c.rms_eps >= 0.f) ||
      !(c.rope_theta > 0.f))
    return DFLASH_ERR_INVALID_ARG;
  if (c.mask_token_id < 0 || c.mask_token_id >= c.vocab) return DFLASH_ERR_INVALID_ARG;
  if (c.head_dim != 64 && c.head_dim != 128) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if (c.hidden % 64 || (c.n_q_heads * c.head_dim) % 64 || c.intermediate % 64 ||
      c.vocab % 32 || c.n_q_heads % c.n_kv_heads || c.page_size != 16 || c.block_size < 2 ||
      c.block_size > 64 || c.n_layers > kMaxLayers)
    return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if (c.block_size * (c.n_q_heads / c.n_kv_heads) > 16 * kAttnMaxComputeWarps)
    return DFLASH_ERR_UNSUPPORTED_SHAPE;
  // tensor-parallel slices: whole kv groups per rank, MLP features in 64s
  if (c.n_kv_heads % tp_size || c.intermediate % (64 * tp_size))
    return DFLASH_ERR_UNSUPPORTED_SHAPE;
  const int L = c.n_layers;
  if (!w->fc_w || !w->hidden_norm_w || !w->embed || !w->lm_head || !w->final_norm_w ||
      !w->in_norm_w || !w->post_norm_w || !w->wq || !w->wk || !w->wv || !w->wo ||
      !w->q_norm_w || !w->k_norm_w || !w->w_gate || !w->w_up || !w->w_down)
    return DFLASH_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l)
    if (!w->in_norm_w[l] || !w->post_norm_w[l] || !w->wq[l] || !w->wk[l] || !w->wv[l] ||
        !w->wo[l] || !w->q_norm_w[l] || !w->k_norm_w[l] || !w->w_gate[l] || !w->w_up[l] ||
        !w->w_down[l])
      return DFLASH_ERR_INVALID_ARG;
  // the GEMM weights are read with 16-byte loads when the handle packs them
  auto misaligned = [](const void* q) { return reinterpret_cast<uintptr_t>(q) % 16 != 0; };
  if (misaligned(w->fc_w)) return DFLASH_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l)
    if (misaligned(w->wq[l]) || misaligned(w->wk[l]) || misaligned(w->wv[l]) ||
        misaligned(w->wo[l]) || misaligned(w->w_gate[l]) || misaligned(w->w_up[l]) ||
        misaligned(w->w_down[l]))
      return DFLASH_ERR_INVALID_ARG;
  if (c.target_layer_ids) {
    for (int t = 0; t < c.n_target_layers; ++t)
      if (c.target_layer_ids[t] < 0) return DFLASH_ERR_INVALID_ARG;
  }
  if (!encode_fn()) return DFLASH_ERR_CUDA;

  dflash_handle* h = new (std::nothrow) dflash_handle();
  if (!h) return DFLASH_ERR_CUDA;
  h->cfg = c;
  // a shard's geometry is its slice of the heads and MLP features
  h->cfg.n_q_heads = c.n_q_heads / tp_size;
  h->cfg.n_kv_heads = c.n_kv_heads / tp_size;
  h->cfg.intermediate = c.intermediate / tp_size;
  h->tp_rank = tp_rank;
  h->tp_size = tp_size;
  h->vocab_start = vocab_start;
  h->vocab_count = vocab_count;
  if (c.target_layer_ids) h->target_layer_ids.assign(c.target_layer_ids, c.target_layer_ids + c.n_target_layers);
  h->cfg.target_layer_ids = h->target_layer_ids.empty() ? nullptr : h->target_layer_ids.data();
  h->device = device;
  auto fail = [h](dflash_status s) {
    free_handle(h);
    return s;
  };
  if (cudaSetDevice(device) != cudaSuccess) return fail(DFLASH_ERR_CUDA);
  if (cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return fail(DFLASH_ERR_CUDA);
  int major = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
  if (major != 10) return fail(DFLASH_ERR_UNSUPPORTED_SHAPE);

  // local (this shard's) sizes, and where its slices start in the whole weights
  const int H = c.hidden, D = c.head_dim, Hq = h->cfg.n_q_heads, Hkv = h->cfg.n_kv_heads,
            I = h->cfg.intermediate;
  const int Hq_all = c.n_q_heads, I_all = c.intermediate;
  auto rows_at = [](const void* base, size_t row, size_t row_len) {
    return static_cast<const void*>(static_cast<const uint16_t*>(base) + row * row_len);
  };
  const size_t q_row0 = static_cast<size_t>(tp_rank) * Hq * D;     // wq rows, wo columns
  const size_t kv_row0 = static_cast<size_t>(tp_rank) * Hkv * D;   // wk / wv rows
  const size_t f_row0 = static_cast<size_t>(tp_rank) * I;          // gate/up rows, down columns
  h->hidden_norm_w = static_cast<const bf16*>(w->hidden_norm_w);
  h->embed = static_cast<const bf16*>(w->embed);
  h->final_norm_w = static_cast<const bf16*>(w->final_norm_w);
  for (int l = 0; l < L; ++l) {
    h->in_norm_w.push_back(static_cast<const bf16*>(w->in_norm_w[l]));
    h->post_norm_w.push_back(static_cast<const bf16*>(w->post_norm_w[l]));
    h->q_norm_w.push_back(static_cast<const bf16*>(w->q_norm_w[l]));
    h->k_norm_w.push_back(static_cast<const bf16*>(w->k_norm_w[l]));
  }

  cudaStream_t st;
  if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess)
    return fail(DFLASH_ERR_CUDA);
  auto fail_st = [&](dflash_status s) {
    cudaStreamSynchronize(st);
    cudaStreamDestroy(st);
    return fail(s);
  };
  const size_t rowb = static_cast<size_t>(H) * 2;
  // QKV: [wq; wk; wv]
  for (int l = 0; l < L; ++l) {
    f16* p = nullptr;
    if (cudaMalloc(&p, static_cast<size_t>(Hq + 2 * Hkv) * D * rowb) != cudaSuccess)
      return fail_st(DFLASH_ERR_CUDA);
    h->wqkv.push_back(p);
    if (cudaMemcpyAsync(p, rows_at(w->wq[l], q_row0, H), static_cast<size_t>(Hq) * D * rowb,
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(p + static_cast<size_t>(Hq) * D * H, rows_at(w->wk[l], kv_row0, H),
                        static_cast<size_t>(Hkv) * D * rowb, cudaMemcpyDeviceToDevice,
                        st) != cudaSuccess ||
        cudaMemcpyAsync(p + static_cast<size_t>(Hq + Hkv) * D * H, rows_at(w->wv[l], kv_row0, H),
                        static_cast<size_t>(Hkv) * D * rowb, cudaMemcpyDeviceToDevice,
                        st) != cudaSuccess)
      return fail_st(DFLASH_ERR_CUDA);
  }
  // gate / up interleaved in blocks of 16 rows: [g 16 | u 16] per 32 packed rows
  for (int l = 0; l < L; ++l) {
    f16* p = nullptr;
    if (cudaMalloc(&p, static_cast<size_t>(2 * I) * rowb) != cudaSuccess)
      return fail_st(DFLASH_ERR_CUDA);
    h->wgu.push_back(p);
    if (cudaMemcpy2DAsync(p, 32 * rowb, rows_at(w->w_gate[l], f_row0, H), 16 * rowb, 16 * rowb,
                          I / 16, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        cudaMemcpy2DAsync(p + 16 * static_cast<size_t>(H), 32 * rowb,
                          rows_at(w->w_up[l], f_row0, H), 16 * rowb, 16 * rowb, I / 16,
                          cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return fail_st(DFLASH_ERR_CUDA);
  }
  // all layers' K/V projections stacked: per layer [wk; wv]
  const size_t kvrows = static_cast<size_t>(Hkv) * D;
  if (cudaMalloc(&h->wkv, static_cast<size_t>(L) * 2 * kvrows * rowb) != cudaSuccess)
    return fail_st(DFLASH_ERR_CUDA);
  for (int l = 0; l < L; ++l) {
    if (cudaMemcpyAsync(h->wkv + (2 * l) * kvrows * H, rows_at(w->wk[l], kv_row0, H),
                        kvrows * rowb, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(h->wkv + (2 * l + 1) * kvrows * H, rows_at(w->wv[l], kv_row0, H),
                        kvrows * rowb, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return fail_st(DFLASH_ERR_CUDA);
  }
  if (cudaMalloc(&h->knorm_all, static_cast<size_t>(L) * D * 2) != cudaSuccess)
    return fail_st(DFLASH_ERR_CUDA);
  for (int l = 0; l < L; ++l)
    if (cudaMemcpyAsync(h->knorm_all + static_cast<size_t>(l) * D, w->k_norm_w[l],
                        static_cast<size_t>(D) * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return fail_st(DFLASH_ERR_CUDA);
  // O projections and the LM head: fp16 copies
  for (int l = 0; l < L; ++l) {
    f16* p = nullptr;
    if (cudaMalloc(&p, static_cast<size_t>(H) * Hq * D * 2) != cudaSuccess)
      return fail_st(DFLASH_ERR_CUDA);
    h->wo.push_back(p);
    // this shard's columns of Wo [H, Hq_all * D] (all of them for one shard)
    if (cudaMemcpy2DAsync(p, static_cast<size_t>(Hq) * D * 2, rows_at(w->wo[l], q_row0, 1),
                          static_cast<size_t>(Hq_all) * D * 2, static_cast<size_t>(Hq) * D * 2, H,
                          cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return fail_st(DFLASH_ERR_CUDA);
  }
  // the LM head rows of this handle: a vocabulary shard (dflash_create_vocab_shard)
  // is given its rows; a tensor-parallel shard takes them out of the whole head
  const void* lm_src = tp_size > 1 ? rows_at(w->lm_head, static_cast<size_t>(vocab_start), H)
                                   : w->lm_head;
  if (cudaMalloc(&h->lm_head16, static_cast<size_t>(vocab_count) * rowb) != cudaSuccess ||
      cudaMemcpyAsync(h->lm_head16, lm_src, static_cast<size_t>(vocab_count) * rowb,
                      cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return fail_st(DFLASH_ERR_CUDA);
  // fp16 range statistics of the converted weights and of the norm weights
  // whose RMSNorm outputs are stored in fp16 (device words, read back below)
  unsigned* stats = nullptr;
  if (cudaMalloc(&stats, 4 * sizeof(unsigned)) != cudaSuccess) return fail_st(DFLASH_ERR_CUDA);
  h->range_stats = stats;
  if (cudaMemsetAsync(stats, 0, 4 * sizeof(unsigned), st) != cudaSuccess)
    return fail_st(DFLASH_ERR_CUDA);
  size_t f16_values = 0;
  {
    auto to_f16 = [&](void* ptr, size_t n) {
      bf16_to_f16_kernel<<<1184, 256, 0, st>>>(static_cast<uint16_t*>(ptr), n, stats);
      f16_values += n;
      return cudaGetLastError() == cudaSuccess;
    };
    auto norm_max = [&](const bf16* w, int n) {
      absmax_bf16_kernel<<<1, 256, 0, st>>>(w, n, stats);
      return cudaGetLastError() == cudaSuccess;
    };
    bool ok = norm_max(h->hidden_norm_w, H) && norm_max(h->final_norm_w, H);
    for (int l = 0; l < L; ++l)
      ok = ok && norm_max(h->in_norm_w[l], H) && norm_max(h->post_norm_w[l], H);
    for (int l = 0; l < L; ++l) {
      ok = ok && to_f16(h->wqkv[l], static_cast<size_t>(Hq + 2 * Hkv) * D * H);
      ok = ok && to_f16(h->wgu[l], static_cast<size_t>(2 * I) * H);
      ok = ok && to_f16(h->wo[l], static_cast<size_t>(H) * Hq * D);
    }
    ok = ok && to_f16(h->wkv, static_cast<size_t>(L) * 2 * kvrows * H);
    ok = ok && to_f16(h->lm_head16, static_cast<size_t>(vocab_count) * H);
    if (!ok) return fail_st(DFLASH_ERR_CUDA);
  }
  // every GEMM weight into the tile-contiguous layout
  {
    // packs row-major [N, K] `src` into a new buffer stored at *out
    auto pack = [&](const void* src, int N, int K, void** out, int ld = 0) {
      const size_t bytes = static_cast<size_t>(cdiv(N, kPackRows)) * kPackRows * K * 2;
      if (cudaMalloc(out, bytes) != cudaSuccess) {
        *out = nullptr;
        return false;
      }
      pack_tiles_kernel<<<1184, 256, 0, st>>>(static_cast<const uint16_t*>(src),
                                              static_cast<uint16_t*>(*out), N, K, ld ? ld : K,
                                              bytes / 16, 0);
      return cudaGetLastError() == cudaSuccess;
    };
    // replaces a row-major copy owned by the handle with its packed form
    auto repack = [&](f16*& rm, int N, int K) {
      void* p = nullptr;
      if (!pack(rm, N, K, &p) || cudaStreamSynchronize(st) != cudaSuccess) {
        cudaFree(p);
        return false;
      }
      cudaFree(rm);
      rm = static_cast<f16*>(p);
      return true;
    };
    bool ok = true;
    for (int l = 0; ok && l < L; ++l) {
      ok = ok && repack(h->wqkv[l], (Hq + 2 * Hkv) * D, H);
      ok = ok && repack(h->wgu[l], 2 * I, H);
      ok = ok && repack(h->wo[l], H, Hq * D);
    }
    ok = ok && repack(h->wkv, L * 2 * Hkv * D, H);
    ok = ok && repack(h->lm_head16, vocab_count, H);
    for (int l = 0; ok && l < L; ++l) {
      void* p = nullptr;
      ok = pack(rows_at(w->w_down[l], f_row0, 1), H, I, &p, I_all);
      if (p) h->wdown.push_back(static_cast<bf16*>(p));
    }
    if (ok) {
      void* p = nullptr;
      ok = pack(w->fc_w, H, c.n_target_layers * H, &p);
      h->fcw = static_cast<bf16*>(p);
    }
    if (!ok || cudaStreamSynchronize(st) != cudaSuccess) return fail_st(DFLASH_ERR_CUDA);
  }
  if (cudaMalloc(&h->rope, static_cast<size_t>(c.max_position) * (D / 2) * sizeof(float2)) !=
      cudaSuccess)
    return fail_st(DFLASH_ERR_CUDA);
  rope_table_kernel<<<c.max_position, 64, 0, st>>>(h->rope, c.max_position, D / 2,
                                                    static_cast<double>(c.rope_theta));
  if (cudaGetLastError() != cudaSuccess) return fail_st(DFLASH_ERR_CUDA);
  if (cudaMalloc(&h->dev_err, sizeof(unsigned)) != cudaSuccess ||
      cudaMemsetAsync(h->dev_err, 0, sizeof(unsigned), st) != cudaSuccess)
    return fail_st(DFLASH_ERR_CUDA);
  if (cudaMalloc(&h->counters, kCounterSlots * sizeof(unsigned)) != cudaSuccess ||
      cudaMemsetAsync(h->counters, 0, kCounterSlots * sizeof(unsigned), st) != cudaSuccess)
    return fail_st(DFLASH_ERR_CUDA);

  // kernel attributes (set once, outside any stream capture)
  if (cudaFuncSetAttribute(gemm_chain_kernel<256, EpiSwiGLU, EpiResidAdd>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kGemmSmemLimit) != cudaSuccess ||
      set_gemm_attrs_all<EpiStoreF32>() != cudaSuccess ||
      set_gemm_attrs_all<EpiResidAdd>() != cudaSuccess ||
      set_gemm_attrs_all<EpiSwiGLU>() != cudaSuccess ||
      set_gemm_attrs_all<EpiArgmax>() != cudaSuccess ||
      set_gemm_attrs_all<EpiQKV<64>>() != cudaSuccess ||
      set_gemm_attrs_all<EpiQKV<128>>() != cudaSuccess ||
      set_gemm_attrs_all<EpiKVInject<64>>() != cudaSuccess ||
      set_gemm_attrs_all<EpiKVInject<128>>() != cudaSuccess ||
      set_attn_attrs<64>() != cudaSuccess || set_attn_attrs<128>() != cudaSuccess)
    return fail_st(DFLASH_ERR_CUDA);
  if (cudaStreamSynchronize(st) != cudaSuccess) return fail_st(DFLASH_ERR_CUDA);
  // the fp16 storage of the path holds these weights and norm outputs only in
  // fp16's range: refuse weights beyond it, weights so small that more than 1%
  // of them would be fp16 subnormals, and norm weights whose RMSNorm outputs
  // (|y_i| <= sqrt(hidden) * max|w|) could overflow fp16
  unsigned hs[4] = {0, 0, 0, 0};
  if (cudaMemcpy(hs, stats, sizeof(hs), cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail_st(DFLASH_ERR_CUDA);
  float wmax, nmax;
  std::memcpy(&wmax, &hs[0], 4);
  std::memcpy(&nmax, &hs[2], 4);
  h->fp16_weight_absmax = wmax;
  h->fp16_subnormal_fraction = f16_values ? static_cast<double>(hs[1]) / f16_values : 0.0;
  h->norm_output_bound = std::sqrt(static_cast<double>(H)) * nmax;
  if (!(wmax <= kFp16Max) || h->fp16_subnormal_fraction > kFp16SubnormalLimit ||
      !(h->norm_output_bound <= kFp16Max))
    return fail_st(DFLASH_ERR_RANGE);
  cudaStreamDestroy(st);
  *out = h;
  return DFLASH_OK;
}
}  // namespace

extern "C" {

void dflash_destroy(dflash_handle* h) {
  if (!h) return;
  cudaSetDevice(h->device);
  free_handle(h);
}

size_t dflash_inject_workspace_bytes(const dflash_handle* h, int max_rows) {
  if (!h || max_rows <= 0) return 0;
  return inject_layout(h, max_rows).total;
}

size_t dflash_propose_workspace_bytes(const dflash_handle* h, int max_batch,
                                      int max_pages_per_seq) {
  if (!h || max_batch <= 0 || max_pages_per_seq <= 0) return 0;
  return propose_layout(h, max_batch, max_pages_per_seq).total;
}

size_t dflash_propose_final_rows_offset(const dflash_handle* h, int B, int max_pages_per_seq) {
  if (!h || B <= 0 || max_pages_per_seq <= 0) return static_cast<size_t>(-1);
  return propose_layout(h, B, max_pages_per_seq).frows;
}


size_t dflash_verify_workspace_bytes(int B, int K, int V) {
  if (B <= 0 || K < 0 || V <= 0) return 0;
  return plan_verify(B, K, V).bytes;
}

dflash_status dflash_paged_slots(const int64_t* positions, const int64_t* req_ids, int n,
                                 const int32_t* block_table, int max_pages_per_seq,
                                 int page_size, int64_t* slots, void* stream) {
  if (n < 0 || max_pages_per_seq <= 0 || page_size <= 0) return DFLASH_ERR_INVALID_ARG;
  if (n == 0) return DFLASH_OK;
  if (!positions || !req_ids || !block_table || !slots) return DFLASH_ERR_INVALID_ARG;
  dflash_status s = set_device_for(static_cast<cudaStream_t>(stream), slots);
  if (s != DFLASH_OK) return s;
  launch_k(pdl_default(), paged_slots_kernel, dim3(cdiv(n, 256)), dim3(256), 0,
           static_cast<cudaStream_t>(stream), positions, req_ids, block_table, n,
           max_pages_per_seq, page_size, slots);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

dflash_status dflash_prepare_proposal_inputs(
    const int64_t* target_positions, int n, const int32_t* last_token_indices, int B,
    const int32_t* cur_sampled, int cur_width, const int32_t* cur_num_draft,
    const int32_t* prev_sampled, int prev_width, const int32_t* prev_num_draft,
    const int32_t* block_table, int max_pages_per_seq, int page_size, int vocab,
    int64_t* positions_out, int64_t* slot_mapping_out, int32_t* seq_lens_out,
    int32_t* bonus_out, unsigned* device_error, void* stream) {
  if (n < 0 || B < 0 || cur_width < 1 || max_pages_per_seq < 1 || page_size < 1 || vocab < 1)
    return DFLASH_ERR_INVALID_ARG;
  if ((prev_sampled == nullptr) != (prev_num_draft == nullptr)) return DFLASH_ERR_INVALID_ARG;
  if (prev_sampled && prev_width < 1) return DFLASH_ERR_INVALID_ARG;
  if (n == 0 && B == 0) return DFLASH_OK;
  if ((n > 0 && (!target_positions || !positions_out || !slot_mapping_out)) ||
      (B > 0 && (!cur_sampled || !cur_num_draft || !seq_lens_out || !bonus_out ||
                 !last_token_indices || !block_table)))
    return DFLASH_ERR_INVALID_ARG;
  dflash_status s = set_device_for(static_cast<cudaStream_t>(stream),
                                   n > 0 ? static_cast<const void*>(positions_out)
                                         : static_cast<const void*>(seq_lens_out));
  if (s != DFLASH_OK) return s;
  launch_k(pdl_default(), prepare_proposal_kernel, dim3(cdiv(std::max(n, B), 256)), dim3(256), 0,
           static_cast<cudaStream_t>(stream), target_positions, n, last_token_indices, B,
           cur_sampled, cur_width, cur_num_draft, prev_sampled, prev_sampled ? prev_width : 1,
           prev_num_draft, block_table, max_pages_per_seq, page_size, vocab, positions_out,
           slot_mapping_out, seq_lens_out, bonus_out, device_error);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

dflash_status dflash_inject_context(dflash_handle* h, const void* aux, const int64_t* positions,
                                    const int64_t* slot_mapping, int n, void* const* k_cache,
                                    void* const* v_cache, int num_pages, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!h || n < 0) return DFLASH_ERR_INVALID_ARG;
  if (n == 0) return DFLASH_OK;
  const dflash_config& c = h->cfg;
  if (!aux || !positions || !slot_mapping || !k_cache || !v_cache || num_pages <= 0 ||
      !workspace)
    return DFLASH_ERR_INVALID_ARG;
  for (int l = 0; l < c.n_layers; ++l)
    if (!k_cache[l] || !v_cache[l]) return DFLASH_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return DFLASH_ERR_INVALID_ARG;
  const InjectWs lw = inject_layout(h, n);
  if (workspace_bytes < lw.total) return DFLASH_ERR_WORKSPACE;
  DF_CUDA(use_device(h->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = c.hidden, D = c.head_dim;
  float* fcx = at<float>(workspace, lw.fcx);
  f16* ctx = at<f16>(workspace, lw.ctx);
  float* partial = at<float>(workspace, lw.partial);

  // (1) fc over the concatenated tapped states
  EpiStoreF32 e1{fcx, H};
  dflash_status s = run_gemm(h, DFLASH_KERNEL_GEMM_FC, false, true, aux, n, c.n_target_layers * H,
                             h->fcw, H, e1, partial, lw.partial_cap, st);
  if (s != DFLASH_OK) return s;
  // (2) hidden_norm
  {
    LaunchScope scope(h, DFLASH_KERNEL_RMSNORM, st);
    launch_k(h->pdl, rmsnorm_rows_kernel, dim3(n), dim3(256), 0, st, fcx, h->hidden_norm_w, ctx, H,
             c.rms_eps, 0, 0);
  }
  if (cudaGetLastError() != cudaSuccess) return DFLASH_ERR_CUDA;
  // (3) every layer's K/V at once, k_norm + RoPE, paged scatter
  const int NKV = c.n_layers * 2 * c.n_kv_heads * D;
  if (D == 128) {
    EpiKVInject<128> e3{};
    for (int l = 0; l < c.n_layers; ++l) {
      e3.k_cache[l] = static_cast<bf16*>(k_cache[l]);
      e3.v_cache[l] = static_cast<bf16*>(v_cache[l]);
    }
    e3.k_norm_w = h->knorm_all;
    e3.rope = h->rope;
    e3.positions = positions;
    e3.slots = slot_mapping;
    e3.max_pos = c.max_position;
    e3.Hkv = c.n_kv_heads;
    e3.P = c.page_size;
    e3.num_pages = num_pages;
    e3.eps = c.rms_eps;
    e3.err = h->dev_err;
    s = run_gemm(h, DFLASH_KERNEL_GEMM_KV_INJECT, true, true, ctx, n, H, h->wkv, NKV, e3, partial,
                 lw.partial_cap, st);
  } else {
    EpiKVInject<64> e3{};
    for (int l = 0; l < c.n_layers; ++l) {
      e3.k_cache[l] = static_cast<bf16*>(k_cache[l]);
      e3.v_cache[l] = static_cast<bf16*>(v_cache[l]);
    }
    e3.k_norm_w = h->knorm_all;
    e3.rope = h->rope;
    e3.positions = positions;
    e3.slots = slot_mapping;
    e3.max_pos = c.max_position;
    e3.Hkv = c.n_kv_heads;
    e3.P = c.page_size;
    e3.num_pages = num_pages;
    e3.eps = c.rms_eps;
    e3.err = h->dev_err;
    s = run_gemm(h, DFLASH_KERNEL_GEMM_KV_INJECT, true, true, ctx, n, H, h->wkv, NKV, e3, partial,
                 lw.partial_cap, st);
  }
  return s;
}


}  // extern "C"

namespace {
// The proposal up to the LM head's greedy pick; then either the drafts
// (draft_keys == nullptr) or this handle's vocabulary shard's ordered keys.
dflash_status propose_impl(dflash_handle* h, const int32_t* bonus_tokens,
                           const int32_t* seq_lens, const int32_t* block_table, int B,
                           int max_pages_per_seq, void* const* k_cache, void* const* v_cache,
                           int num_pages, int32_t* draft_tokens, int32_t* block_tokens,
                           int64_t* draft_keys, float* logits_out, void* workspace,
                           size_t workspace_bytes, void* stream,
                           dflash_allreduce_fn exchange = nullptr, void* user = nullptr) {
  if (!h || B < 0) return DFLASH_ERR_INVALID_ARG;
  // a tensor-parallel shard proposes only through dflash_propose_tp (with an
  // exchange hook), and only a shard takes one
  if ((h->tp_size > 1) != (exchange != nullptr)) return DFLASH_ERR_INVALID_ARG;
  if (B == 0) return DFLASH_OK;
  const dflash_config& c = h->cfg;
  if (!bonus_tokens || !seq_lens || !block_table || max_pages_per_seq <= 0 || !k_cache ||
      !v_cache || num_pages <= 0 || !(draft_tokens || draft_keys) || !workspace)
    return DFLASH_ERR_INVALID_ARG;
  for (int l = 0; l < c.n_layers; ++l)
    if (!k_cache[l] || !v_cache[l]) return DFLASH_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return DFLASH_ERR_INVALID_ARG;
  // (the attention grid carries the request index in its y dimension)
  if (static_cast<int64_t>(B) * c.block_size > (1 << 24) || B > kMaxAttnRequests)
    return DFLASH_ERR_UNSUPPORTED_SHAPE;
  const ProposeWs lw = propose_layout(h, B, max_pages_per_seq);
  if (workspace_bytes < lw.total) return DFLASH_ERR_WORKSPACE;
  DF_CUDA(use_device(h->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int bs = c.block_size, K = bs - 1, M = B * bs, H = c.hidden;
  float* x = at<float>(workspace, lw.x);
  f16* nrm = at<f16>(workspace, lw.nrm);
  f16* frows = at<f16>(workspace, lw.frows);
  unsigned long long* keys = at<unsigned long long>(workspace, lw.keys);
  float* partial = at<float>(workspace, lw.partial);

  {
    LaunchScope scope(h, DFLASH_KERNEL_EMBED_NORM, st);
    launch_k(h->pdl, embed_norm_kernel, dim3(M), dim3(256), 0, st, bonus_tokens, c.mask_token_id,
             h->embed, h->in_norm_w[0], x, nrm, keys, B * K, bs, H, c.vocab, c.rms_eps,
             h->dev_err);
  }
  if (cudaGetLastError() != cudaSuccess) return DFLASH_ERR_CUDA;
  dflash_status s = (c.head_dim == 128)
                        ? propose_layers<128>(h, lw, workspace, seq_lens, block_table, B,
                                              max_pages_per_seq, k_cache, v_cache, num_pages, st,
                                              exchange, user)
                        : propose_layers<64>(h, lw, workspace, seq_lens, block_table, B,
                                             max_pages_per_seq, k_cache, v_cache, num_pages, st,
                                             exchange, user);
  if (s != DFLASH_OK) return s;
  // aliased target LM head (this handle's vocabulary rows) with the greedy
  // pick fused into its epilogue
  EpiArgmax ea{keys, logits_out, h->vocab_count, static_cast<uint32_t>(h->vocab_start)};
  s = run_gemm(h, DFLASH_KERNEL_GEMM_LM_HEAD, true, true, frows, B * K, H, h->lm_head16,
               h->vocab_count, ea, partial, lw.partial_cap, st);
  if (s != DFLASH_OK) return s;
  {
    LaunchScope scope(h, DFLASH_KERNEL_ARGMAX_FINALIZE, st);
    if (draft_keys)
      launch_k(h->pdl, keys_export_kernel, dim3(cdiv(B * K, 256)), dim3(256), 0, st, keys,
               B * K, draft_keys);
    else
      launch_k(h->pdl, argmax_finalize_kernel, dim3(cdiv(M, 256)), dim3(256), 0, st, keys,
               bonus_tokens, draft_tokens, block_tokens, B, bs);
  }
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}
}  // namespace

extern "C" {

dflash_status dflash_propose(dflash_handle* h, const int32_t* bonus_tokens,
                             const int32_t* seq_lens, const int32_t* block_table, int B,
                             int max_pages_per_seq, void* const* k_cache, void* const* v_cache,
                             int num_pages, int32_t* draft_tokens, int32_t* block_tokens,
                             float* logits_out, void* workspace, size_t workspace_bytes,
                             void* stream) {
  // a vocabulary shard's own argmax is not a draft: dflash_propose_keys
  if (h && h->vocab_count != h->cfg.vocab) return DFLASH_ERR_INVALID_ARG;
  if (!draft_tokens && B > 0) return DFLASH_ERR_INVALID_ARG;
  return propose_impl(h, bonus_tokens, seq_lens, block_table, B, max_pages_per_seq, k_cache,
                      v_cache, num_pages, draft_tokens, block_tokens, nullptr, logits_out,
                      workspace, workspace_bytes, stream);
}

dflash_status dflash_propose_keys(dflash_handle* h, const int32_t* bonus_tokens,
                                  const int32_t* seq_lens, const int32_t* block_table, int B,
                                  int max_pages_per_seq, void* const* k_cache,
                                  void* const* v_cache, int num_pages, int64_t* draft_keys,
                                  float* logits_out, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (!draft_keys && B > 0) return DFLASH_ERR_INVALID_ARG;
  return propose_impl(h, bonus_tokens, seq_lens, block_table, B, max_pages_per_seq, k_cache,
                      v_cache, num_pages, nullptr, nullptr, draft_keys, logits_out, workspace,
                      workspace_bytes, stream);
}

dflash_status dflash_propose_tp(dflash_handle* h, const int32_t* bonus_tokens,
                                const int32_t* seq_lens, const int32_t* block_table, int B,
                                int max_pages_per_seq, void* const* k_cache,
                                void* const* v_cache, int num_pages, int64_t* draft_keys,
                                float* logits_out, void* workspace, size_t workspace_bytes,
                                void* stream, dflash_allreduce_fn exchange, void* user) {
  if (!h || h->tp_size < 2 || !exchange) return DFLASH_ERR_INVALID_ARG;
  if (!draft_keys && B > 0) return DFLASH_ERR_INVALID_ARG;
  return propose_impl(h, bonus_tokens, seq_lens, block_table, B, max_pages_per_seq, k_cache,
                      v_cache, num_pages, nullptr, nullptr, draft_keys, logits_out, workspace,
                      workspace_bytes, stream, exchange, user);
}

dflash_status dflash_finalize_draft_keys(const int64_t* draft_keys, const int32_t* bonus_tokens,
                                         int B, int block_size, int vocab,
                                         int32_t* draft_tokens, int32_t* block_tokens,
                                         unsigned* device_error, void* stream) {
  if (B < 0 || block_size < 2 || vocab < 1) return DFLASH_ERR_INVALID_ARG;
  if (B == 0) return DFLASH_OK;
  if (!draft_keys || !bonus_tokens || !draft_tokens) return DFLASH_ERR_INVALID_ARG;
  dflash_status s = set_device_for(static_cast<cudaStream_t>(stream), draft_tokens);
  if (s != DFLASH_OK) return s;
  launch_k(pdl_default(), draft_keys_finalize_kernel, dim3(cdiv(B * block_size, 256)), dim3(256),
           0, static_cast<cudaStream_t>(stream), draft_keys, bonus_tokens, B, block_size, vocab,
           draft_tokens, block_tokens, device_error);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

dflash_status dflash_verify_greedy(const int32_t* drafts, const float* target_logits, int B,
                                   int K, int V, int32_t* out_tokens, int32_t* num_accepted,
                                   int32_t* bonus, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (B < 0 || K < 0 || V <= 0 || K > 128) return DFLASH_ERR_INVALID_ARG;
  if (B == 0) return DFLASH_OK;
  if (static_cast<int64_t>(B) * (K + 1) > (1 << 30)) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if ((K > 0 && !drafts) || !target_logits || !out_tokens || !num_accepted || !bonus ||
      !workspace)
    return DFLASH_ERR_INVALID_ARG;
  const VerifyPlan vp = plan_verify(B, K, V);
  if (workspace_bytes < vp.bytes) return DFLASH_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(target_logits) % 16 && V % 4 == 0)
    return DFLASH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dflash_status s = set_device_for(st, out_tokens);
  if (s != DFLASH_OK) return s;
  unsigned long long* part = static_cast<unsigned long long*>(workspace);
  launch_k(pdl_default(), verify_partial_kernel, dim3(vp.chunks, std::min(B * (K + 1), 65535)),
           dim3(256), 0, st, target_logits, V, vp.chunk_len, vp.chunks, B * (K + 1), part);
  launch_k(pdl_default(), verify_final_kernel, dim3(B), dim3(256), 0, st, part, vp.chunks, drafts,
           K, out_tokens, num_accepted, bonus);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// the whole speculative step
// ---------------------------------------------------------------------------
namespace {
struct StepWs {
  size_t ver = 0, inj = 0, prop = 0, total = 0;
};
StepWs step_layout(const dflash_handle* h, int B, int n, int W) {
  StepWs w;
  const int K = h->cfg.block_size - 1;
  size_t off = 0;
  w.ver = off;
  off += align_up(std::max<size_t>(plan_verify(B, K, h->cfg.vocab).bytes, kAlign));
  w.inj = off;
  off += align_up(std::max<size_t>(inject_layout(h, n).total, kAlign));
  w.prop = off;
  off += align_up(propose_layout(h, B, W).total);
  w.total = off;
  return w;
}

// Every host check of the four calls of the step, before any launch.
dflash_status check_step(const dflash_handle* h, const dflash_step_io* io, const void* ws,
                         size_t bytes) {
  if (!h || !io || io->B < 0 || io->n < 0) return DFLASH_ERR_INVALID_ARG;
  if (h->vocab_count != h->cfg.vocab) return DFLASH_ERR_INVALID_ARG;   // a vocabulary shard
  if (h->tp_size > 1) return DFLASH_ERR_INVALID_ARG;                   // a head-parallel shard
  if (io->B == 0) return DFLASH_OK;
  const dflash_config& c = h->cfg;
  const int K = c.block_size - 1;
  if (io->n < io->B || K > 128 || io->max_pages_per_seq < 1 || io->num_pages < 1)
    return DFLASH_ERR_INVALID_ARG;
  if ((K > 0 && !io->prev_drafts) || !io->target_logits || !io->target_positions ||
      !io->last_token_indices || !io->num_draft || !io->aux || !io->block_table ||
      !io->k_cache || !io->v_cache || !io->out_tokens || !io->num_accepted || !io->positions ||
      !io->slot_mapping || !io->seq_lens || !io->bonus || !io->draft_tokens || !ws)
    return DFLASH_ERR_INVALID_ARG;
  if ((io->prev_sampled == nullptr) != (io->prev_num_draft == nullptr))
    return DFLASH_ERR_INVALID_ARG;
  if (io->prev_sampled && io->prev_width < 1) return DFLASH_ERR_INVALID_ARG;
  for (int l = 0; l < c.n_layers; ++l)
    if (!io->k_cache[l] || !io->v_cache[l]) return DFLASH_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return DFLASH_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(io->target_logits) % 16 && c.vocab % 4 == 0)
    return DFLASH_ERR_INVALID_ARG;
  if (static_cast<int64_t>(io->B) * c.block_size > (1 << 24) || io->B > kMaxAttnRequests)
    return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if (bytes < step_layout(h, io->B, io->n, io->max_pages_per_seq).total)
    return DFLASH_ERR_WORKSPACE;
  return DFLASH_OK;
}
}  // namespace

struct dflash_step_graph {
  int device = 0;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

extern "C" {

size_t dflash_spec_step_workspace_bytes(const dflash_handle* h, int B, int n,
                                        int max_pages_per_seq) {
  if (!h || B <= 0 || n < B || max_pages_per_seq <= 0) return 0;
  return step_layout(h, B, n, max_pages_per_seq).total;
}

dflash_status dflash_spec_step(dflash_handle* h, const dflash_step_io* io, void* workspace,
                               size_t workspace_bytes, void* stream) {
  dflash_status s = check_step(h, io, workspace, workspace_bytes);
  if (s != DFLASH_OK || io->B == 0) return s;
  DF_CUDA(use_device(h->device));
  const dflash_config& c = h->cfg;
  const int B = io->B, n = io->n, K = c.block_size - 1, W = io->max_pages_per_seq;
  const StepWs w = step_layout(h, B, n, W);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  // 1. greedy verification of the previous drafts
  s = dflash_verify_greedy(io->prev_drafts, io->target_logits, B, K, c.vocab, io->out_tokens,
                           io->num_accepted, io->bonus, base + w.ver, w.inj - w.ver, stream);
  if (s != DFLASH_OK) return s;
  // 2. corrected positions, context slots, post-verify lengths, bonus tokens
  s = dflash_prepare_proposal_inputs(
      io->target_positions, n, io->last_token_indices, B, io->out_tokens, K + 1, io->num_draft,
      io->prev_sampled, io->prev_width, io->prev_num_draft, io->block_table, W, c.page_size,
      c.vocab, io->positions, io->slot_mapping, io->seq_lens, io->bonus,
      io->device_error ? io->device_error : h->dev_err, stream);
  if (s != DFLASH_OK) return s;
  // 3. context fusion and K/V injection of the target rows
  s = dflash_inject_context(h, io->aux, io->positions, io->slot_mapping, n, io->k_cache,
                            io->v_cache, io->num_pages, base + w.inj, w.prop - w.inj, stream);
  if (s != DFLASH_OK) return s;
  // 4. the next block's drafts
  return dflash_propose(h, io->bonus, io->seq_lens, io->block_table, B, W, io->k_cache,
                        io->v_cache, io->num_pages, io->draft_tokens, io->block_tokens, nullptr,
                        base + w.prop, w.total - w.prop, stream);
}

dflash_status dflash_step_graph_create(dflash_handle* h, const dflash_step_io* io,
                                       void* workspace, size_t workspace_bytes,
                                       dflash_step_graph** out) {
  if (!out) return DFLASH_ERR_INVALID_ARG;
  *out = nullptr;
  dflash_status s = check_step(h, io, workspace, workspace_bytes);
  if (s != DFLASH_OK) return s;
  // per-launch profiling events would be baked into the graph
  if (h->prof_on) return DFLASH_ERR_INVALID_ARG;
  auto* g = new (std::nothrow) dflash_step_graph;
  if (!g) return DFLASH_ERR_CUDA;
  g->device = h->device;
  if (io->B == 0) {  // nothing to run: launches are no-ops
    *out = g;
    return DFLASH_OK;
  }
  if (use_device(h->device) != cudaSuccess) {
    delete g;
    return DFLASH_ERR_CUDA;
  }
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    delete g;
    return DFLASH_ERR_CUDA;
  }
  cudaError_t e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
  if (e == cudaSuccess) {
    s = dflash_spec_step(h, io, workspace, workspace_bytes, cs);
    e = cudaStreamEndCapture(cs, &g->graph);
  }
  cudaStreamDestroy(cs);
  if (s == DFLASH_OK && e == cudaSuccess && g->graph)
    e = cudaGraphInstantiate(&g->exec, g->graph, 0);
  if (s != DFLASH_OK || e != cudaSuccess || !g->exec) {
    cudaGetLastError();
    if (g->graph) cudaGraphDestroy(g->graph);
    delete g;
    return s != DFLASH_OK ? s : DFLASH_ERR_CUDA;
  }
  *out = g;
  return DFLASH_OK;
}

dflash_status dflash_step_graph_launch(dflash_step_graph* g, void* stream) {
  if (!g) return DFLASH_ERR_INVALID_ARG;
  if (!g->exec) return DFLASH_OK;
  DF_CUDA(use_device(g->device));
  DF_CUDA(cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)));
  return DFLASH_OK;
}

void dflash_step_graph_destroy(dflash_step_graph* g) {
  if (!g) return;
  use_device(g->device);
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  delete g;
}

dflash_status dflash_plan_attention_info(int B, int n_kv_heads, int max_pages_per_seq,
                                         int page_size, int block_size, int q_per_kv,
                                         int head_dim, int num_sms, int forced_ring, int flags,
                                         dflash_attention_plan* out) {
  if (!out || B <= 0 || n_kv_heads <= 0 || max_pages_per_seq <= 0 || page_size <= 0 ||
      block_size <= 0 || q_per_kv <= 0 || head_dim <= 0 || num_sms <= 0)
    return DFLASH_ERR_INVALID_ARG;
  const AttnPlan ap = plan_attention(B, n_kv_heads, max_pages_per_seq, page_size, block_size,
                                     q_per_kv, head_dim, num_sms, (flags & 1) != 0, forced_ring,
                                     (flags & 2) != 0, (flags & 4) ? 32 : 64);
  out->tcgen05 = ap.tc ? 1 : 0;
  out->keys_per_tile = ap.tc ? ap.kt : kAttnTileKeys;
  out->ring_depth = ap.tc ? (ap.tc2 || ap.kt == kTcKeysSmall ? ap.st : kTcStages) : 0;
  out->ctas_per_sm =
      ap.tc2 || (ap.tc && ap.kt == kTcKeysSmall && ap.st == kTcStages && !ap.cluster) ? 2 : 1;
  out->transposed_pv = ap.tc2 ? 1 : 0;
  out->chunk_keys = ap.chunk_keys;
  out->max_splits = ap.max_splits;
  out->cluster = ap.cluster ? 1 : 0;
  out->persistent = ap.persist && !ap.cluster && ap.kt == kTcKeysSmall ? 1 : 0;
  return DFLASH_OK;
}

dflash_status dflash_plan_gemm_info(int M, int N, int K, int group, int num_sms,
                                    int pair_split_cap, dflash_gemm_plan* out) {
  if (!out || M <= 0 || N <= 0 || K <= 0 || K % kGemmBK || num_sms < 2 || pair_split_cap < 0 ||
      (group != 32 && group != 64 && group != 128))
    return DFLASH_ERR_INVALID_ARG;
  std::array<int, 9> cap{};
  for (int S = 2; S <= 8; ++S) cap[S] = num_sms / S;
  GemmPlan pl = plan_gemm(M, N, K, group, num_sms);
  if (gemm_staged(pl.a_rows) && pl.tiles <= num_sms)
    pl = plan_gemm(M, N, K, group, num_sms, 0, 0, cap.data());
  const PairChoice pc = gemm_pair_choice(pl, M, N, group, num_sms, pair_split_cap);
  *out = dflash_gemm_plan{};
  if (pc.bn) {
    out->pair = 1;
    out->tile_m = 2 * kPairRows;
    out->tile_n = pc.bn;
    out->k_splits = pc.ks;
    out->tiles = cdiv(M, 2 * kPairRows) * cdiv(N, pc.bn);
    out->grid = pc.ks == 2 ? 4 * out->tiles : 2 * std::min(out->tiles, num_sms / 2);
  } else {
    out->tile_m = kGemmBM;
    out->tile_n = pl.BN;
    out->k_splits = pl.cluster_s;
    out->stream_k = pl.stream_k;
    out->staged = gemm_staged(pl.a_rows) ? 1 : 0;
    out->tiles = pl.tiles;
    out->grid = pl.grid;
  }
  return DFLASH_OK;
}

size_t dflash_linear_workspace_bytes(const dflash_handle* h, int M, int N, int K) {
  if (!h || M <= 0 || N <= 0 || K <= 0) return 0;
  return align_up(std::max<size_t>(plan_gemm(M, N, K, 32, h->num_sms).partial_bytes, kAlign));
}

dflash_status dflash_linear(dflash_handle* h, const void* A, const void* W, int M, int N, int K,
                            float* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!h || M < 0 || N <= 0 || K <= 0) return DFLASH_ERR_INVALID_ARG;
  if (M == 0) return DFLASH_OK;
  if (!A || !W || !out || !workspace) return DFLASH_ERR_INVALID_ARG;
  if (K % 64 || N % 32) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if (reinterpret_cast<uintptr_t>(A) % 16 || reinterpret_cast<uintptr_t>(W) % 16 ||
      reinterpret_cast<uintptr_t>(out) % 16)
    return DFLASH_ERR_INVALID_ARG;
  const size_t need = dflash_linear_workspace_bytes(h, M, N, K);
  if (workspace_bytes < need) return DFLASH_ERR_WORKSPACE;
  DF_CUDA(use_device(h->device));
  EpiStoreF32 e{out, N};
  return run_gemm(h, DFLASH_KERNEL_LINEAR, false, false, A, M, K, W, N, e,
                  static_cast<float*>(workspace), workspace_bytes,
                  static_cast<cudaStream_t>(stream));
}

dflash_status dflash_linear_ex(dflash_handle* h, const void* A, const void* W, int M, int N,
                               int K, float* out, int block_n, int splits, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (!h || M < 0 || N <= 0 || K <= 0 || block_n < 0 || splits < 0)
    return DFLASH_ERR_INVALID_ARG;
  if (M == 0) return DFLASH_OK;
  if (!A || !W || !out || !workspace) return DFLASH_ERR_INVALID_ARG;
  if (K % 64 || N % 32) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if (reinterpret_cast<uintptr_t>(A) % 16 || reinterpret_cast<uintptr_t>(W) % 16 ||
      reinterpret_cast<uintptr_t>(out) % 16)
    return DFLASH_ERR_INVALID_ARG;
  DF_CUDA(use_device(h->device));
  EpiStoreF32 e{out, N};
  return run_gemm(h, DFLASH_KERNEL_LINEAR, false, false, A, M, K, W, N, e,
                  static_cast<float*>(workspace), workspace_bytes,
                  static_cast<cudaStream_t>(stream), block_n, splits);
}

size_t dflash_attention_workspace_bytes(const dflash_handle* h, int B, int max_pages_per_seq) {
  if (!h || B <= 0 || max_pages_per_seq <= 0) return 0;
  const dflash_config& c = h->cfg;
  const AttnPlan ap = plan_attention(B, c.n_kv_heads, max_pages_per_seq, c.page_size,
                                     c.block_size, c.n_q_heads / c.n_kv_heads, c.head_dim,
                                     h->num_sms, h->attn_cluster, h->attn_ring,
                                     h->attn_persist, h->attn_tile);
  return align_up(ap.part_o_bytes) + align_up(ap.part_ml_bytes) + kAlign;
}

dflash_status dflash_block_attention(dflash_handle* h, const void* q, const int32_t* seq_lens,
                                     const int32_t* block_table, int B, int max_pages_per_seq,
                                     const void* k_cache, const void* v_cache, int num_pages,
                                     void* o, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!h || B < 0) return DFLASH_ERR_INVALID_ARG;
  if (B == 0) return DFLASH_OK;
  if (!q || !seq_lens || !block_table || max_pages_per_seq <= 0 || !k_cache || !v_cache ||
      num_pages <= 0 || !o || !workspace)
    return DFLASH_ERR_INVALID_ARG;
  const dflash_config& c = h->cfg;
  if (B > kMaxAttnRequests) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < dflash_attention_workspace_bytes(h, B, max_pages_per_seq))
    return DFLASH_ERR_WORKSPACE;
  DF_CUDA(use_device(h->device));
  const AttnPlan ap = plan_attention(B, c.n_kv_heads, max_pages_per_seq, c.page_size,
                                     c.block_size, c.n_q_heads / c.n_kv_heads, c.head_dim,
                                     h->num_sms, h->attn_cluster, h->attn_ring,
                                     h->attn_persist, h->attn_tile);
  AttnParams prm;
  prm.q = static_cast<const bf16*>(q);
  prm.o = static_cast<f16*>(o);
  prm.part_o = static_cast<float*>(workspace);
  prm.part_ml = at<float>(workspace, align_up(ap.part_o_bytes));
  prm.seq_lens = seq_lens;
  prm.block_table = block_table;
  prm.B = B;
  prm.W = max_pages_per_seq;
  prm.bs = c.block_size;
  prm.Hq = c.n_q_heads;
  prm.Hkv = c.n_kv_heads;
  prm.G = c.n_q_heads / c.n_kv_heads;
  prm.R = ap.R;
  prm.num_pages = num_pages;
  prm.chunk_keys = ap.chunk_keys;
  prm.max_splits = ap.max_splits;
  prm.scale_log2 =
      static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.head_dim)));
  prm.err = h->dev_err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return c.head_dim == 128 ? run_attention<128>(h, ap, prm, k_cache, v_cache, num_pages, st)
                           : run_attention<64>(h, ap, prm, k_cache, v_cache, num_pages, st);
}

unsigned long long dflash_launch_count(const dflash_handle* h) { return h ? h->launches : 0; }

const char* dflash_kernel_name(int kind) {
  switch (kind) {
    case DFLASH_KERNEL_EMBED_NORM: return "embed_norm";
    case DFLASH_KERNEL_GEMM_QKV: return "gemm_qkv";
    case DFLASH_KERNEL_ATTENTION: return "attention";
    case DFLASH_KERNEL_ATTN_COMBINE: return "attn_combine";
    case DFLASH_KERNEL_GEMM_O: return "gemm_o";
    case DFLASH_KERNEL_RMSNORM: return "rmsnorm";
    case DFLASH_KERNEL_GEMM_GATE_UP: return "gemm_gate_up";
    case DFLASH_KERNEL_GEMM_DOWN: return "gemm_down";
    case DFLASH_KERNEL_GEMM_LM_HEAD: return "gemm_lm_head";
    case DFLASH_KERNEL_ARGMAX_FINALIZE: return "argmax_finalize";
    case DFLASH_KERNEL_GEMM_FC: return "gemm_fc";
    case DFLASH_KERNEL_GEMM_KV_INJECT: return "gemm_kv_inject";
    case DFLASH_KERNEL_LINEAR: return "linear";
    case DFLASH_KERNEL_GEMM_MLP: return "gemm_mlp";
  }
  return nullptr;
}

dflash_status dflash_profile_enable(dflash_handle* h, int max_launches) {
  if (!h || max_launches <= 0) return DFLASH_ERR_INVALID_ARG;
  DF_CUDA(use_device(h->device));
  for (auto e : h->prof_events) cudaEventDestroy(e);
  h->prof_events.clear();
  h->prof_kind.clear();
  h->prof_next = 0;
  for (int i = 0; i < 2 * max_launches; ++i) {
    cudaEvent_t e;
    DF_CUDA(cudaEventCreate(&e));
    h->prof_events.push_back(e);
  }
  h->prof_on = true;
  return DFLASH_OK;
}

dflash_status dflash_profile_read(dflash_handle* h, int n_kinds, int* launches,
                                  double* total_ms) {
  if (!h || n_kinds < 0 || (n_kinds && (!launches || !total_ms))) return DFLASH_ERR_INVALID_ARG;
  DF_CUDA(use_device(h->device));
  for (int k = 0; k < n_kinds; ++k) {
    launches[k] = 0;
    total_ms[k] = 0.0;
  }
  DF_CUDA(cudaDeviceSynchronize());
  for (size_t i = 0; i < h->prof_kind.size(); ++i) {
    float ms = 0.f;
    DF_CUDA(cudaEventElapsedTime(&ms, h->prof_events[2 * i], h->prof_events[2 * i + 1]));
    const int k = h->prof_kind[i];
    if (k >= 0 && k < n_kinds) {
      launches[k] += 1;
      total_ms[k] += ms;
    }
  }
  h->prof_kind.clear();
  h->prof_next = 0;
  return DFLASH_OK;
}

dflash_status dflash_profile_disable(dflash_handle* h) {
  if (!h) return DFLASH_ERR_INVALID_ARG;
  h->prof_on = false;
  h->prof_kind.clear();
  h->prof_next = 0;
  return DFLASH_OK;
}

dflash_status dflash_check_device_errors(dflash_handle* h, unsigned* bits) {
  if (bits) *bits = 0;
  if (!h) return DFLASH_ERR_INVALID_ARG;
  DF_CUDA(use_device(h->device));
  DF_CUDA(cudaDeviceSynchronize());
  unsigned v = 0;
  DF_CUDA(cudaMemcpy(&v, h->dev_err, sizeof(unsigned), cudaMemcpyDeviceToHost));
  DF_CUDA(cudaMemset(h->dev_err, 0, sizeof(unsigned)));
  if (v & DFLASH_DEVERR_TIMEOUT) {
    // a kernel that gave up may have left split-K arrival counters behind
    DF_CUDA(cudaMemset(h->counters, 0, kCounterSlots * sizeof(unsigned)));
  }
  if (bits) *bits = v;
  if (v == 0) return DFLASH_OK;
  return (v & DFLASH_DEVERR_TIMEOUT) ? DFLASH_ERR_DEVICE_TIMEOUT : DFLASH_ERR_DEVICE_BOUNDS;
}

}  // extern "C"

// ===========================================================================
// Greedy verification that allocates nothing
// ===========================================================================
// Some callers cannot hand this library a workspace: an embedding runtime that
// reserved all device memory for its own pool at start-up (a cudaMalloc from
// here could fail or fragment that pool), a plugin that only ever receives its
// input and output buffers from the host framework and owns no allocator, or
// a latency-critical decode loop where cudaMalloc / cudaFree would synchronize
// the device.  dflash_verify_greedy_noalloc serves them with scratch that the
// library already owns: a fixed array in this module's device memory.
namespace {

// One 64-bit partial argmax key per (request, target row, vocabulary chunk).
// Every device that loads this library holds these 64 KiB until the process
// exits.  Calls share the array; it keeps whatever the last call wrote.
constexpr int kNoAllocVerifyKeys = DFLASH_VERIFY_NOALLOC_MAX_PARTIALS;
static __device__ __align__(256) unsigned long long g_verify_scratch[kNoAllocVerifyKeys];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_verify_scratch_mu;
struct ScratchAddr {
  unsigned long long ctx_id = 0;       // context the address belongs to (0: none yet)
  unsigned long long* ptr = nullptr;
};
ScratchAddr g_verify_scratch_dev[kNoAllocMaxDevices];

// Unique id of the calling thread's current CUDA context (driver entry points
// looked up once; no link-time libcuda dependency).  0 if unavailable.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// On the host, g_verify_scratch only names the symbol; a kernel given that
// name would read the wrong memory.  The array's device address is looked up
// per device (with that device current) and cached together with the id of
// the context it belongs to: after a device reset the runtime builds a new
// context, the id changes, and the address is looked up again.
dflash_status verify_scratch_on_current_device(unsigned long long** out) {
  int dev = -1;
  DF_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  const unsigned long long ctx = current_context_id();   // 0 before the context exists
  std::lock_guard<std::mutex> lk(g_verify_scratch_mu);
  ScratchAddr& a = g_verify_scratch_dev[dev];
  if (!a.ptr || ctx == 0 || a.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_verify_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return DFLASH_ERR_CUDA;
    }
    a.ptr = static_cast<unsigned long long*>(p);
    a.ctx_id = current_context_id();
  }
  *out = a.ptr;
  return DFLASH_OK;
}

}  // namespace

extern "C" dflash_status dflash_verify_greedy_noalloc(const int32_t* drafts,
                                                      const float* target_logits, int B, int K,
                                                      int V, int32_t* out_tokens,
                                                      int32_t* num_accepted, int32_t* bonus,
                                                      void* stream) {
  if (B < 0 || K < 0 || V <= 0 || K > 128) return DFLASH_ERR_INVALID_ARG;
  if (B == 0) return DFLASH_OK;
  if (static_cast<int64_t>(B) * (K + 1) > (1 << 30)) return DFLASH_ERR_UNSUPPORTED_SHAPE;
  if ((K > 0 && !drafts) || !target_logits || !out_tokens || !num_accepted || !bonus)
    return DFLASH_ERR_INVALID_ARG;
  const VerifyPlan vp = plan_verify(B, K, V);
  if (static_cast<int64_t>(B) * (K + 1) * vp.chunks > kNoAllocVerifyKeys)
    return DFLASH_ERR_WORKSPACE;  // needs more partial keys than the fixed scratch holds
  if (reinterpret_cast<uintptr_t>(target_logits) % 16 && V % 4 == 0)
    return DFLASH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dflash_status s = set_device_for(st, out_tokens);
  if (s != DFLASH_OK) return s;
  unsigned long long* part = nullptr;
  s = verify_scratch_on_current_device(&part);
  if (s != DFLASH_OK) return s;
  // Nothing in the scratch has to start at zero: the second kernel reads only
  // the keys the first one writes in this same call.
  launch_k(pdl_default(), verify_partial_kernel, dim3(vp.chunks, std::min(B * (K + 1), 65535)),
           dim3(256), 0, st, target_logits, V, vp.chunk_len, vp.chunks, B * (K + 1), part);
  launch_k(pdl_default(), verify_final_kernel, dim3(B), dim3(256), 0, st, part, vp.chunks, drafts,
           K, out_tokens, num_accepted, bonus);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

// ===========================================================================
// A small causal target model on the device (the on-device lossless loop)
// ===========================================================================
struct dflash_target {
  dflash_target_config cfg{};
  std::vector<int> capture;          // pre-layer capture indices, request order
  int device = 0;
  const float *embed = nullptr, *final_norm_w = nullptr, *lm_head = nullptr;
  std::vector<const float*> in_norm_w, post_norm_w, q_norm_w, k_norm_w, wo, wdown;
  std::vector<float*> wqkv, wgu;     // owned: [Wq; Wk; Wv] and [Wgate; Wup] per layer
  float *kcache = nullptr, *vcache = nullptr;   // owned: [L][max_len][Hkv][D] each
  unsigned* dev_err = nullptr;
};

namespace {
struct TargetWs {
  size_t x, y, qkv, q, o, gu, hm, total;
};
TargetWs target_layout(const dflash_target_config& c, int n) {
  TargetWs w{};
  size_t off = 0;
  auto take = [&off](size_t floats) {
    const size_t at = off;
    off += align_up(floats * 4);
    return at;
  };
  const size_t rows = static_cast<size_t>(n);
  w.x = take(rows * c.hidden);
  w.y = take(rows * c.hidden);
  w.qkv = take(rows * (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim);
  w.q = take(rows * c.n_q_heads * c.head_dim);
  w.o = take(rows * c.n_q_heads * c.head_dim);
  w.gu = take(rows * 2 * c.intermediate);
  w.hm = take(rows * c.intermediate);
  w.total = off;
  return w;
}
void free_target(dflash_target* t) {
  if (!t) return;
  for (auto p : t->wqkv) cudaFree(p);
  for (auto p : t->wgu) cudaFree(p);
  cudaFree(t->kcache);
  cudaFree(t->vcache);
  cudaFree(t->dev_err);
  delete t;
}
}  // namespace

extern "C" {

dflash_status dflash_aux_capture_layers(const int* target_layer_ids, int n, int target_n_layers,
                                        int* capture_layers) {
  if (n < 0 || target_n_layers <= 0 || (n > 0 && (!target_layer_ids || !capture_layers)))
    return DFLASH_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    // the state after layer i is the state before layer i + 1
    const int j = target_layer_ids[i] + 1;
    if (target_layer_ids[i] < 0 || j > target_n_layers) return DFLASH_ERR_INVALID_ARG;
    capture_layers[i] = j;
  }
  return DFLASH_OK;
}

dflash_status dflash_target_create(const dflash_target_config* cfg, const dflash_target_weights* w,
                                   int device, dflash_target** out) {
  if (!out) return DFLASH_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || !w) return DFLASH_ERR_INVALID_ARG;
  const dflash_target_config& c = *cfg;
  if (c.hidden <= 0 || c.n_layers <= 0 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 ||
      c.head_dim <= 0 || c.intermediate <= 0 || c.vocab <= 0 || c.max_len <= 0 ||
      c.n_capture < 0 || (c.n_capture > 0 && !c.capture_layers) || !(c.rms_eps >= 0.f) ||
      !(c.rope_theta > 0.f))
    return DFLASH_ERR_INVALID_ARG;
  if (c.head_dim % 32 || c.head_dim > 128 || c.n_q_heads % c.n_kv_heads || c.head_dim % 2)
    return DFLASH_ERR_UNSUPPORTED_SHAPE;
  for (int i = 0; i < c.n_capture; ++i)
    if (c.capture_layers[i] < 0 || c.capture_layers[i] > c.n_layers) return DFLASH_ERR_INVALID_ARG;
  const int L = c.n_layers;
  if (!w->embed || !w->final_norm_w || !w->lm_head || !w->in_norm_w || !w->post_norm_w ||
      !w->wq || !w->wk || !w->wv || !w->wo || !w->q_norm_w || !w->k_norm_w || !w->w_gate ||
      !w->w_up || !w->w_down)
    return DFLASH_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l)
    if (!w->in_norm_w[l] || !w->post_norm_w[l] || !w->wq[l] || !w->wk[l] || !w->wv[l] ||
        !w->wo[l] || !w->q_norm_w[l] || !w->k_norm_w[l] || !w->w_gate[l] || !w->w_up[l] ||
        !w->w_down[l])
      return DFLASH_ERR_INVALID_ARG;
  dflash_target* t = new (std::nothrow) dflash_target();
  if (!t) return DFLASH_ERR_CUDA;
  t->cfg = c;
  t->capture.assign(c.capture_layers, c.capture_layers + c.n_capture);
  t->cfg.capture_layers = t->capture.empty() ? nullptr : t->capture.data();
  t->device = device;
  auto fail = [t](dflash_status s) {
    free_target(t);
    return s;
  };
  if (cudaSetDevice(device) != cudaSuccess) return fail(DFLASH_ERR_CUDA);
  const int H = c.hidden, D = c.head_dim, Hq = c.n_q_heads, Hkv = c.n_kv_heads, I = c.intermediate;
  t->embed = w->embed;
  t->final_norm_w = w->final_norm_w;
  t->lm_head = w->lm_head;
  const size_t row = static_cast<size_t>(H) * 4;
  for (int l = 0; l < L; ++l) {
    t->in_norm_w.push_back(w->in_norm_w[l]);
    t->post_norm_w.push_back(w->post_norm_w[l]);
    t->q_norm_w.push_back(w->q_norm_w[l]);
    t->k_norm_w.push_back(w->k_norm_w[l]);
    t->wo.push_back(w->wo[l]);
    t->wdown.push_back(w->w_down[l]);
    float* p = nullptr;
    if (cudaMalloc(&p, static_cast<size_t>(Hq + 2 * Hkv) * D * row) != cudaSuccess)
      return fail(DFLASH_ERR_CUDA);
    t->wqkv.push_back(p);
    if (cudaMemcpy(p, w->wq[l], static_cast<size_t>(Hq) * D * row, cudaMemcpyDeviceToDevice) !=
            cudaSuccess ||
        cudaMemcpy(p + static_cast<size_t>(Hq) * D * H, w->wk[l], static_cast<size_t>(Hkv) * D * row,
                   cudaMemcpyDeviceToDevice) != cudaSuccess ||
        cudaMemcpy(p + static_cast<size_t>(Hq + Hkv) * D * H, w->wv[l],
                   static_cast<size_t>(Hkv) * D * row, cudaMemcpyDeviceToDevice) != cudaSuccess)
      return fail(DFLASH_ERR_CUDA);
    if (cudaMalloc(&p, static_cast<size_t>(2 * I) * row) != cudaSuccess) return fail(DFLASH_ERR_CUDA);
    t->wgu.push_back(p);
    if (cudaMemcpy(p, w->w_gate[l], static_cast<size_t>(I) * row, cudaMemcpyDeviceToDevice) !=
            cudaSuccess ||
        cudaMemcpy(p + static_cast<size_t>(I) * H, w->w_up[l], static_cast<size_t>(I) * row,
                   cudaMemcpyDeviceToDevice) != cudaSuccess)
      return fail(DFLASH_ERR_CUDA);
  }
  const size_t cache = static_cast<size_t>(L) * c.max_len * Hkv * D * 4;
  if (cudaMalloc(&t->kcache, cache) != cudaSuccess || cudaMalloc(&t->vcache, cache) != cudaSuccess ||
      cudaMemset(t->kcache, 0, cache) != cudaSuccess || cudaMemset(t->vcache, 0, cache) != cudaSuccess ||
      cudaMalloc(&t->dev_err, sizeof(unsigned)) != cudaSuccess ||
      cudaMemset(t->dev_err, 0, sizeof(unsigned)) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess)
    return fail(DFLASH_ERR_CUDA);
  *out = t;
  return DFLASH_OK;
}

void dflash_target_destroy(dflash_target* t) {
  if (!t) return;
  cudaSetDevice(t->device);
  free_target(t);
}

size_t dflash_target_workspace_bytes(const dflash_target* t, int n) {
  if (!t || n <= 0) return 0;
  return target_layout(t->cfg, n).total;
}

dflash_status dflash_target_forward(dflash_target* t, const int32_t* tokens, int n, int start_pos,
                                    float* logits, void* aux, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!t || n < 0) return DFLASH_ERR_INVALID_ARG;
  if (n == 0) return DFLASH_OK;
  const dflash_target_config& c = t->cfg;
  if (!tokens || !logits || !workspace || (c.n_capture > 0 && !aux)) return DFLASH_ERR_INVALID_ARG;
  if (start_pos < 0 || static_cast<int64_t>(start_pos) + n > c.max_len)
    return DFLASH_ERR_INVALID_ARG;
  const TargetWs ws = target_layout(c, n);
  if (workspace_bytes < ws.total) return DFLASH_ERR_WORKSPACE;
  DF_CUDA(use_device(t->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = c.hidden, D = c.head_dim, Hq = c.n_q_heads, Hkv = c.n_kv_heads,
            I = c.intermediate, V = c.vocab, L = c.n_layers;
  float* x = at<float>(workspace, ws.x);
  float* y = at<float>(workspace, ws.y);
  float* qkv = at<float>(workspace, ws.qkv);
  float* q = at<float>(workspace, ws.q);
  float* o = at<float>(workspace, ws.o);
  float* gu = at<float>(workspace, ws.gu);
  float* hm = at<float>(workspace, ws.hm);
  bf16* ax = static_cast<bf16*>(aux);
  TargetDims d{H, Hq, Hkv, D, I, V, c.max_len, c.rms_eps, c.rope_theta};
  auto linear = [&](const float* a, const float* W, int N, int K, float* dst, int acc) {
    target_linear_kernel<<<dim3(cdiv(N, 8), n), 256, 0, st>>>(a, W, N, K, dst, acc);
  };
  auto capture = [&](int layer) {
    for (int k = 0; k < c.n_capture; ++k)
      if (t->capture[k] == layer)
        target_capture_kernel<<<cdiv(n * H, 256), 256, 0, st>>>(x, n, H, c.n_capture, k, ax);
  };
  target_embed_kernel<<<n, 256, 0, st>>>(tokens, t->embed, H, V, x, t->dev_err);
  const size_t layer_cache = static_cast<size_t>(c.max_len) * Hkv * D;
  for (int l = 0; l < L; ++l) {
    capture(l);
    target_rmsnorm_kernel<<<n, 256, 0, st>>>(x, t->in_norm_w[l], H, c.rms_eps, y);
    linear(y, t->wqkv[l], (Hq + 2 * Hkv) * D, H, qkv, 0);
    target_qkv_kernel<<<cdiv(n * (Hq + Hkv), 8), 256, 0, st>>>(
        qkv, n, start_pos, d, t->q_norm_w[l], t->k_norm_w[l], q, t->kcache + l * layer_cache,
        t->vcache + l * layer_cache, t->dev_err);
    target_attention_kernel<<<cdiv(n * Hq, 8), 256, 0, st>>>(
        q, n, start_pos, d, t->kcache + l * layer_cache, t->vcache + l * layer_cache, o);
    linear(o, t->wo[l], H, Hq * D, x, 1);
    target_rmsnorm_kernel<<<n, 256, 0, st>>>(x, t->post_norm_w[l], H, c.rms_eps, y);
    linear(y, t->wgu[l], 2 * I, H, gu, 0);
    target_swiglu_kernel<<<cdiv(n * I, 256), 256, 0, st>>>(gu, I, n, hm);
    linear(hm, t->wdown[l], H, I, x, 1);
  }
  capture(L);
  target_rmsnorm_kernel<<<n, 256, 0, st>>>(x, t->final_norm_w, H, c.rms_eps, y);
  linear(y, t->lm_head, V, H, logits, 0);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

dflash_status dflash_target_check_device_errors(dflash_target* t, unsigned* bits) {
  if (bits) *bits = 0;
  if (!t) return DFLASH_ERR_INVALID_ARG;
  DF_CUDA(use_device(t->device));
  DF_CUDA(cudaDeviceSynchronize());
  unsigned v = 0;
  DF_CUDA(cudaMemcpy(&v, t->dev_err, sizeof(unsigned), cudaMemcpyDeviceToHost));
  DF_CUDA(cudaMemset(t->dev_err, 0, sizeof(unsigned)));
  if (bits) *bits = v;
  return v ? DFLASH_ERR_DEVICE_BOUNDS : DFLASH_OK;
}

}  // extern "C"

