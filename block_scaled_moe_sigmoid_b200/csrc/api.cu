// C ABI of the MoE layer (include/moe.h): argument checks, workspace carving, TMA
// descriptor encoding and the launch sequence.  All arithmetic runs in the kernels of
// kernels.cuh and gemm.cuh.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <atomic>
#include <vector>

#include "../../include/moe.h"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "kernels.cuh"
#include "router.cuh"

using namespace moe;

namespace {

// Routed grouped-GEMM tile configurations (token rows per tile), chosen per call:
//   176 (default when T*k > 8*E): swap-AB, 256 weight rows on the MMA's M side and up to
//   176 token rows on N, 4-stage smem ring (56 KB stages).  Kimi-K3 prefill (T=8192) gives
//   an expert ~146 +- 12 rows, so 176 keeps all but a handful of experts in one tile (with
//   160, one in eight was split in two half-full tiles, each costing as much tensor time as
//   a full one);
//   32 (default when T*k <= 8*E, decode): swap-AB with up to 32 token rows, 6 stages
//   (36 KB of tiles + 1.5 KB of scale atoms each, the whole 227 KB): with a few tokens per
//   expert the weight stream is the whole cost, and each stage keeps another 16 KB weight
//   tile per SM in flight (5 -> 4 stages measured 6% slower);
//   128 (selectable): the WN orientation (gemm.cuh), token rows on M and 256 weight rows on
//   N, 4 stages (50 KB).  Half the MMAs of swap-AB per weight byte, bit-identical results,
//   but measured slower at every token count, so never the default.
constexpr int kBN = 176, kStages = 4;
constexpr int kBNMid = 128, kStagesMid = 4;
constexpr int kBNPair = 160, kStagesPair = 5;   // CTA-pair configuration (gemm_pair.cuh)
constexpr int kBNSmall = 32, kStagesSmall = 6;
constexpr int kBNMin = kBNSmall;   // workspace sizing: the most tiles either configuration forms
constexpr int kPermThreads = 256;
constexpr int kRouterBN = 128;  // tokens per router tile
constexpr int kRouterStages = 3;
constexpr int kRouterMaxCtas = 256;   // bound on split router tiles (sizes the partials)
constexpr int kMaxExperts = 4096;
constexpr int kSplitMaxCtas = 256;    // bound on split-K dense GEMM tiles (sizes their partials)

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
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

// 2-D tiled map, 128-byte swizzle.  inner = elements per row, rows = row count,
// row_bytes = stride between rows.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
              uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return f(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Token-row maps for the grouped GEMM: box heights 16, 32, ... rows (one per MMA N).
bool make_bmaps(BMaps* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                uint64_t row_bytes, uint32_t box_inner) {
  for (int i = 0; i < MAX_BOX; ++i)
    if (!make_map(&m->box[i], dt, base, inner, rows, row_bytes, box_inner, (uint32_t)(BOX_ROWS * (i + 1))))
      return false;
  return true;
}

inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
inline size_t up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline cudaStream_t S(void* s) { return (cudaStream_t)s; }

}  // namespace

// Optional per-stage timing: CUDA events recorded on the caller's stream around each
// stage of moe_route / moe_forward, summed by moe_plan_stage_ms.
struct StageProfiler {
  bool on = false;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  struct Rec { int stage; cudaEvent_t a, b; };
  std::vector<Rec> recs;
  int open_stage = -1;
  cudaEvent_t open_ev = nullptr;
  cudaEvent_t next() {
    if (used == pool.size()) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
      pool.push_back(e);
    }
    return pool[used++];
  }
  void begin(int stage, cudaStream_t s) {
    if (!on) return;
    open_stage = stage;
    open_ev = next();
    if (open_ev) cudaEventRecord(open_ev, s);
  }
  void end(cudaStream_t s) {
    if (!on || !open_ev) return;
    cudaEvent_t b = next();
    if (!b) return;
    cudaEventRecord(b, s);
    recs.push_back({open_stage, open_ev, b});
    open_ev = nullptr;
  }
  ~StageProfiler() {
    for (auto e : pool) cudaEventDestroy(e);
  }
};

struct moe_plan_s {
  StageProfiler prof;
  int T_max, d, E, k, I, Is;
  int num_sms = 148;
  int last_T = 0;
  int pf_dist = 0, pf_b = 0;  // GEMM L2 prefetch (moe_plan_set_option)
  int act = MOE_ACT_SILU_GLU;
  int bias_mode = MOE_BIAS_LOGIT;
  int flags = 0;
  const void* planes_of = nullptr;   // W_r the router planes were last split from
  int tile_n_opt = 0;         // MOE_OPT_TILE_N: 0 = automatic, else 32, 128, 160 or 176
  int last_bn = 0;            // token rows per tile in the last moe_forward
  int last_ksplit = 0;        // router K splits in the last moe_route
  int last_shared_split = 0;     // shared-expert gate/up K splits in the last moe_forward
  int last_shared_split_dn = 0;  // shared-expert down K splits in the last moe_forward
  size_t zpart_floats = 0;    // capacity of the router partials
  // token rows per routed GEMM tile for a call with T tokens
  int tile_rows(int T) const {
    if (tile_n_opt) return tile_n_opt;
    return (long long)T * k <= 8ll * E ? kBNSmall : kBN;   // <= 8 tokens per expert on average
  }
  // token rows per tile of the dense (shared-expert, latent projection) GEMMs
  int dense_rows(int T) const { return (long long)T * k <= 8ll * E ? kBNSmall : kBN; }
  char* ws = nullptr;
  size_t ws_bytes = 0;
  // workspace carve (byte offsets)
  size_t o_status, o_chunk, o_counts, o_offsets, o_tiles, o_perm, o_inv, o_logits, o_zpart,
      o_planes, o_xq, o_xs_tok, o_xs, o_hq, o_hs, o_O, o_hsh, o_ys, o_spart, o_theta, o_qbuf, o_xl, o_xn, o_yl,
      o_yr, total;
  int dl = 0;              // latent option: expert width (0 = off)
  float eps_lat = 1e-5f;
  int tokens_per_chunk() const { return kPermThreads; }
  int nchunks(int T) const { return (T + kPermThreads - 1) / kPermThreads; }
  template <class P>
  P* at(size_t off) const { return (P*)(ws + off); }
};

static void carve(moe_plan_s* p) {
  const size_t A = (size_t)p->T_max * p->k;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = up(o + bytes, 1024); return r; };
  p->o_status = take(256);
  p->o_chunk = take((size_t)p->nchunks(p->T_max) * p->E * 4);
  p->o_counts = take((size_t)p->E * 4);
  p->o_offsets = take((size_t)(p->E + 1) * 4);
  p->o_tiles = take((size_t)(p->E + 1) * 4);
  p->o_perm = take(A * 4);
  p->o_inv = take(A * 4);
  p->o_logits = take((size_t)p->T_max * p->E * 4);
  // K-split router partials [ksplit][T][E]: few tokens split up to kRouterMaxCtas tiles
  // (ksplit * T * E <= kRouterMaxCtas * 128 * 128), many tokens split at most 3 ways
  p->zpart_floats = std::max((size_t)kRouterMaxCtas * kRouterBN * 128, (size_t)3 * p->T_max * p->E);
  p->o_zpart = take(p->zpart_floats * 4);
  p->o_planes = take((size_t)p->E * 3 * p->d * 2);
  p->o_xq = take(A * p->d);
  // token-side scale blocks, tile-major: at most A / bn + E group-tiles
  const size_t max_tiles = A / kBNMin + p->E + 1;
  p->o_xs_tok = take((size_t)p->T_max * (p->d / 32));
  p->o_xs = take(max_tiles * (p->d / 128) * SF_TILE_BYTES);
  p->o_hq = take(A * p->I);
  p->o_hs = take(max_tiles * (p->I / 128) * SF_TILE_BYTES);
  p->o_O = take(A * p->d * 2);
  p->o_hsh = take((size_t)p->T_max * (p->Is ? p->Is : 1) * 2);
  p->o_ys = take((size_t)p->T_max * p->d * 4);
  // split-K partials of the dense shared-expert GEMMs: ksplit * tiles <= kSplitMaxCtas, so
  // ksplit * T * M <= kSplitMaxCtas * kBN * 256 floats
  p->o_spart = take((size_t)kSplitMaxCtas * kBN * 256 * 4);
  // Quantile Balancing inputs: each token's k-th largest key, and the quantiles handed to
  // a bias rule
  p->o_theta = take((size_t)std::max(p->T_max, 1) * 4);
  p->o_qbuf = take((size_t)kMaxQuantLevels * p->E * 4);
  if (p->dl > 0) {   // latent option: x_l fp32, x_n bf16, y_l bf16 [T][dl], y_r fp32 [T][d]
    p->o_xl = take((size_t)p->T_max * p->dl * 4);
    p->o_xn = take((size_t)p->T_max * p->dl * 2);
    p->o_yl = take((size_t)p->T_max * p->dl * 2);
    p->o_yr = take((size_t)p->T_max * p->d * 4);
  } else {
    p->o_xl = p->o_xn = p->o_yl = p->o_yr = 0;
  }
  p->total = o;
}

// Launch with programmatic stream serialization: the kernel may start its prologue while
// the previous kernel on the stream finishes; every kernel of the layer waits for that one
// (griddep_wait) before its first global memory access.
template <typename... KArgs, typename... Args>
static cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// cudaFuncSetAttribute acts on the current device: remember, per kernel and per device
// (bit d of `done`), which ones already had their dynamic shared-memory limit raised.
template <class K>
static cudaError_t ensure_smem_attr(K kern, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int KIND, int EPI, int BN, int STAGES, bool WN = false>
static cudaError_t launch_gemm_cfg(const GemmArgs& a, const CUtensorMap& tA, const BMaps& tB, int grid,
                                   cudaStream_t s) {
  using Cfg = GemmCfg<KIND, BN, STAGES, WN>;
  auto kern = gemm_kernel<KIND, EPI, BN, STAGES, WN>;
  static std::atomic<uint64_t> attr_done{0};
  const cudaError_t e = ensure_smem_attr(kern, Cfg::SMEM_BYTES, attr_done);
  if (e != cudaSuccess) return e;
  if (grid <= 0) return cudaSuccess;
  return launch_k(kern, grid, Cfg::NUM_THREADS, Cfg::SMEM_BYTES, s, a, tA, tB);
}

// The CTA-pair routed GEMM: clusters of two CTAs (grid rounded down to an even number of
// SMs), programmatic stream serialization as for the other launches.
template <int EPI>
static cudaError_t launch_gemm_pair(const GemmArgs& a, const CUtensorMap& tA, const BMaps& tB, int grid,
                                   cudaStream_t s) {
  using Cfg = PairCfg<kBNPair, kStagesPair>;
  auto kern = gemm_pair_kernel<EPI, kBNPair, kStagesPair>;
  static std::atomic<uint64_t> attr_done{0};
  const cudaError_t e = ensure_smem_attr(kern, Cfg::SMEM_BYTES, attr_done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(Cfg::NUM_THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // The kernel is persistent: every pair must be resident at once, and pairs of SMs that
  // each hold a 222 KB CTA must share a GPC, so fewer pairs than SMs / 2 may fit.
  static std::atomic<int> max_pairs_cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  int max_pairs = dev < 64 ? max_pairs_cache[dev].load(std::memory_order_acquire) : 0;
  if (max_pairs <= 0) {
    cfg.gridDim = dim3(grid & ~1);
    if (cudaOccupancyMaxActiveClusters(&max_pairs, kern, &cfg) != cudaSuccess || max_pairs <= 0) return cudaErrorInvalidConfiguration;
    if (dev < 64) max_pairs_cache[dev].store(max_pairs, std::memory_order_release);
  }
  grid = std::min(grid & ~1, 2 * max_pairs);
  if (grid <= 0) return cudaSuccess;
  cfg.gridDim = dim3(grid);
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a, tA, tB);
}

// Routed (block-scaled) GEMMs: the configurations above.  Dense (bf16) GEMMs:
// swap-AB with 32 or 176 token rows (128 is only ever asked for the routed ones).
template <int KIND, int EPI>
static cudaError_t launch_gemm(int bn, const GemmArgs& a, const CUtensorMap& tA, const BMaps& tB, int grid,
                               cudaStream_t s) {
  if constexpr (KIND == KIND_MX) {
    if (bn == kBNMid) return launch_gemm_cfg<KIND, EPI, kBNMid, kStagesMid, true>(a, tA, tB, grid, s);
    if (bn == kBNPair) {
      // pairs of 256-row m-tiles; an odd m-tile count runs the same tiles on single CTAs
      if (a.dense_rows < 0 && a.m_tiles % 2 == 0 && a.M_total % 256 == 0)
        return launch_gemm_pair<EPI>(a, tA, tB, grid, s);
      return launch_gemm_cfg<KIND, EPI, kBNPair, 4>(a, tA, tB, grid, s);
    }
  }
  if (bn == kBNSmall) return launch_gemm_cfg<KIND, EPI, kBNSmall, kStagesSmall>(a, tA, tB, grid, s);
  return launch_gemm_cfg<KIND, EPI, kBN, kStages>(a, tA, tB, grid, s);
}

// K splits for a dense GEMM with `tiles` output tiles and k_tiles K tiles: when the tiles
// would fill less than half the SMs (few tokens), split K so that up to one CTA runs per SM,
// keeping at least 4 K tiles per split and the fp32 partials (ksplit * elems) within the
// workspace.  1 = no split.  No split is empty: (ks - 1) * ceil(k_tiles / ks) < k_tiles.
static int dense_ksplit(const moe_plan_s* p, int tiles, int k_tiles, size_t elems) {
  const int cap = std::min(p->num_sms, kSplitMaxCtas);
  if (tiles <= 0 || 2 * tiles > cap) return 1;
  int ks = std::min(cap / tiles, k_tiles / 4);
  while (ks > 1 && (size_t)ks * elems > (size_t)kSplitMaxCtas * kBN * 256) --ks;
  if (ks <= 1) return 1;
  const int per = (k_tiles + ks - 1) / ks;
  return (k_tiles + per - 1) / per;   // no empty split
}

static GemmArgs base_args(const moe_plan_s* p) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.status = p->at<unsigned int>(p->o_status);
  a.dense_rows = -1;
  a.ksplit = 1;
  a.pf_dist = p->pf_dist;
  a.pf_b = p->pf_b;
  return a;
}

static cudaError_t set_smem_attrs() {
  static std::atomic<uint64_t> place_done{0};
  return ensure_smem_attr(perm_place_kernel, 160 * 1024, place_done);
}

// histogram -> scan -> placement into the plan workspace
static cudaError_t run_permute(moe_plan_s* p, const int32_t* idx, int T, int bn, cudaStream_t s) {
  if (set_smem_attrs() != cudaSuccess) return cudaErrorInvalidValue;
  const int nch = p->nchunks(T);
  int* chunk = p->at<int>(p->o_chunk);
  launch_k(perm_histogram_kernel, nch, 256, p->E * 4, s, idx, T, p->k, p->E, p->tokens_per_chunk(), chunk,
                                                   p->at<unsigned int>(p->o_status));
  launch_k(perm_scan_kernel, 1, 1024, (2 * p->E + 32) * 4, s, chunk, nch, p->E, bn, p->at<int>(p->o_counts),
                                                         p->at<int>(p->o_offsets), p->at<int>(p->o_tiles));
  launch_k(perm_place_kernel, nch, kPermThreads, (kPermThreads / 32) * p->E * 4, s,
      idx, T, p->k, p->E, p->tokens_per_chunk(), chunk, p->at<int>(p->o_perm), p->at<int>(p->o_inv));
  return cudaGetLastError();
}

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_ALIGNMENT: return "misaligned pointer";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_NOT_INITIALIZED: return "no workspace attached";
    case MOE_ERR_DEVICE_FAULT: return "device flagged invalid input";
  }
  return "unknown status";
}

moe_status_t moe_plan_create(int T_max, int d, int E, int k, int I, int I_shared, moe_act_t act,
                             moe_bias_mode_t bias_mode, int flags, moe_plan_t* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if ((act != MOE_ACT_SILU_GLU && act != MOE_ACT_CLAMPED_SWIGLU) ||
      (bias_mode != MOE_BIAS_LOGIT && bias_mode != MOE_BIAS_SELECT_ONLY) || (flags & ~MOE_FLAG_STATIC_ROUTER))
    return MOE_ERR_INVALID_ARG;
  if (T_max < 0 || d <= 0 || E <= 0 || k <= 0 || I <= 0 || I_shared < 0) return MOE_ERR_INVALID_ARG;
  if (d % 128 || I % 128 || I_shared % 128 || k > E || k > 32 || E > kMaxExperts)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T_max * k > (1ll << 30)) return MOE_ERR_UNSUPPORTED_SHAPE;
  moe_plan_s* p = new moe_plan_s();
  p->T_max = T_max; p->d = d; p->E = E; p->k = k; p->I = I; p->Is = I_shared;
  p->act = act;
  p->bias_mode = bias_mode;
  p->flags = flags;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
      p->num_sms = sms;
  }
  carve(p);
  *out = p;
  return MOE_OK;
}

moe_status_t moe_plan_workspace_bytes(moe_plan_t p, size_t* bytes) {
  if (!p || !bytes) return MOE_ERR_INVALID_ARG;
  *bytes = p->total;
  return MOE_OK;
}

moe_status_t moe_plan_set_workspace(moe_plan_t p, void* dev_ptr, size_t bytes) {
  if (!p || !dev_ptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(dev_ptr, 256)) return MOE_ERR_ALIGNMENT;
  if (bytes < p->total) return MOE_ERR_INVALID_ARG;
  p->ws = (char*)dev_ptr;
  p->ws_bytes = bytes;
  p->planes_of = nullptr;   // the router planes live in the workspace
  if (cudaMemset(p->ws + p->o_status, 0, 256) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_plan_check(moe_plan_t p, void* stream, unsigned int* bits) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!p->ws) return MOE_ERR_NOT_INITIALIZED;
  unsigned int v = 0;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&v, p->ws + p->o_status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(p->ws + p->o_status, 0, 4) != cudaSuccess) return MOE_ERR_CUDA;
  if (bits) *bits = v;
  if (v & MOE_DEV_ERR_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (v) return MOE_ERR_DEVICE_FAULT;
  return MOE_OK;
}

moe_status_t moe_plan_destroy(moe_plan_t p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  delete p;
  return MOE_OK;
}

moe_status_t moe_quant_mxfp8(const void* x, int rows, int cols, uint8_t* q, uint8_t* sc, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 32) return rows < 0 ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!x || !q || !sc) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16)) return MOE_ERR_ALIGNMENT;
  const long long n = (long long)rows * (cols / 32);
  const int threads = 256;
  quant_mxfp8_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, S(stream)>>>(
      (const uint16_t*)x, rows, cols, q, sc);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_permute(moe_plan_t p, const int32_t* idx, int T, int32_t* counts, int32_t* offsets,
                         int32_t* perm_tok, int32_t* inv, void* stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!p->ws) return MOE_ERR_NOT_INITIALIZED;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T > p->T_max) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!counts || !offsets || (T > 0 && (!idx || !perm_tok || !inv))) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = S(stream);
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, p->E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(offsets, 0, (p->E + 1) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (run_permute(p, idx, T, p->tile_rows(T), s) != cudaSuccess) return MOE_ERR_CUDA;
  const size_t A = (size_t)T * p->k;
  if (cudaMemcpyAsync(counts, p->ws + p->o_counts, p->E * 4, cudaMemcpyDeviceToDevice, s) ||
      cudaMemcpyAsync(offsets, p->ws + p->o_offsets, (p->E + 1) * 4, cudaMemcpyDeviceToDevice, s) ||
      cudaMemcpyAsync(perm_tok, p->ws + p->o_perm, A * 4, cudaMemcpyDeviceToDevice, s) ||
      cudaMemcpyAsync(inv, p->ws + p->o_inv, A * 4, cudaMemcpyDeviceToDevice, s))
    return MOE_ERR_CUDA;
  p->last_T = T;
  return MOE_OK;
}

moe_status_t moe_route(moe_plan_t p, const void* x, int T, const float* W_r, const float* bias,
                       int32_t* idx, float* w, float* logits_opt, void* stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!p->ws) return MOE_ERR_NOT_INITIALIZED;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T > p->T_max) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!x || !W_r || !idx || !w) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(W_r, 16)) return MOE_ERR_ALIGNMENT;
  cudaStream_t s = S(stream);
  const int d = p->d, E = p->E;
  __nv_bfloat16* planes = p->at<__nv_bfloat16>(p->o_planes);
  float* z = logits_opt ? logits_opt : p->at<float>(p->o_logits);
  if (!aligned(z, 16)) return MOE_ERR_ALIGNMENT;
  if (!(p->flags & MOE_FLAG_STATIC_ROUTER) || p->planes_of != (const void*)W_r) {
    p->prof.begin(MOE_STAGE_ROUTER_SPLIT, s);
    launch_k(router_split_kernel, dim3((E + 31) / 32, (d + 63) / 64), dim3(256), 0, s, W_r, d, E, planes);
    p->prof.end(s);
    p->planes_of = W_r;
  }
  CUtensorMap tA, tB;
  if (!make_map(&tA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, planes, 3ull * d, E, 3ull * d * 2, 64, 128) ||
      !make_map(&tB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, d, T, (uint64_t)d * 2, 64, 32))
    return MOE_ERR_CUDA;
  RouterArgs ra;
  ra.T = T;
  ra.d = d;
  ra.E = E;
  ra.m_tiles = (E + 127) / 128;
  // MOE_BIAS_SELECT_ONLY: z stays unbiased; the bias only enters the top-k key
  const bool select_only = p->bias_mode == MOE_BIAS_SELECT_ONLY;
  ra.bias = select_only ? nullptr : bias;
  ra.z = z;
  ra.zpart = p->at<float>(p->o_zpart);
  ra.status = p->at<unsigned int>(p->o_status);
  {
    // Split K (i) when the expert x token tiles would fill less than half the SMs, so that
    // the plane reads (3 x E x d bf16) spread over the whole GPU, and (ii) otherwise by up
    // to 3 when that evens out the last wave of the persistent grid (T=8192: 448 tiles on
    // 148 SMs run 4 waves for 3.03 waves of work; split 3 runs 10 for 9.08).
    const int chains = d / 64;
    const int base_tiles = ((T + kRouterBN - 1) / kRouterBN) * ra.m_tiles;
    const int cap = std::min(p->num_sms, kRouterMaxCtas);
    int ksplit = 1;
    if (2 * base_tiles <= cap) {
      ksplit = std::min(chains, cap / base_tiles);
    } else {
      double best = 0.0;
      for (int sp = 1; sp <= 3 && chains / sp >= 16; ++sp) {
        const long long units = (long long)base_tiles * sp;
        const double eff = (double)units / (double)(((units + p->num_sms - 1) / p->num_sms) * p->num_sms);
        if (eff > best + 0.03) { best = eff; ksplit = sp; }
      }
    }
    ra.chains_per = (chains + ksplit - 1) / ksplit;
    ra.ksplit = (chains + ra.chains_per - 1) / ra.chains_per;
    if ((size_t)ra.ksplit * T * E > p->zpart_floats) {   // cannot happen with the sizing above
      ra.ksplit = 1;
      ra.chains_per = chains;
    }
    p->last_ksplit = ra.ksplit;
    using RC = RouterCfg<kRouterBN, kRouterStages>;
    auto kern = router_kernel<kRouterBN, kRouterStages>;
    static std::atomic<uint64_t> router_done{0};
    if (ensure_smem_attr(kern, RC::SMEM_BYTES, router_done) != cudaSuccess) return MOE_ERR_CUDA;
    const int tiles = base_tiles * ra.ksplit;
    p->prof.begin(MOE_STAGE_ROUTER_GEMM, s);
    launch_k(kern, std::min(tiles, p->num_sms), 320, RC::SMEM_BYTES, s, ra, tA, tB);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    p->prof.end(s);
  }
  {
    // selection (and, after a K split, the sum of the partials): 8 tokens per CTA when
    // there are enough to fill the GPU that way, else one; their keys in shared memory
    const int tpc = T >= 8 * p->num_sms ? 8 : 1;
    const int grid = std::min((T + tpc - 1) / tpc, 32 * p->num_sms);
    const float* sel = select_only ? bias : nullptr;
    const float* lbias = select_only ? nullptr : bias;
    const long long plane = (long long)T * E;
    const int k = p->k;
    const int smem = tpc * E * 4;   // <= 8 * 4096 * 4 = 128 KB
    cudaError_t err = cudaSuccess;
    auto launch = [&](auto kern, std::atomic<uint64_t>& done) {
      err = ensure_smem_attr(kern, 8 * kMaxExperts * 4, done);
      if (err == cudaSuccess) launch_k(kern, grid, 256, smem, s, ra.zpart, ra.ksplit, plane, lbias, sel, z, T, E, k, tpc, idx, w);
    };
    static std::atomic<uint64_t> sel_done[5];
    p->prof.begin(MOE_STAGE_TOPK, s);
    if (E <= 256)       launch(route_select_kernel<1>, sel_done[0]);
    else if (E <= 512)  launch(route_select_kernel<2>, sel_done[1]);
    else if (E <= 1024) launch(route_select_kernel<4>, sel_done[2]);
    else if (E <= 2048) launch(route_select_kernel<8>, sel_done[3]);
    else                launch(route_select_kernel<16>, sel_done[4]);
    if (err != cudaSuccess || cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    p->prof.end(s);
  }
  p->last_T = T;
  return MOE_OK;
}

// A dense bf16 GEMM of the latent option: out fp32 [T][M] = act [T][K] . W [M][K]^T.
static cudaError_t dense_bf16_f32(const moe_plan_s* p, const void* W, int M, const void* act, int K, int T,
                                  float* out, int bn, cudaStream_t s) {
  CUtensorMap tA;
  BMaps tB;
  if (!make_map(&tA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, K, M, (uint64_t)K * 2, 64, 256) ||
      !make_bmaps(&tB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, K, T, (uint64_t)K * 2, 64))
    return cudaErrorInvalidValue;
  GemmArgs a = base_args(p);
  a.dense_rows = T;
  a.num_groups = 1;
  a.M_total = M;
  a.m_tiles = (M + 255) / 256;
  a.k_tiles = K / 64;
  a.kb_wrap = a.k_tiles;
  a.B_rows = T;
  a.out0 = out;
  a.ld_out = M;
  const int tiles = ((T + bn - 1) / bn) * a.m_tiles;
  return launch_gemm<KIND_BF16, EPI_F32>(bn, a, tA, tB, std::min(tiles, p->num_sms), s);
}

static moe_status_t forward_impl(moe_plan_t p, const void* x, int T, const int32_t* idx, const float* w,
                                 const moe_latent_bf16* lat, const moe_experts_mxfp4* ex,
                                 const moe_shared_bf16* sh, void* y, void* stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!p->ws) return MOE_ERR_NOT_INITIALIZED;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T > p->T_max) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!x || !idx || !w || !ex || !y || !ex->w_gu || !ex->s_gu || !ex->w_dn || !ex->s_dn)
    return MOE_ERR_INVALID_ARG;
  if ((p->Is > 0) != (sh != nullptr)) return MOE_ERR_INVALID_ARG;
  if (sh && (!sh->w_gu || !sh->w_dn)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ex->w_gu, 256) || !aligned(ex->w_dn, 256) ||
      !aligned(ex->s_gu, 16) || !aligned(ex->s_dn, 16) ||
      (sh && (!aligned(sh->w_gu, 16) || !aligned(sh->w_dn, 16))))
    return MOE_ERR_ALIGNMENT;
  if ((lat != nullptr) != (p->dl > 0)) return MOE_ERR_INVALID_ARG;
  if (lat && (!lat->w_down || !lat->gamma || !lat->w_up)) return MOE_ERR_INVALID_ARG;
  if (lat && (!aligned(lat->w_down, 16) || !aligned(lat->w_up, 16) || !aligned(lat->gamma, 4)))
    return MOE_ERR_ALIGNMENT;
  cudaStream_t s = S(stream);
  const int d = p->d, E = p->E, k = p->k, I = p->I, Is = p->Is;
  const int de = lat ? p->dl : d;   // width the routed experts act on
  const int A = T * k;
  const int bn = p->tile_rows(T);                    // routed GEMM tiles
  const int dbn = p->dense_rows(T);                  // dense GEMM tiles

  // latent option: x_l = x W_ld^T, x_n = bf16(RMSNorm(x_l) * gamma) feeds the experts
  const void* xin = x;
  if (lat) {
    float* xl = p->at<float>(p->o_xl);
    __nv_bfloat16* xn = p->at<__nv_bfloat16>(p->o_xn);
    p->prof.begin(MOE_STAGE_LATENT_IN, s);
    if (dense_bf16_f32(p, lat->w_down, de, x, d, T, xl, dbn, s) != cudaSuccess) return MOE_ERR_CUDA;
    launch_k(rmsnorm_bf16_kernel, T, 256, 0, s, xl, lat->gamma, de, p->eps_lat, xn);
    p->prof.end(s);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    xin = xn;
  }

  // a4: group assignments by expert
  p->prof.begin(MOE_STAGE_PERMUTE, s);
  if (run_permute(p, idx, T, bn, s) != cudaSuccess) return MOE_ERR_CUDA;
  p->prof.end(s);
  // a1: quantise x to MXFP8 and scatter rows into expert order
  uint8_t* xq = p->at<uint8_t>(p->o_xq);
  uint8_t* xs = p->at<uint8_t>(p->o_xs);
  {
    const long long n = (long long)T * (de / 32);
    p->prof.begin(MOE_STAGE_QUANT, s);
    uint8_t* xs_tok = p->at<uint8_t>(p->o_xs_tok);
    launch_k(quant_scatter_kernel, (unsigned)((n + 255) / 256), 256, 0, s,
        (const uint16_t*)xin, T, de, k, p->at<int>(p->o_inv), A, xq, xs_tok);
    const int max_gt = A / bn + E + 1;   // bound on the group-tiles of this call
    launch_k(scale_tiles_kernel, max_gt, 256, 0, s, xs_tok, de / 32, p->at<int>(p->o_perm), p->at<int>(p->o_counts),
                                              p->at<int>(p->o_offsets), p->at<int>(p->o_tiles), E, de / 128, xs);
    p->prof.end(s);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  uint8_t* hq = p->at<uint8_t>(p->o_hq);
  uint8_t* hs = p->at<uint8_t>(p->o_hs);
  __nv_bfloat16* O = p->at<__nv_bfloat16>(p->o_O);
  // a5/a6: gate/up grouped GEMM, SiLU-GLU and MXFP8 requantisation in the epilogue
  {
    CUtensorMap tA;
    BMaps tB;
    // tile-major weights: 128-element rows of 64 B, one 256-row box per (expert, m-tile, k-tile)
    if (!make_map(&tA, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, ex->w_gu, 128, (uint64_t)E * 2 * I * (de / 128), 64, 128, 256) ||
        !make_bmaps(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, de, A, de, 128))
      return MOE_ERR_CUDA;
    GemmArgs a = base_args(p);
    a.counts = p->at<int>(p->o_counts);
    a.offsets = p->at<int>(p->o_offsets);
    a.tile_prefix = p->at<int>(p->o_tiles);
    a.num_groups = E;
    a.M_total = 2 * I;
    a.m_tiles = 2 * I / 256;
    a.k_tiles = de / 128;
    a.kb_wrap = a.k_tiles;
    a.B_rows = A;
    a.sfa = (const uint8_t*)ex->s_gu;
    a.a_ptr = (const uint8_t*)ex->w_gu;
    a.sfb = xs;
    a.out0 = hq;
    a.out1 = hs;
    a.ld_out = I;
    p->prof.begin(MOE_STAGE_GATE_UP, s);
    const cudaError_t e = p->act == MOE_ACT_CLAMPED_SWIGLU
        ? launch_gemm<KIND_MX, EPI_GLU_MX8_CLAMPED>(bn, a, tA, tB, p->num_sms, s)
        : launch_gemm<KIND_MX, EPI_GLU_MX8>(bn, a, tA, tB, p->num_sms, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    p->prof.end(s);
  }
  // a7: down grouped GEMM -> O (bf16, expert order)
  {
    CUtensorMap tA;
    BMaps tB;
    if (!make_map(&tA, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, ex->w_dn, 128,
                  (uint64_t)E * ((de + 255) / 256) * 256 * (I / 128), 64, 128, 256) ||
        !make_bmaps(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, hq, I, A, I, 128))
      return MOE_ERR_CUDA;
    GemmArgs a = base_args(p);
    a.counts = p->at<int>(p->o_counts);
    a.offsets = p->at<int>(p->o_offsets);
    a.tile_prefix = p->at<int>(p->o_tiles);
    a.num_groups = E;
    a.M_total = de;
    a.m_tiles = (de + 255) / 256;
    a.k_tiles = I / 128;
    a.kb_wrap = a.k_tiles;
    a.B_rows = A;
    a.sfa = (const uint8_t*)ex->s_dn;
    a.a_ptr = (const uint8_t*)ex->w_dn;
    a.sfb = hs;
    a.out0 = O;
    a.ld_out = de;
    p->prof.begin(MOE_STAGE_DOWN, s);
    if (launch_gemm<KIND_MX, EPI_BF16>(bn, a, tA, tB, p->num_sms, s) != cudaSuccess) return MOE_ERR_CUDA;
    p->prof.end(s);
  }
  // a8: shared expert (bf16)
  float* ys = nullptr;
  if (sh) {
    __nv_bfloat16* hsh = p->at<__nv_bfloat16>(p->o_hsh);
    ys = p->at<float>(p->o_ys);
    CUtensorMap tA;
    BMaps tB;
    if (!make_map(&tA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sh->w_gu, d, 2ull * Is, (uint64_t)d * 2, 64, 256) ||
        !make_bmaps(&tB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, d, T, (uint64_t)d * 2, 64))
      return MOE_ERR_CUDA;
    GemmArgs a = base_args(p);
    a.dense_rows = T;
    a.num_groups = 1;
    a.M_total = 2 * Is;
    a.m_tiles = 2 * Is / 256;
    a.k_tiles = d / 64;
    a.kb_wrap = a.k_tiles;
    a.B_rows = T;
    a.out0 = hsh;
    a.ld_out = Is;
    int tiles = ((T + dbn - 1) / dbn) * a.m_tiles;
    float* spart = p->at<float>(p->o_spart);
    p->prof.begin(MOE_STAGE_SHARED_GATE_UP, s);
    const int ks_gu = dense_ksplit(p, tiles, a.k_tiles, (size_t)T * 2 * Is);
    if (ks_gu > 1) {
      // few token tiles: split K over the SMs, fp32 partials, then sum + GLU + bf16
      a.ksplit = ks_gu;
      a.k_per = (a.k_tiles + ks_gu - 1) / ks_gu;
      a.split_stride = (long long)T * 2 * Is;
      a.out0 = spart;
      a.ld_out = 2 * Is;
      if (launch_gemm<KIND_BF16, EPI_F32>(dbn, a, tA, tB, std::min(tiles * ks_gu, p->num_sms), s) != cudaSuccess)
        return MOE_ERR_CUDA;
      const long long n = (long long)T * Is;
      if (p->act == MOE_ACT_CLAMPED_SWIGLU)
        launch_k(split_glu_reduce_kernel<1>, (unsigned)((n + 255) / 256), 256, 0, s, spart, ks_gu, T, Is, a.split_stride, hsh);
      else
        launch_k(split_glu_reduce_kernel<0>, (unsigned)((n + 255) / 256), 256, 0, s, spart, ks_gu, T, Is, a.split_stride, hsh);
      if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    } else {
      const cudaError_t e = p->act == MOE_ACT_CLAMPED_SWIGLU
          ? launch_gemm<KIND_BF16, EPI_GLU_BF16_CLAMPED>(dbn, a, tA, tB, std::min(tiles, p->num_sms), s)
          : launch_gemm<KIND_BF16, EPI_GLU_BF16>(dbn, a, tA, tB, std::min(tiles, p->num_sms), s);
      if (e != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    p->last_shared_split = ks_gu;
    p->prof.end(s);
    CUtensorMap tA2;
    BMaps tB2;
    if (!make_map(&tA2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sh->w_dn, Is, d, (uint64_t)Is * 2, 64, 256) ||
        !make_bmaps(&tB2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, hsh, Is, T, (uint64_t)Is * 2, 64))
      return MOE_ERR_CUDA;
    GemmArgs b = base_args(p);
    b.dense_rows = T;
    b.num_groups = 1;
    b.M_total = d;
    b.m_tiles = (d + 255) / 256;
    b.k_tiles = Is / 64;
    b.kb_wrap = b.k_tiles;
    b.B_rows = T;
    b.out0 = ys;
    b.ld_out = d;
    tiles = ((T + dbn - 1) / dbn) * b.m_tiles;
    p->prof.begin(MOE_STAGE_SHARED_DOWN, s);
    const int ks_dn = dense_ksplit(p, tiles, b.k_tiles, (size_t)T * d);
    if (ks_dn > 1) {
      b.ksplit = ks_dn;
      b.k_per = (b.k_tiles + ks_dn - 1) / ks_dn;
      b.split_stride = (long long)T * d;
      b.out0 = spart;
      if (launch_gemm<KIND_BF16, EPI_F32>(dbn, b, tA2, tB2, std::min(tiles * ks_dn, p->num_sms), s) != cudaSuccess)
        return MOE_ERR_CUDA;
      const long long n = (long long)T * d;
      launch_k(split_sum_kernel, (unsigned)((n + 255) / 256), 256, 0, s, spart, ks_dn, n, b.split_stride, ys);
      if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    } else {
      if (launch_gemm<KIND_BF16, EPI_F32>(dbn, b, tA2, tB2, std::min(tiles, p->num_sms), s) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    p->last_shared_split_dn = ks_dn;
    p->prof.end(s);
  } else {
    p->last_shared_split = p->last_shared_split_dn = 0;
  }
  if (!lat) {
    // a9: weighted combine with the shared output
    p->prof.begin(MOE_STAGE_COMBINE, s);
    launch_k(combine_kernel, dim3(T, (d + kCombineCols - 1) / kCombineCols), kCombineThreads, k * 8, s,
        O, ys, w, p->at<int>(p->o_inv), T, d, k, (__nv_bfloat16*)y);
    p->prof.end(s);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    // latent option: y_l = bf16(sum_j w_j O_j) in the latent, y = bf16(y_l W_lu^T + y_s)
    __nv_bfloat16* yl = p->at<__nv_bfloat16>(p->o_yl);
    float* yr = p->at<float>(p->o_yr);
    p->prof.begin(MOE_STAGE_COMBINE, s);
    launch_k(combine_kernel, dim3(T, (de + kCombineCols - 1) / kCombineCols), kCombineThreads, k * 8, s,
        O, nullptr, w, p->at<int>(p->o_inv), T, de, k, yl);
    p->prof.end(s);
    p->prof.begin(MOE_STAGE_LATENT_OUT, s);
    if (dense_bf16_f32(p, lat->w_up, d, yl, de, T, yr, dbn, s) != cudaSuccess) return MOE_ERR_CUDA;
    const long long n = (long long)T * d;
    launch_k(add_bf16_kernel, (unsigned)((n / 4 + 255) / 256), 256, 0, s, yr, ys, n, (__nv_bfloat16*)y);
    p->prof.end(s);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  p->last_T = T;
  p->last_bn = bn;
  return MOE_OK;
}

moe_status_t moe_forward(moe_plan_t p, const void* x, int T, const int32_t* idx, const float* w,
                         const moe_experts_mxfp4* ex, const moe_shared_bf16* sh, void* y, void* stream) {
  if (p && p->dl > 0) return MOE_ERR_INVALID_ARG;   // a latent plan takes moe_forward_latent
  return forward_impl(p, x, T, idx, w, nullptr, ex, sh, y, stream);
}

moe_status_t moe_forward_latent(moe_plan_t p, const void* x, int T, const int32_t* idx, const float* w,
                                const moe_latent_bf16* latent, const moe_experts_mxfp4* ex,
                                const moe_shared_bf16* sh, void* y, void* stream) {
  if (!latent) return MOE_ERR_INVALID_ARG;
  return forward_impl(p, x, T, idx, w, latent, ex, sh, y, stream);
}

moe_status_t moe_plan_set_latent(moe_plan_t p, int d_latent, float eps) {
  if (!p || p->ws) return MOE_ERR_INVALID_ARG;
  if (d_latent <= 0 || d_latent > p->d || eps <= 0.0f) return MOE_ERR_INVALID_ARG;
  if (d_latent % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  p->dl = d_latent;
  p->eps_lat = eps;
  carve(p);
  return MOE_OK;
}

moe_status_t moe_expert_bytes(int d, int I, int E, size_t* w_gu, size_t* s_gu, size_t* w_dn, size_t* s_dn) {
  if (d <= 0 || I <= 0 || E <= 0 || !w_gu || !s_gu || !w_dn || !s_dn) return MOE_ERR_INVALID_ARG;
  if (d % 128 || I % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  *w_gu = (size_t)E * 2 * I * (d / 2);
  *s_gu = (size_t)E * (2 * I / 256) * (d / 128) * 1024;
  *w_dn = (size_t)E * ((d + 255) / 256) * 256 * (I / 2);
  *s_dn = (size_t)E * ((d + 255) / 256) * (I / 128) * 1024;
  return MOE_OK;
}

moe_status_t moe_pack_expert_mxfp4(int d, int I, int e, const float* wg, const float* wu, const float* wd,
                                   const moe_experts_mxfp4* dst, void* stream) {
  if (d <= 0 || I <= 0 || e < 0 || !wg || !wu || !wd || !dst || !dst->w_gu || !dst->s_gu || !dst->w_dn ||
      !dst->s_dn)
    return MOE_ERR_INVALID_ARG;
  if (d % 128 || I % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(wg, 16) || !aligned(wu, 16) || !aligned(wd, 16)) return MOE_ERR_ALIGNMENT;
  cudaStream_t s = S(stream);
  const size_t gu_w = (size_t)2 * I * (d / 2), gu_s = (size_t)(2 * I / 256) * (d / 128) * 1024;
  const size_t dn_w = (size_t)((d + 255) / 256) * 256 * (I / 2), dn_s = (size_t)((d + 255) / 256) * (I / 128) * 1024;
  uint8_t* wgu = (uint8_t*)dst->w_gu + (size_t)e * gu_w;
  uint8_t* sgu = (uint8_t*)dst->s_gu + (size_t)e * gu_s;
  uint8_t* wdn = (uint8_t*)dst->w_dn + (size_t)e * dn_w;
  uint8_t* sdn = (uint8_t*)dst->s_dn + (size_t)e * dn_s;
  // the down weights' last 256-row tile may have an unused half: keep it defined
  if (cudaMemsetAsync(sdn, 0, dn_s, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (d % 256 && cudaMemsetAsync(wdn, 0, dn_w, s) != cudaSuccess) return MOE_ERR_CUDA;
  long long n = 2ll * I * (d / 32);
  pack_mxfp4_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(wg, wu, I, d, 1, wgu, sgu);
  n = (long long)d * (I / 32);
  pack_mxfp4_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(wd, nullptr, d, I, 0, wdn, sdn);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_pack_shared_bf16(int d, int Is, const void* wg, const void* wu, const void* wd,
                                  const moe_shared_bf16* dst, void* stream) {
  if (d <= 0 || Is <= 0 || !wg || !wu || !wd || !dst || !dst->w_gu || !dst->w_dn) return MOE_ERR_INVALID_ARG;
  if (d % 128 || Is % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = S(stream);
  const size_t row = (size_t)d * 2;
  for (int b = 0; b < Is / 128; ++b) {
    char* out = (char*)dst->w_gu + (size_t)256 * b * row;
    if (cudaMemcpyAsync(out, (const char*)wg + (size_t)128 * b * row, 128 * row, cudaMemcpyDeviceToDevice, s) ||
        cudaMemcpyAsync(out + 128 * row, (const char*)wu + (size_t)128 * b * row, 128 * row,
                        cudaMemcpyDeviceToDevice, s))
      return MOE_ERR_CUDA;
  }
  if (cudaMemcpyAsync(dst->w_dn, wd, (size_t)d * Is * 2, cudaMemcpyDeviceToDevice, s)) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_route_margin_quantiles(moe_plan_t p, const float* logits, const float* select_bias, int T,
                                        const double* levels, int n_levels, float* quantiles, void* stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!p->ws) return MOE_ERR_NOT_INITIALIZED;
  if (T <= 0 || n_levels <= 0 || !logits || !levels || !quantiles) return MOE_ERR_INVALID_ARG;
  if (T > p->T_max || n_levels > kMaxQuantLevels) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(logits, 4) || !aligned(quantiles, 4) || (select_bias && !aligned(select_bias, 4)))
    return MOE_ERR_ALIGNMENT;
  QuantRanks rk;
  memset(&rk, 0, sizeof(rk));
  for (int i = 0; i < n_levels; ++i) {
    const double q = levels[i];
    if (!(q >= 0.0 && q <= 1.0)) return MOE_ERR_INVALID_ARG;   // also rejects NaN
    const double j = std::ceil(q * (double)T);
    rk.r[i] = (int)std::min<double>(std::max<double>(j, 1.0), (double)T);
  }
  cudaStream_t s = S(stream);
  static std::atomic<uint64_t> kth_done{0};
  if (ensure_smem_attr(kth_key_kernel, 160 * 1024, kth_done) != cudaSuccess) return MOE_ERR_CUDA;
  float* theta = p->at<float>(p->o_theta);
  const int wpb = 8;
  kth_key_kernel<<<(T + wpb - 1) / wpb, wpb * 32, (size_t)wpb * p->E * 4, s>>>(logits, select_bias, T, p->E, p->k,
                                                                               theta);
  margin_quantile_kernel<<<dim3((p->E + 31) / 32, n_levels), kQuantThreads, 0, s>>>(logits, select_bias, theta, T,
                                                                                     p->E, rk, quantiles);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_quantile_balance(moe_plan_t p, const float* logits, const float* bias, int T,
                                  const double* levels, int n_levels, moe_bias_rule_t rule, void* user,
                                  float* bias_next, void* stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!p->ws) return MOE_ERR_NOT_INITIALIZED;
  if (!rule || !bias || !bias_next) return MOE_ERR_INVALID_ARG;
  if (!aligned(bias, 4) || !aligned(bias_next, 4)) return MOE_ERR_ALIGNMENT;
  // the margins read the selection key: z + b in the select-only mode, z otherwise (a
  // logit bias is already inside z)
  const float* sel = p->bias_mode == MOE_BIAS_SELECT_ONLY ? bias : nullptr;
  float* q = p->at<float>(p->o_qbuf);
  const moe_status_t st = moe_route_margin_quantiles(p, logits, sel, T, levels, n_levels, q, stream);
  if (st != MOE_OK) return st;
  rule(q, n_levels, p->E, bias, bias_next, stream, user);
  return MOE_OK;
}

moe_status_t moe_plan_set_option(moe_plan_t p, int option, int value) {
  if (!p) return MOE_ERR_INVALID_ARG;
  switch (option) {
    case MOE_OPT_PREFETCH_DIST:
      if (value < 0 || value > 64) return MOE_ERR_INVALID_ARG;
      p->pf_dist = value;
      return MOE_OK;
    case MOE_OPT_PREFETCH_B:
      p->pf_b = value != 0;
      return MOE_OK;
    case MOE_OPT_TILE_N:
      if (value != 0 && value != kBNSmall && value != kBNMid && value != kBNPair && value != kBN)
        return MOE_ERR_INVALID_ARG;
      p->tile_n_opt = value;
      return MOE_OK;
  }
  return MOE_ERR_INVALID_ARG;
}

moe_status_t moe_plan_get_option(moe_plan_t p, int option, int* value) {
  if (!p || !value) return MOE_ERR_INVALID_ARG;
  switch (option) {
    case MOE_OPT_PREFETCH_DIST: *value = p->pf_dist; return MOE_OK;
    case MOE_OPT_PREFETCH_B: *value = p->pf_b; return MOE_OK;
    case MOE_OPT_TILE_N: *value = p->last_bn; return MOE_OK;
    case MOE_OPT_ROUTER_SPLIT: *value = p->last_ksplit; return MOE_OK;
    case MOE_OPT_SHARED_SPLIT: *value = p->last_shared_split; return MOE_OK;
    case MOE_OPT_SHARED_SPLIT_DOWN: *value = p->last_shared_split_dn; return MOE_OK;
  }
  return MOE_ERR_INVALID_ARG;
}

moe_status_t moe_plan_set_profiling(moe_plan_t p, int enable) {
  if (!p) return MOE_ERR_INVALID_ARG;
  p->prof.on = enable != 0;
  p->prof.recs.clear();
  p->prof.used = 0;
  return MOE_OK;
}

moe_status_t moe_plan_stage_ms(moe_plan_t p, float* ms, int* launches, int n) {
  if (!p || !ms || n < MOE_NUM_STAGES) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    ms[i] = 0.0f;
    if (launches) launches[i] = 0;
  }
  for (const auto& r : p->prof.recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return MOE_ERR_CUDA;
    float t = 0.0f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return MOE_ERR_CUDA;
    ms[r.stage] += t;
    if (launches) launches[r.stage] += 1;
  }
  p->prof.recs.clear();
  p->prof.used = 0;
  return MOE_OK;
}

moe_status_t moe_debug_timeout_probe(moe_plan_t p, void* stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!p->ws) return MOE_ERR_NOT_INITIALIZED;
  timeout_probe_kernel<<<1, 32, 0, S(stream)>>>(p->at<unsigned int>(p->o_status));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_debug_buffer(moe_plan_t p, int which, void** ptr, size_t* bytes) {
  if (!p || !ptr || !bytes) return MOE_ERR_INVALID_ARG;
  if (!p->ws) return MOE_ERR_NOT_INITIALIZED;
  const size_t A = (size_t)p->last_T * p->k, T = p->last_T;
  size_t off, n;
  switch (which) {
    case 0: off = p->o_xq; n = A * p->d; break;
    case 1: off = p->o_xs; n = (A / kBNMin + p->E + 1) * (p->d / 128) * SF_TILE_BYTES; break;
    case 2: off = p->o_hq; n = A * p->I; break;
    case 3: off = p->o_hs; n = (A / kBNMin + p->E + 1) * (p->I / 128) * SF_TILE_BYTES; break;
    case 4: off = p->o_O; n = A * p->d * 2; break;
    case 5: off = p->o_ys; n = T * p->d * 4; break;
    case 6: off = p->o_logits; n = T * p->E * 4; break;
    case 7: off = p->o_qbuf; n = (size_t)kMaxQuantLevels * p->E * 4; break;
    default: return MOE_ERR_INVALID_ARG;
  }
  *ptr = p->ws + off;
  *bytes = n;
  return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- grouping without allocation
// Fixed device scratch for moe_permute_noalloc: status word, per-chunk expert counts and
// the tile table.  Every device that loads this library keeps it until the process exits.
static constexpr size_t kNoAllocScratchBytes = 256 * 1024;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array in the current context.  In host code the array's
// name is only a host-side stand-in, so the address is looked up with the device current
// (cudaGetSymbolAddress, return code checked) once per device and context, and cached.  The
// cache is keyed on the context's unique id (cuCtxGetId): after cudaDeviceReset, or under
// another context on the same device, the address is looked up again.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

static bool current_ctx_id(unsigned long long* id) {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = (CtxGetCurrentFn)p;
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (CtxGetIdFn)p;
  });
  if (!get_cur || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

static void* noalloc_scratch(moe_status_t* st) {
  static std::mutex mu;
  static void* addr[64] = {};
  static unsigned long long ctx_of[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *st = MOE_ERR_CUDA;
    return nullptr;
  }
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || !have_id || ctx_of[dev] != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      *st = MOE_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
    ctx_of[dev] = have_id ? id : 0;
  }
  return addr[dev];
}

extern "C" moe_status_t moe_permute_noalloc(const int32_t* idx, int T, int E, int k, int32_t* counts,
                                            int32_t* offsets, int32_t* perm_tok, int32_t* inv,
                                            void* stream) {
  if (T < 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  if (k > E || k > 32 || E > kMaxExperts) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!counts || !offsets || (T > 0 && (!idx || !perm_tok || !inv))) return MOE_ERR_INVALID_ARG;
  const int nch = (T + kPermThreads - 1) / kPermThreads;
  const size_t o_chunk = 256, o_tiles = o_chunk + up((size_t)nch * E * 4, 256);
  if (o_tiles + (size_t)(E + 1) * 4 > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = S(stream);
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, (size_t)E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  moe_status_t st = MOE_OK;
  char* scratch = (char*)noalloc_scratch(&st);
  if (!scratch) return st;
  if (set_smem_attrs() != cudaSuccess) return MOE_ERR_CUDA;
  unsigned int* status = (unsigned int*)scratch;
  int* chunk = (int*)(scratch + o_chunk);
  int* tiles = (int*)(scratch + o_tiles);
  // the status word is the only part read before it is written: clear it
  if (cudaMemsetAsync(status, 0, 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  perm_histogram_kernel<<<nch, 256, E * 4, s>>>(idx, T, k, E, kPermThreads, chunk, status);
  perm_scan_kernel<<<1, 1024, (2 * E + 32) * 4, s>>>(chunk, nch, E, kBN, counts, offsets, tiles);
  perm_place_kernel<<<nch, kPermThreads, (kPermThreads / 32) * E * 4, s>>>(idx, T, k, E, kPermThreads,
                                                                         chunk, perm_tok, inv);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
