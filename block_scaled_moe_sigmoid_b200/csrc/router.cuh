// Router logits z = x . W_r + bias on the tensor cores, accurate to about fp32.
//
// W_r (fp32) is split into three bf16 planes, W = hi + mid + lo exactly, so each product
// x * plane is exact and the only rounding is in the accumulation.  The tensor core's
// fp32 accumulator loses about half an ulp per K=16 step (in one direction), which over
// K = 3 x 7168 would cost ~1e-4 absolute.  So every 64 columns of x (12 MMA steps over the
// three planes) form one short chain in a TMEM partial accumulator, and the epilogue warps
// add each partial into fp32 registers (round-to-nearest).  Two partial buffers let the
// tensor core run the next chain while the last one is drained.
//
// Tile: 128 experts (MMA M = lanes) x up to RBN tokens (MMA N = columns) x a range of
// 64-column chains.  With few tokens (decode) the expert x token tiles alone would occupy
// a handful of SMs, so K is split: split s covers chains [s * chains_per, ...) and writes
// its fp32 partial to zpart[s].  Roles as in gemm.cuh: warp 0 loads (TMA), warp 1 issues
// MMAs, warps 2..9 drain and store.
//
// Selection runs in the next launch (route_select_kernel in kernels.cuh), which also sums
// the split partials: a kernel boundary publishes the logits to it, where a selection fused
// into this epilogue needs GPU-scope fences and counters between CTAs, which measured far
// slower under this kernel's load.
#pragma once
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

struct RouterArgs {
  int T, d, E;
  int m_tiles;     // ceil(E / 128)
  int ksplit;      // K splits (1: no split)
  int chains_per;  // 64-column chains per split
  const float* bias;        // logit bias added to z (ksplit == 1), or NULL
  float* z;        // [T][E] logits (ksplit == 1)
  float* zpart;    // [ksplit][T][E] partials without bias (ksplit > 1)
  unsigned int* status;
};

struct RouterTile {
  int mt, row0, split, c0, c1;
};
__device__ __forceinline__ RouterTile router_tile(const RouterArgs& a, int rbn, int t) {
  const int n_tok_tiles = (a.T + rbn - 1) / rbn;
  const int per_split = n_tok_tiles * a.m_tiles;
  RouterTile r;
  r.split = t / per_split;
  const int rest = t - r.split * per_split;
  r.mt = rest % a.m_tiles;
  r.row0 = (rest / a.m_tiles) * rbn;
  r.c0 = r.split * a.chains_per;
  r.c1 = min(a.d / 64, r.c0 + a.chains_per);
  return r;
}

template <int RBN, int STAGES>
struct RouterCfg {
  static constexpr int A_PLANE = 128 * 128;          // 128 rows x 64 bf16
  static constexpr int A_BYTES = 3 * A_PLANE;
  static constexpr int B_BYTES = RBN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 1024;
  static constexpr int TMEM_COLS = 2 * RBN <= 256 ? 256 : 512;
  static_assert(RBN % 64 == 0 && RBN <= 256, "RBN");
  static_assert(STAGE_BYTES % 1024 == 0, "alignment");
  static_assert(SMEM_BYTES <= 232448, "smem");
};

template <int RBN, int STAGES>
__global__ void __launch_bounds__(320, 1)
    router_kernel(const __grid_constant__ RouterArgs args, const __grid_constant__ CUtensorMap tmA,
                  const __grid_constant__ CUtensorMap tmB) {
  using C = RouterCfg<RBN, STAGES>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full_bar = (uint64_t*)(smem + STAGES * C::STAGE_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* pfull = empty_bar + STAGES;   // [2] partial buffer written
  uint64_t* pempty = pfull + 2;           // [2] partial buffer drained
  uint64_t* drain_bar = pempty + 2;
  uint32_t* tmem_holder = (uint32_t*)(drain_bar + 1);
  volatile int* abort_flag = (volatile int*)(tmem_holder + 1);
  int* fills = (int*)(tmem_holder + 2);   // abort cleanup: [0] loads armed, [1] loads consumed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tok_tiles = (args.T + RBN - 1) / RBN;
  const int num_tiles = n_tok_tiles * args.m_tiles * args.ksplit;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(full_bar + s), 1);
      mbar_init(smem_u32(empty_bar + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(pfull + b), 1);
      mbar_init(smem_u32(pempty + b), 8);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fills[0] = fills[1] = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // the prologue above touches no global memory; the previous kernel's results are read
  // (and buffers it may still read are written) only after this
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------- loads
    const uint64_t pol = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int nfill = 0;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      const RouterTile rt = router_tile(args, RBN, t);
      const int mt = rt.mt, row0 = rt.row0;
      const int n_mma = (min(RBN, args.T - row0) + 15) & ~15;
      const int nB = (n_mma + 31) >> 5;
      for (int c = rt.c0; c < rt.c1; ++c) {
        if (lane == 0) ok = mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, args.status, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (lane == 0) {
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          const uint32_t fb = smem_u32(full_bar + stage);
          mbar_arrive_expect_tx(fb, C::A_BYTES + nB * 4096);
#pragma unroll
          for (int p = 0; p < 3; ++p)
            tma_load_2d(smem_u32(sA + p * C::A_PLANE), &tmA, fb, p * args.d + c * 64, mt * 128, pol);
          for (int i = 0; i < nB; ++i) tma_load_2d(smem_u32(sB + i * 4096), &tmB, fb, c * 64, row0 + 32 * i, pol);
        }
        __syncwarp();
        ++nfill;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (lane == 0) fills[0] = nfill;
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA: one chain per stage
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t g = 0;  // chain counter across tiles: buffer g & 1, phase (g >> 1) & 1
      bool ok = true;
      int nfill = 0;
      const uint64_t desc0 = smem_desc(smem_u32(smem), 16, 1024, 2);  // stage 0, plane 0
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const RouterTile rt = router_tile(args, RBN, t);
        const int row0 = rt.row0;
        const int n_mma = (min(RBN, args.T - row0) + 15) & ~15;
        const uint32_t idesc = idesc_bf16(128, n_mma);
        for (int c = rt.c0; c < rt.c1; ++c, ++g) {
          const uint32_t b = g & 1, pph = (g >> 1) & 1;
          ok = mbar_wait(smem_u32(pempty + b), pph ^ 1, args.status, abort_flag);
          if (!ok) break;
          ok = mbar_wait(smem_u32(full_bar + stage), phase, args.status, abort_flag);
          if (!ok) break;
          ++nfill;
          tc_fence_after();
          const uint64_t a_desc = desc0 + (uint64_t)((stage * C::STAGE_BYTES) >> 4);
          const uint64_t b_desc = a_desc + (uint64_t)(C::A_BYTES >> 4);
          const uint32_t d_tmem = tmem_base + b * RBN;
#pragma unroll
          for (int p = 0; p < 3; ++p)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_bf16(d_tmem, a_desc + (uint64_t)((p * C::A_PLANE + 32 * j) >> 4), b_desc + (uint64_t)((32 * j) >> 4),
                       idesc, (p | j) ? 1u : 0u);
          tc_commit(smem_u32(empty_bar + stage));
          tc_commit(smem_u32(pfull + b));
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // every MMA this thread issued finishes before TMEM is released
      tc_commit(smem_u32(drain_bar));
      mbar_wait_drain(smem_u32(drain_bar), 0);
      fills[1] = nfill;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- drain + store
    const int q = warp & 3, cs = (warp - 2) >> 2;  // lane quarter, column half
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint32_t g = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      const RouterTile rt = router_tile(args, RBN, t);
      const int mt = rt.mt, row0 = rt.row0;
      const int n_valid = min(RBN, args.T - row0);
      const int nchunks = ((n_valid + 15) & ~15) >> 4;
      constexpr int MYCH = RBN / 32;  // this warp's chunks of 16 columns: cs*MYCH .. cs*MYCH+MYCH-1
      float accv[MYCH][16];
#pragma unroll
      for (int i = 0; i < MYCH; ++i)
#pragma unroll
        for (int j = 0; j < 16; ++j) accv[i][j] = 0.0f;
      for (int c = rt.c0; c < rt.c1; ++c, ++g) {
        const uint32_t b = g & 1, pph = (g >> 1) & 1;
        if (lane == 0) ok = mbar_wait(smem_u32(pfull + b), pph, args.status, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        tc_fence_after();
        // all of this warp's chunks in flight, one wait: the drain keeps pace with the
        // 12-MMA chain that refills the other buffer
        uint32_t r[MYCH][16];
#pragma unroll
        for (int i = 0; i < MYCH; ++i)
          if (cs * MYCH + i < nchunks) tmem_ld16(tmem_base + lane_off + b * RBN + (cs * MYCH + i) * 16, r[i]);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < MYCH; ++i)
          if (cs * MYCH + i < nchunks)
#pragma unroll
            for (int j = 0; j < 16; ++j) accv[i][j] += __uint_as_float(r[i][j]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(pempty + b));
      }
      if (!ok) break;
      const int e = mt * 128 + q * 32 + lane;
      const bool split = args.ksplit > 1;
      if (e < args.E) {
        const float bias = (!split && args.bias) ? __ldg(args.bias + e) : 0.0f;
        float* out = split ? args.zpart + (size_t)rt.split * args.T * args.E : args.z;
#pragma unroll
        for (int i = 0; i < MYCH; ++i)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = (cs * MYCH + i) * 16 + j;
            if (n < n_valid) out[(size_t)(row0 + n) * args.E + e] = split ? accv[i][j] : accv[i][j] + bias;
          }
      }
    }
  }

  __syncthreads();
  if (*abort_flag) {
    // a role gave up: the loads already issued land before the CTA exits
    if (threadIdx.x == 0) drain_ring(full_bar, STAGES, fills, 1, fills[1]);
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace moe
