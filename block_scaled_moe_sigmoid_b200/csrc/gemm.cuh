// Persistent, warp-specialised grouped GEMM on the 5th-generation tensor cores (sm_100a).
//
// Computes, per tile, D = A_tile * B_tile^T where
//   A = weight rows (output channels, K-major), 256 rows per tile as two 128-row halves
//   B = token rows (K-major), up to BN_MAX rows per tile (the MMA's N dimension)
// so the accumulator's TMEM lane is the output channel and its column is the token
// ("swap-AB": a Kimi-K3 expert sees ~146 tokens at T=8192, which fits one N tile
// while the weights fill the 128-row M dimension).
//
// Kinds:
//   KIND_MX:   tcgen05.mma kind::mxf8f6f4.block_scale, A = E2M1 (MXFP4 weights, loaded by
//              TMA with the 16U4_ALIGN16B unpacking type), B = E4M3 (MXFP8 activations),
//              one E8M0 scale per 32 K-elements on both sides, fp32 accumulation.  The
//              weights are stored tile-major, [group][m-tile][k-tile][256 rows][64 B], so
//              each stage's weight tile is one contiguous 16 KB block in HBM.
//   KIND_BF16: tcgen05.mma kind::f16 with bf16 A and B, fp32 accumulation.
//
// Groups: rows of B are grouped (one group per expert, contiguous rows
// [offsets[g], offsets[g+1])); each group is split into ceil(rows / BN_MAX) tiles of
// balanced size.  "dense" mode is one implicit group of dense_rows rows.  Tile t
// covers group-tile t / m_tiles and weight m-tile t % m_tiles, so CTAs running at the
// same time share the group's B rows through L2.
//
// Roles (384 threads): warp 0 loads the weight tiles (TMA, plus a bulk copy of their
// scales), warp 10 loads the token rows (one TMA box, plus a bulk copy of their scales),
// warp 11 copies each stage's scale factors into TMEM (KIND_MX), warp 1 owns TMEM and one
// lane issues the MMAs, one or two K tiles per round, warps 2..9 run the epilogue (lane quarter =
// warp % 4).  The producers and the scale warp complete the same stage independently.
//
// Orientation WN (KIND_MX, a few tokens per expert): the token rows are the MMA's M side
// (128 lanes, of which the tile's rows are the first n) and all 256 weight rows of the tile
// are its N side, so each K block is one M=128 x N=256 instruction instead of two M=128 x
// N=n ones.  Issued back to back from one thread, a block-scaled M=128 x N x K=32
// tcgen05.mma takes max(~51, N/2) cycles (the N/2 is the FP8 rate; ~51 is the issue floor
// of one thread), so with few tokens one N=256 instruction (128 cycles) replaces two
// floor-bound ones (~102).  Measured, it is slower all the same (fewer pipeline stages fit);
// it stays selectable.
// The accumulator is then tokens x (gate | up) or tokens x output channels; the epilogue
// reads a token row per thread.  Shared memory, producers and scale copies are as above
// (the weight scales become the B side's, the token scales the A side's).
#pragma once
#include "ptx.cuh"
#include "tiling.cuh"

namespace moe {

enum { KIND_MX = 0, KIND_BF16 = 1 };
enum {
  EPI_GLU_MX8 = 0,          // a = silu(gate) * up, requantised to MXFP8 along the channels
  EPI_GLU_BF16 = 1,         // a = silu(gate) * up, stored as bf16
  EPI_BF16 = 2,             // D stored as bf16
  EPI_F32 = 3,              // D stored as fp32
  EPI_GLU_MX8_CLAMPED = 4,  // as EPI_GLU_MX8 with the clamped SwiGLU (glu_f<1>)
  EPI_GLU_BF16_CLAMPED = 5  // as EPI_GLU_BF16 with the clamped SwiGLU
};
template <int EPI>
struct EpiTraits {
  static constexpr bool glu = EPI == EPI_GLU_MX8 || EPI == EPI_GLU_BF16 || EPI == EPI_GLU_MX8_CLAMPED ||
                              EPI == EPI_GLU_BF16_CLAMPED;
  static constexpr bool mx8_out = EPI == EPI_GLU_MX8 || EPI == EPI_GLU_MX8_CLAMPED;
  static constexpr int act = (EPI == EPI_GLU_MX8_CLAMPED || EPI == EPI_GLU_BF16_CLAMPED) ? 1 : 0;
};

struct GemmArgs {
  const int* counts;       // [G] rows per group (routed mode)
  const int* offsets;      // [G+1] first row of each group
  const int* tile_prefix;  // [G+1] first group-tile of each group
  int num_groups;
  int dense_rows;   // >= 0: one implicit group with this many rows (no group arrays)
  int M_total;      // A rows per group (output channels)
  int m_tiles;      // ceil(M_total / 256)
  int k_tiles;      // K / BK
  int kb_wrap;      // B's K-tile coordinate is taken modulo kb_wrap
  int B_rows;       // rows of the B tensor
  const uint8_t* sfa;   // KIND_MX: A scales, [G][m_tiles][k_tiles][2 halves][512 B atom]
  const uint8_t* sfb;   // KIND_MX: B scales, tile-major [group-tiles][k_tiles][1 KB] (tiling.cuh)
  void* out0;
  void* out1;
  int ld_out;           // elements per output row
  unsigned int* status;
  int pf_dist;          // L2 prefetch distance in k-tiles (0 = off), KIND_MX weights
  int pf_b;             // reserved
  const uint8_t* a_ptr; // KIND_MX: packed weights (base of the tile-major code array)
  // Split K (dense mode with EPI_F32 only): tiles also walk ksplit ranges of k_per K tiles,
  // and split s writes its fp32 partial at out0 + s * split_stride elements.
  int ksplit;
  int k_per;
  long long split_stride;
};

template <int KIND, int BN_MAX, int STAGES, bool WN = false>
struct GemmCfg {
  static constexpr int BM = 256;                               // two 128-row halves
  static constexpr int BK = KIND == KIND_MX ? 128 : 64;        // elements per K tile (128 B rows)
  static constexpr int A_BYTES = BM * 128;                     // smem (FP4 padded to 1 B/elem)
  static constexpr int B_BYTES = BN_MAX * 128;
  static constexpr int SFA_BYTES = KIND == KIND_MX ? 1024 : 0;   // two 512 B atoms
  static constexpr int SFB_ATOMS = (BN_MAX + 127) / 128;
  static constexpr int SFB_BYTES = KIND == KIND_MX ? SFB_ATOMS * 512 : 0;
  // Shared memory: the stages' A and B tiles (1024-byte aligned for the swizzled layouts),
  // then every stage's scale atoms, then the control block.  Keeping the small scale atoms
  // out of the tile stride lets the 32-row configuration hold six stages.
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;
  static constexpr int SF_OFFSET = STAGES * STAGE_BYTES;
  static constexpr int CTRL_OFFSET = SF_OFFSET + STAGES * SF_STAGE_BYTES;
  static constexpr int A_TX = KIND == KIND_MX ? BM * BK / 2 : BM * BK * 2;  // global bytes
  static constexpr int SMEM_BYTES = CTRL_OFFSET + 1024 /*barriers*/ + 1024 /*align*/;
  // scale factors in TMEM, one 16-column buffer per pipeline stage:
  //   weights: 4 columns per 128-row half (+0, +4), tokens: 4 columns per 128 rows (+8, +12)
  // after the accumulator buffers (each two halves of BN_MAX columns, or WN: 256 columns)
  static constexpr int TMEM_COLS = 512;
  // Two accumulator buffers where TMEM holds them next to the scale buffers (the 32-row
  // configuration): the MMAs of a tile then run while the epilogue drains the previous one.
  static constexpr int ACC_BUFS = !WN && 4 * BN_MAX + 16 * STAGES <= TMEM_COLS ? 2 : 1;
  static constexpr int ACC_COLS = 2 * BN_MAX;
  static constexpr int TMEM_SF = WN ? 256 : ACC_BUFS * ACC_COLS;
  static constexpr int NUM_THREADS = 384;
  static_assert(BN_MAX % 16 == 0 && BN_MAX <= 256, "BN_MAX");
  static_assert(SFB_ATOMS <= 2, "scale buffer holds two B atoms");
  static_assert(TMEM_SF + 16 * STAGES <= TMEM_COLS, "TMEM budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SF_STAGE_BYTES % 128 == 0, "scale atom alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // WN: the M=128 MMA reads 128 token rows (16 KB) from the token region whatever the
  // tile's row count, so the region must hold 128 rows (rows past the tile's are stale and
  // only reach accumulator lanes that nothing reads)
  static_assert(!WN || (KIND == KIND_MX && BN_MAX == 128), "WN: block-scaled, a 128-row token region");
};

struct TileInfo {
  int grp, gt, mt, row0, n_valid, n_mma;  // gt: group-tile index
  int split, kb, ke;                       // K split and its K-tile range [kb, ke)
};

__device__ __forceinline__ int gemm_num_tiles(const GemmArgs& a, int bn_max) {
  if (a.dense_rows >= 0) return ((a.dense_rows + bn_max - 1) / bn_max) * a.m_tiles * a.ksplit;
  return __ldg(a.tile_prefix + a.num_groups) * a.m_tiles;
}

__device__ __forceinline__ void gemm_decode_tile(const GemmArgs& a, int bn_max, int t, TileInfo& ti) {
  ti.split = 0;
  ti.kb = 0;
  ti.ke = a.k_tiles;
  if (a.dense_rows >= 0 && a.ksplit > 1) {   // the split is the slowest index of t
    const int per_split = ((a.dense_rows + bn_max - 1) / bn_max) * a.m_tiles;
    ti.split = t / per_split;
    t -= ti.split * per_split;
    ti.kb = ti.split * a.k_per;
    ti.ke = min(a.k_tiles, ti.kb + a.k_per);
  }
  const int gt = t / a.m_tiles;
  ti.mt = t - gt * a.m_tiles;
  int grp, nt, ntiles, Me, base;
  if (a.dense_rows >= 0) {
    grp = 0;
    nt = gt;
    Me = a.dense_rows;
    ntiles = (Me + bn_max - 1) / bn_max;
    base = 0;
  } else {
    int lo = 0, hi = a.num_groups - 1;  // last group whose first tile is <= gt
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(a.tile_prefix + mid) <= gt) lo = mid; else hi = mid - 1;
    }
    grp = lo;
    const int tp = __ldg(a.tile_prefix + grp);
    nt = gt - tp;
    ntiles = __ldg(a.tile_prefix + grp + 1) - tp;
    Me = __ldg(a.counts + grp);
    base = __ldg(a.offsets + grp);
  }
  const int n_per = tile_rows_per(Me, ntiles);
  ti.grp = grp;
  ti.gt = gt;
  ti.row0 = base + nt * n_per;
  ti.n_valid = min(n_per, Me - nt * n_per);
  ti.n_mma = (ti.n_valid + 15) & ~15;
}

__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }
// a = glu(g, u): ACT 0 SiLU-GLU; ACT 1 clamped SwiGLU, (clamp(u, -7, 7) + 1) * g_c *
// sigmoid(1.702 g_c) with g_c = min(g, 7)
template <int ACT>
__device__ __forceinline__ float glu_f(float g, float u);

// Split-K partials of a gate/up product, rows interleaved in 128-channel blocks (gate
// block, up block, ...): h[t][c] = bf16(glu(sum_s g, sum_s u)), sums in split order.
template <int ACT>
__global__ void split_glu_reduce_kernel(const float* __restrict__ part, int nsplit, int T, int I,
                                        long long split_stride, __nv_bfloat16* __restrict__ h) {
  griddep_wait();
  griddep_launch_dependents();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)T * I) return;
  const int t = (int)(i / I), c = (int)(i - (long long)t * I);
  const size_t gcol = (size_t)256 * (c >> 7) + (c & 127);
  const float* row = part + (size_t)t * 2 * I;
  float g = 0.0f, u = 0.0f;
  for (int sp = 0; sp < nsplit; ++sp) {
    g += __ldg(row + sp * split_stride + gcol);
    u += __ldg(row + sp * split_stride + gcol + 128);
  }
  h[i] = __float2bfloat16_rn(glu_f<ACT>(g, u));
}

// out[i] = sum over s, in order, of part[s * split_stride + i].
__global__ void split_sum_kernel(const float* __restrict__ part, int nsplit, long long n, long long split_stride,
                                 float* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float v = 0.0f;
  for (int sp = 0; sp < nsplit; ++sp) v += __ldg(part + sp * split_stride + i);
  out[i] = v;
}

template <int ACT>
__device__ __forceinline__ float glu_f(float g, float u) {
  if constexpr (ACT == 0) {
    return silu_f(g) * u;
  } else {
    const float gc = fminf(g, 7.0f);
    const float uc = fminf(fmaxf(u, -7.0f), 7.0f);
    return (uc + 1.0f) * __fdividef(gc, 1.0f + __expf(-1.702f * gc));
  }
}

// MXFP8 (E4M3) encoding of v with block scale exponent from the block's amax bits.
__device__ __forceinline__ int mx_exp_e4m3(uint32_t amax_bits) {
  const int ex = (int)((amax_bits >> 23) & 0xFF);
  const int e = (ex == 0) ? -127 : ex - 127 - 8;   // floor(log2 amax) - emax(E4M3)
  return max(e, -127);
}
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Token-row tensor maps with box heights 16, 32, ..., 16 * MAX_BOX rows (one per MMA N).
constexpr int BOX_ROWS = 16;
constexpr int MAX_BOX = 16;
struct BMaps {
  CUtensorMap box[MAX_BOX];
};

// Swap-AB epilogue of one tile (accumulator lanes = output channels, columns = tokens):
// warps 2..9, lane quarter q, column half `sub`.  release_tmem() hands the accumulator back
// to the MMA issuer as soon as this warp has read what it needs.
template <int KIND, int EPI, int BN_MAX, class Release>
__device__ __forceinline__ void epilogue_swapab(const GemmArgs& args, const TileInfo& ti, uint32_t lane_base, int q,
                                                int sub, int lane, Release&& release_tmem) {
  const int nchunks = ti.n_mma >> 4;
  constexpr int CH = BN_MAX / 16;
  if constexpr (EpiTraits<EPI>::glu) {
    // a = glu(g, u) for this warp's chunks (c = sub + 2 i) straight out of TMEM;
    // TMEM goes back to the MMA warp before the quantisation and stores.
    constexpr int CH2 = (CH + 1) / 2;   // this warp's chunks: c = sub + 2 i
    float a[CH2][16];
#pragma unroll
    for (int i = 0; i < CH2; ++i) {
      const int c = sub + 2 * i;
      if (c < nchunks) {
        uint32_t g[16], u[16];
        tmem_ld16(lane_base + c * 16, g);
        tmem_ld16(lane_base + BN_MAX + c * 16, u);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) a[i][j] = glu_f<EpiTraits<EPI>::act>(__uint_as_float(g[j]), __uint_as_float(u[j]));
      }
    }
    release_tmem();
    const int ch = ti.mt * 128 + q * 32 + lane;  // intermediate channel
#pragma unroll
    for (int i = 0; i < CH2; ++i) {
      const int c = sub + 2 * i;
      if (c >= nchunks) break;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int n = c * 16 + j;
        if (n >= ti.n_valid) break;
        const size_t row = (size_t)(ti.row0 + n);
        if constexpr (EpiTraits<EPI>::mx8_out) {
          const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(a[i][j]) & 0x7FFFFFFFu);
          const int e = mx_exp_e4m3(amax);
          const float qv = a[i][j] * __uint_as_float((uint32_t)(127 - e) << 23);
          const uint32_t code = f32x2_to_e4m3x2(qv, 0.0f) & 0xFFu;
          ((uint8_t*)args.out0)[row * args.ld_out + ch] = (uint8_t)code;
          if (lane == 0)   // scale byte for the down GEMM: K tile mt, block q, tile-major
            ((uint8_t*)args.out1)[((size_t)ti.gt * args.m_tiles + ti.mt) * SF_TILE_BYTES +
                                  sf_atom_offset(n) + q] = (uint8_t)(e + 127);
        } else {
          ((__nv_bfloat16*)args.out0)[row * args.ld_out + ch] = __float2bfloat16_rn(a[i][j]);
        }
      }
    }
  } else if constexpr (EPI == EPI_BF16) {
    // round to bf16 pairs while draining TMEM, release it, then store
    const int h = sub;
    const bool half_ok = ti.mt * 256 + h * 128 < args.M_total;
    uint32_t v[CH][8];
    if (half_ok) {
#pragma unroll
      for (int c = 0; c < CH; ++c)
        if (c < nchunks) {
          uint32_t r[16];
          tmem_ld16(lane_base + h * BN_MAX + c * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const __nv_bfloat162 p2 =
                __floats2bfloat162_rn(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
            v[c][j] = *(const uint32_t*)&p2;
          }
        }
    }
    release_tmem();
    const int ch = ti.mt * 256 + h * 128 + q * 32 + lane;  // output channel
    if (half_ok && ch < args.M_total) {
      uint16_t* out = (uint16_t*)args.out0;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        if (c >= nchunks) break;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c * 16 + j;
          if (n >= ti.n_valid) break;
          out[(size_t)(ti.row0 + n) * args.ld_out + ch] = (uint16_t)(v[c][j >> 1] >> ((j & 1) * 16));
        }
      }
    }
  } else {
    // fp32 results: store straight from TMEM chunk by chunk, release at the end
    const int h = sub;
    const int ch = ti.mt * 256 + h * 128 + q * 32 + lane;  // output channel
    const bool half_ok = ti.mt * 256 + h * 128 < args.M_total;
    if (half_ok) {
      const bool ch_ok = ch < args.M_total;
      for (int c = 0; c < nchunks; ++c) {
        uint32_t v[16];
        tmem_ld16(lane_base + h * BN_MAX + c * 16, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c * 16 + j;
          if (n >= ti.n_valid) break;
          if (!ch_ok) continue;
          ((float*)args.out0)[(size_t)ti.split * args.split_stride + (size_t)(ti.row0 + n) * args.ld_out + ch] =
              __uint_as_float(v[j]);
        }
      }
    }
    release_tmem();
  }
}

template <int KIND, int EPI, int BN_MAX, int STAGES, bool WN = false>
__global__ void __launch_bounds__(384, 1)
    gemm_kernel(const __grid_constant__ GemmArgs args, const __grid_constant__ CUtensorMap tmA,
                const __grid_constant__ BMaps tmB) {
  using C = GemmCfg<KIND, BN_MAX, STAGES, WN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ctrl = smem + C::CTRL_OFFSET;
  uint64_t* full_bar = (uint64_t*)ctrl;
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* sf_full = empty_bar + STAGES;        // scale blocks of the stage are in smem
  uint64_t* acc_full = sf_full + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain_bar = acc_empty + 2;
  uint64_t* drain_sf = drain_bar + 1;
  uint32_t* tmem_holder = (uint32_t*)(drain_sf + 1);
  volatile int* abort_flag = (volatile int*)(tmem_holder + 1);
  // Fill counters for the abort cleanup: [0] weight producer, [1] token producer, [2] scale
  // warp (sf_full fills consumed = full-barrier arrivals made), [3] MMA (fills consumed).
  int* fills = (int*)(tmem_holder + 2);
  // MMA N of the tile a stage belongs to, written by the token producer before it arrives
  // on the stage's full barrier (so the MMA thread never decodes routed tiles itself: that
  // takes dependent global loads, a binary search over the expert tile table)
  int* stage_n = fills + 4;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // one arrival per producer warp, plus (KIND_MX) the scale warp's commit once the
      // stage's scale factors are in TMEM: a full stage is ready for the MMAs as it stands
      mbar_init(smem_u32(full_bar + s), KIND == KIND_MX ? 3 : 2);
      mbar_init(smem_u32(empty_bar + s), 1);
      mbar_init(smem_u32(sf_full + s), 2);   // weight-scale and token-scale copies
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(acc_full + b), 1);
      mbar_init(smem_u32(acc_empty + b), 8);
    }
    mbar_init(smem_u32(drain_bar), 1);
    mbar_init(smem_u32(drain_sf), 1);
    *abort_flag = 0;
    for (int r = 0; r < 4; ++r) fills[r] = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
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

  const int num_tiles = gemm_num_tiles(args, BN_MAX);

  if (warp == 0) {
    // ------------------------------------------------------------- producer: weights
    // One TMA box of 256 weight rows x one K tile, plus (KIND_MX) a 1 KB bulk copy of
    // the matching scale-factor atoms.
    const uint64_t pol_a = policy_evict_first();  // weights stream through once
    int stage = 0;
    uint32_t phase = 0;
    // L2 prefetch cursor, pf_dist k-tiles ahead of the loads along the (tile, k) sequence.
    int pf_t = args.pf_dist > 0 ? (int)blockIdx.x : num_tiles, pf_kt = 0;
    TileInfo pf;
    if (pf_t < num_tiles) gemm_decode_tile(args, BN_MAX, pf_t, pf);
    auto prefetch_one = [&]() {
      if (pf_t >= num_tiles) return;
      if constexpr (KIND == KIND_MX) {
        // the 16 KB weight tile is contiguous: 128 lines of 128 B, 4 per lane
        const uint8_t* tile = args.a_ptr + (((size_t)pf.grp * args.m_tiles + pf.mt) * args.k_tiles + pf_kt) * (C::BM * 64);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(tile + (i * 32 + lane) * 128));
      }
      if (++pf_kt == args.k_tiles) {
        pf_kt = 0;
        pf_t += gridDim.x;
        if (pf_t < num_tiles) gemm_decode_tile(args, BN_MAX, pf_t, pf);
      }
    };
    for (int i = 0; i < args.pf_dist; ++i) prefetch_one();
    bool ok = true;
    int nfill = 0;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      TileInfo ti;
      gemm_decode_tile(args, BN_MAX, t, ti);
      const int a_row = ti.grp * args.M_total + ti.mt * C::BM;
      for (int kt = ti.kb; kt < ti.ke; ++kt) {
        if (lane == 0) {
          ok = mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, args.status, abort_flag);
          if (ok) {
            uint8_t* sA = smem + stage * C::STAGE_BYTES;
            const uint32_t fb = smem_u32(full_bar + stage);
            if constexpr (KIND == KIND_MX) {
              // the scale atoms first: the scale warp's copies into TMEM then run while the
              // large tile is still landing
              const uint32_t sb = smem_u32(sf_full + stage);
              mbar_arrive_expect_tx(sb, C::SFA_BYTES);
              const uint8_t* sfa_src =
                  args.sfa + (((size_t)ti.grp * args.m_tiles + ti.mt) * args.k_tiles + kt) * 1024;
              asm volatile(
                  "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], 1024, [%2];" ::
                      "r"(smem_u32(smem + C::SF_OFFSET + stage * C::SF_STAGE_BYTES)),
                  "l"(sfa_src), "r"(sb)
                  : "memory");
            }
            mbar_arrive_expect_tx(fb, C::A_TX);
            if constexpr (KIND == KIND_MX)   // tile-major weights: one contiguous 16 KB block
              tma_load_2d(smem_u32(sA), &tmA, fb, 0, ((ti.grp * args.m_tiles + ti.mt) * args.k_tiles + kt) * C::BM, pol_a);
            else
              tma_load_2d(smem_u32(sA), &tmA, fb, kt * C::BK, a_row, pol_a);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++nfill;
        prefetch_one();
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (lane == 0) fills[0] = nfill;
  } else if (warp == 10) {
    // ------------------------------------------------------------- producer: token rows
    // One TMA box of the tile's n_mma rows (a multiple of 16: box height 16 * nB) and
    // (KIND_MX) one bulk copy of the tile's scale atoms for this K tile.
    const uint64_t pol_b = policy_evict_last();   // token rows are shared by the m-tiles
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int nfill = 0;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      TileInfo ti;
      gemm_decode_tile(args, BN_MAX, t, ti);
      const int nB = ti.n_mma / BOX_ROWS;
      for (int kt = ti.kb; kt < ti.ke; ++kt) {
        if (lane == 0) ok = mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, args.status, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        uint8_t* sB = smem + stage * C::STAGE_BYTES + C::A_BYTES;
        const uint32_t fb = smem_u32(full_bar + stage);
        if (lane == 0) {
          stage_n[stage] = ti.n_mma;
          if constexpr (KIND == KIND_MX) {
            const int sfb_bytes = ((ti.n_mma + 127) >> 7) * 512;
            const uint32_t sb = smem_u32(sf_full + stage);
            mbar_arrive_expect_tx(sb, sfb_bytes);
            const uint8_t* src = args.sfb + ((size_t)ti.gt * args.k_tiles + kt) * SF_TILE_BYTES;
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
                    "r"(smem_u32(smem + C::SF_OFFSET + stage * C::SF_STAGE_BYTES + C::SFA_BYTES)),
                "l"(src), "r"(sfb_bytes), "r"(sb)
                : "memory");
          }
          mbar_arrive_expect_tx(fb, nB * BOX_ROWS * 128);
          tma_load_2d(smem_u32(sB), &tmB.box[nB - 1], fb, (kt % args.kb_wrap) * C::BK, ti.row0, pol_b);
        }
        __syncwarp();
        ++nfill;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (lane == 0) fills[1] = nfill;
  } else if (warp == 11) {
    // ------------------------------------------------------------- scale factors -> TMEM
    // tcgen05.cp of each stage's scale atoms into that stage's TMEM buffer, off the MMA
    // thread's instruction stream, as soon as the small scale blocks land (their own
    // barrier, ahead of the large tiles).  The copies' commit is the third arrival on the
    // stage's full barrier.  A buffer is rewritten only after the stage was released for
    // refilling, i.e. after the MMAs that read it committed.
    if (KIND == KIND_MX && lane == 0) {
      // no-swizzle descriptor of stage 0's A scale atoms (32 rows x 16 B, 128 B per 8 rows)
      const uint64_t sf_desc0 = smem_desc(smem_u32(smem) + C::SF_OFFSET, 16, 128, 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int nfill = 0;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        TileInfo ti;
        gemm_decode_tile(args, BN_MAX, t, ti);
        const bool h1 = ti.mt * C::BM + 128 < args.M_total;
        const int atoms = (ti.n_mma + 127) >> 7;
        for (int kt = ti.kb; kt < ti.ke; ++kt) {
          ok = mbar_wait(smem_u32(sf_full + stage), phase, args.status, abort_flag);
          if (!ok) break;
          ++nfill;
          tc_fence_after();
          const uint64_t sfa_desc = sf_desc0 + (uint64_t)((stage * C::SF_STAGE_BYTES) >> 4);
          const uint64_t sfb_desc = sfa_desc + (uint64_t)(C::SFA_BYTES >> 4);
          const uint32_t tsf = tmem_base + C::TMEM_SF + 16 * stage;
          tc_cp_32x128b_warpx4(tsf, sfa_desc);
          if (h1 || WN) tc_cp_32x128b_warpx4(tsf + 4, sfa_desc + (uint64_t)(512 >> 4));
          tc_cp_32x128b_warpx4(tsf + 8, sfb_desc);
          if (atoms > 1) tc_cp_32x128b_warpx4(tsf + 12, sfb_desc + (uint64_t)(512 >> 4));
          tc_commit(smem_u32(full_bar + stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // every scale copy this warp issued lands before TMEM is released
      tc_commit(smem_u32(drain_sf));
      mbar_wait_drain(smem_u32(drain_sf), 0);
      fills[2] = nfill;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // 128-byte-swizzled K-major descriptor of stage 0's A tile; other tiles are offsets
      const uint64_t desc0 = smem_desc(smem_u32(smem), 16, 1024, 2);
      int stage = 0;
      uint32_t phase = 0;
      int tcount = 0;
      bool ok = true;
      int nfill = 0;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        // The tile's K range and weight m-tile are arithmetic; its MMA N comes with its
        // first stage (stage_n, below).
        TileInfo ti;
        if (args.dense_rows >= 0) {
          gemm_decode_tile(args, BN_MAX, t, ti);
        } else {
          ti.mt = t % args.m_tiles;
          ti.kb = 0;
          ti.ke = args.k_tiles;
        }
        const bool h1 = ti.mt * C::BM + 128 < args.M_total;
        uint32_t idesc[4];
        bool first = true;
        // this CTA's tile count picks the accumulator buffer and its barrier phase
        const int abuf = tcount % C::ACC_BUFS;
        const uint32_t acc_phase = (uint32_t)(tcount / C::ACC_BUFS) & 1u;
        const uint32_t acc_t = tmem_base + (uint32_t)(abuf * C::ACC_COLS);
        // the MMAs of the K tile held by smem stage st: 4 K-blocks x 2 halves (WN: 4 K-blocks)
        auto issue_stage = [&](int st, uint32_t acc0) {
          const uint64_t a_desc = desc0 + (uint64_t)((st * C::STAGE_BYTES) >> 4);
          const uint64_t b_desc = a_desc + (uint64_t)(C::A_BYTES >> 4);
          const uint32_t tsf = tmem_base + C::TMEM_SF + 16 * st;
          if constexpr (WN) {
            // token tile (A, M=128) x all 256 weight rows (B, N=256), one MMA per K block
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_mxf8f6f4(acc_t, b_desc + (uint64_t)((32 * j) >> 4), a_desc + (uint64_t)((32 * j) >> 4), idesc[j],
                           (tsf + 8) | ((uint32_t)j << 30), tsf | ((uint32_t)j << 30), j > 0 ? 1u : acc0);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                if (h == 1 && !h1) continue;
                const uint64_t adesc = a_desc + (uint64_t)((h * 16384 + 32 * j) >> 4);
                const uint64_t bdesc = b_desc + (uint64_t)((32 * j) >> 4);
                const uint32_t acc = j > 0 ? 1u : acc0;
                if constexpr (KIND == KIND_MX)
                  mma_mxf8f6f4(acc_t + h * BN_MAX, adesc, bdesc, idesc[j], (tsf + 4 * h) | ((uint32_t)j << 30),
                               (tsf + 8) | ((uint32_t)j << 30), acc);
                else
                  mma_bf16(acc_t + h * BN_MAX, adesc, bdesc, idesc[j], acc);
              }
            }
          }
        };
        // One or two K tiles per round: after the blocking wait for this stage, the next
        // stage's barrier is tested once without waiting; if it has landed too, both
        // stages' 16 MMAs are issued in one run.  Each mbarrier wait costs the issuing
        // thread about as much as one or two MMAs, so pairing landed stages halves that
        // overhead, while a stage is never held back waiting for its successor to land
        // (which would keep its slot, and the loads it could make room for, waiting).
        // Each stage is released as soon as its own MMAs commit.
        for (int kt = ti.kb; kt < ti.ke;) {
          const int kt0 = kt;
          const int stage2 = stage + 1 == STAGES ? 0 : stage + 1;
          const uint32_t phase2 = stage + 1 == STAGES ? phase ^ 1u : phase;
          ok = mbar_wait(smem_u32(full_bar + stage), phase, args.status, abort_flag);
          if (ok) ++nfill;
          const bool two = ok && kt + 1 < ti.ke && mbar_try_wait(smem_u32(full_bar + stage2), phase2);
          if (two) ++nfill;
          kt += two ? 2 : 1;
          if (!ok) break;
          if (first) {
            // Everything the MMAs of a stage need except the stage offset is fixed per
            // tile: the issue loop only adds constants (the tcgen05.mma issue rate is set
            // by how fast this one thread can form its operands).
            const int n_mma = stage_n[stage];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              idesc[j] = WN ? idesc_mx_e4m3_e2m1(128, 256, j, j)
                            : (KIND == KIND_MX ? idesc_mx_e2m1_e4m3(128, n_mma, j, j) : idesc_bf16(128, n_mma));
            // the accumulator buffer is free once the epilogue has drained the tile that
            // last used it (the previous tile, or the one before with two buffers)
            ok = mbar_wait(smem_u32(acc_empty + abuf), acc_phase ^ 1, args.status, abort_flag);
            if (!ok) break;
            first = false;
          }
          tc_fence_after();
          issue_stage(stage, kt0 > ti.kb ? 1u : 0u);
          tc_commit(smem_u32(empty_bar + stage));
          if (two) {
            issue_stage(stage2, 1u);
            tc_commit(smem_u32(empty_bar + stage2));
          }
          stage = stage2;
          phase = phase2;
          if (two) {
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(acc_full + abuf));
        ++tcount;
      }
      // make sure every MMA this thread issued has finished before TMEM is released
      tc_commit(smem_u32(drain_bar));
      mbar_wait_drain(smem_u32(drain_bar), 0);
      fills[3] = nfill;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int sub = (warp - 2) >> 2;   // 0 or 1
    const uint32_t lane_base0 = tmem_base + ((uint32_t)(q * 32) << 16);
    int tcount = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      TileInfo ti;
      gemm_decode_tile(args, BN_MAX, t, ti);
      bool ok = true;
      const int abuf = tcount % C::ACC_BUFS;
      const uint32_t acc_phase = (uint32_t)(tcount / C::ACC_BUFS) & 1u;
      const uint32_t lane_base = lane_base0 + (uint32_t)(abuf * C::ACC_COLS);
      if (lane == 0) ok = mbar_wait(smem_u32(acc_full + abuf), acc_phase, args.status, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      auto release_tmem = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(acc_empty + abuf));
      };
      if constexpr (WN) {
        // TMEM lane = token row of the tile (quarter q: rows 32q..32q+31), column = weight
        // row of the tile.  tcgen05.ld is warp-wide, so a warp without valid rows only
        // releases TMEM.
        const int r = q * 32 + lane;
        const bool any = q * 32 < ti.n_valid;
        const bool row_ok = r < ti.n_valid;
        const size_t row = (size_t)(ti.row0 + r);
        if constexpr (EpiTraits<EPI>::glu) {
          // columns c < 128: gate of channel mt*128 + c; 128 + c: its up.  Warp half `sub`
          // takes the 32-channel blocks 2 sub and 2 sub + 1.
          float a[2][32];
          if (any) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int b = 2 * sub + i;
              uint32_t g0[16], g1[16], u0[16], u1[16];
              tmem_ld16(lane_base + 32 * b, g0);
              tmem_ld16(lane_base + 32 * b + 16, g1);
              tmem_ld16(lane_base + 128 + 32 * b, u0);
              tmem_ld16(lane_base + 128 + 32 * b + 16, u1);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                a[i][j] = glu_f<EpiTraits<EPI>::act>(__uint_as_float(g0[j]), __uint_as_float(u0[j]));
                a[i][16 + j] = glu_f<EpiTraits<EPI>::act>(__uint_as_float(g1[j]), __uint_as_float(u1[j]));
              }
            }
          }
          release_tmem();
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int b = 2 * sub + i;
              const size_t col = (size_t)ti.mt * 128 + 32 * b;
              if constexpr (EpiTraits<EPI>::mx8_out) {
                float amax = 0.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(a[i][j]));
                const int e = mx_exp_e4m3(__float_as_uint(amax));
                const float sc = __uint_as_float((uint32_t)(127 - e) << 23);
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  w[j] = f32x2_to_e4m3x2(a[i][4 * j] * sc, a[i][4 * j + 1] * sc) |
                         (f32x2_to_e4m3x2(a[i][4 * j + 2] * sc, a[i][4 * j + 3] * sc) << 16);
                uint4* dst = (uint4*)((uint8_t*)args.out0 + row * args.ld_out + col);
                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                // scale byte for the down GEMM: K tile mt, block b, tile-major
                ((uint8_t*)args.out1)[((size_t)ti.gt * args.m_tiles + ti.mt) * SF_TILE_BYTES + sf_atom_offset(r) + b] =
                    (uint8_t)(e + 127);
              } else {
                uint32_t w[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  const __nv_bfloat162 p2 = __floats2bfloat162_rn(a[i][2 * j], a[i][2 * j + 1]);
                  w[j] = *(const uint32_t*)&p2;
                }
                uint4* dst = (uint4*)((__nv_bfloat16*)args.out0 + row * args.ld_out + col);
#pragma unroll
                for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
              }
            }
          }
        } else {
          // output channels mt*256 + 128 sub + c, c < 128, rounded to bf16 (EPI_BF16)
          static_assert(EPI == EPI_BF16, "WN epilogues: GLU (MXFP8 / bf16) or bf16");
          const int ch0 = ti.mt * 256 + 128 * sub;
          const bool half_ok = ch0 < args.M_total;
          uint32_t v[64];
          if (any && half_ok) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t rr[16];
              tmem_ld16(lane_base + 128 * sub + 16 * c, rr);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const __nv_bfloat162 p2 = __floats2bfloat162_rn(__uint_as_float(rr[2 * j]), __uint_as_float(rr[2 * j + 1]));
                v[8 * c + j] = *(const uint32_t*)&p2;
              }
            }
          }
          release_tmem();
          if (half_ok && row_ok) {
            uint4* dst = (uint4*)((uint16_t*)args.out0 + row * args.ld_out + ch0);
#pragma unroll
            for (int i = 0; i < 16; ++i) dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      } else {
        epilogue_swapab<KIND, EPI, BN_MAX>(args, ti, lane_base, q, sub, lane, release_tmem);
      }
      ++tcount;

    }
  }

  __syncthreads();
  if (*abort_flag) {
    // A role gave up: let every copy still in flight into this CTA's shared memory land
    // (supplying the arrivals of the roles that stopped early) before the CTA exits.
    if (threadIdx.x == 0) {
      drain_ring(full_bar, STAGES, fills, KIND == KIND_MX ? 3 : 2, fills[3]);
      if constexpr (KIND == KIND_MX) drain_ring(sf_full, STAGES, fills, 2, fills[2]);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace moe
