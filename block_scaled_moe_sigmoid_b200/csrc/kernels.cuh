// CUDA-core kernels of the MoE layer: MXFP8 quantiser (plain and scatter-to-expert-order),
// token->expert histogram / scan / stable placement, sigmoid top-k selection,
// weighted combine, and the setup-time weight packers (MXFP4 experts, bf16 router planes).
#pragma once
#include "ptx.cuh"
#include "tiling.cuh"

namespace moe {

// ---------------------------------------------------------------- MX element conversion
// OCP MX block rule: scale exponent e = floor(log2(amax)) - emax, clamped below at -127;
// elements are round-to-nearest-even, saturating, sign kept (-0 stays -0).
__device__ __forceinline__ int mx_scale_exp(float amax, int emax) {
  const uint32_t b = __float_as_uint(amax);
  const int ex = (int)((b >> 23) & 0xFF);
  const int e = (ex == 0) ? -127 : ex - 127 - emax;  // subnormal or zero amax -> clamp
  return max(e, -127);
}
__device__ __forceinline__ float pow2_neg(int e) {  // 2^-e for e in [-127, 126]
  return __uint_as_float((uint32_t)(127 - e) << 23);
}
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}\n"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// One 32-element bf16 block -> 32 E4M3 bytes (as 8 words) + scale byte.
__device__ __forceinline__ uint32_t quant_block_e4m3(const uint4 (&in)[4], uint32_t (&out)[8]) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w[4] = {in[i].x, in[i].y, in[i].z, in[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[i * 8 + 2 * j] = __uint_as_float(w[j] << 16);
      v[i * 8 + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int e = mx_scale_exp(amax, 8);
  const float s = pow2_neg(e);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = cvt_e4m3x2(v[4 * i] * s, v[4 * i + 1] * s);
    const uint32_t hi = cvt_e4m3x2(v[4 * i + 2] * s, v[4 * i + 3] * s);
    out[i] = lo | (hi << 16);
  }
  return (uint32_t)(e + 127);
}

// x bf16 [rows][cols] -> q E4M3 [rows][cols], scale E8M0 [rows][cols/32].
__global__ void quant_mxfp8_kernel(const uint16_t* __restrict__ x, int rows, int cols,
                                   uint8_t* __restrict__ q, uint8_t* __restrict__ sc) {
  const int nb = cols >> 5;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)rows * nb) return;
  const long long r = gid / nb;
  const int b = (int)(gid - r * nb);
  const uint4* src = (const uint4*)(x + r * cols + b * 32);
  uint4 in[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) in[i] = __ldg(src + i);
  uint32_t out[8];
  const uint32_t s = quant_block_e4m3(in, out);
  uint4* dst = (uint4*)(q + r * cols + b * 32);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  sc[r * nb + b] = (uint8_t)s;
}

// Quantise token rows and write each to its k positions in expert order:
// xq[inv[t][j]][:] = E4M3 codes of x[t]; the block scales go once per token to
// xs_tok[t][cols/32] (scale_tiles_kernel turns them into the GEMM's tile-major blocks).
__global__ void quant_scatter_kernel(const uint16_t* __restrict__ x, int T, int cols, int k,
                                     const int* __restrict__ inv, int A_rows,
                                     uint8_t* __restrict__ xq, uint8_t* __restrict__ xs_tok) {
  griddep_wait();
  griddep_launch_dependents();
  const int nb = cols >> 5;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)T * nb) return;
  const long long t = gid / nb;
  const int b = (int)(gid - t * nb);
  const uint4* src = (const uint4*)(x + t * cols + b * 32);
  uint4 in[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) in[i] = __ldg(src + i);
  uint32_t out[8];
  xs_tok[gid] = (uint8_t)quant_block_e4m3(in, out);
  uint4 o0 = make_uint4(out[0], out[1], out[2], out[3]);
  uint4 o1 = make_uint4(out[4], out[5], out[6], out[7]);
  // When a warp's 32 blocks are one token's 1 KB run (cols % 1024 == 0, so that no warp
  // straddles two tokens), regroup the codes through shuffles so that each warp-wide store
  // writes 512 contiguous bytes: lane l stores bytes [16 l, 16 l + 16) and [512 + 16 l, ...)
  // of the run, i.e. half (l % 2) of blocks l / 2 and 16 + l / 2.  Otherwise lane l stores
  // its own block's 32 bytes.
  int boff0 = b * 32, boff1 = b * 32 + 16;
  if ((nb & 31) == 0) {
    const int lane = threadIdx.x & 31;
    const int s0 = lane >> 1, s1 = 16 + (lane >> 1);
    const bool hi = lane & 1;
    uint32_t a[4], c[4];
    const uint32_t w0[4] = {o0.x, o0.y, o0.z, o0.w}, w1[4] = {o1.x, o1.y, o1.z, o1.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t x0 = __shfl_sync(0xffffffffu, w0[i], s0), x1 = __shfl_sync(0xffffffffu, w1[i], s0);
      const uint32_t y0 = __shfl_sync(0xffffffffu, w0[i], s1), y1 = __shfl_sync(0xffffffffu, w1[i], s1);
      a[i] = hi ? x1 : x0;
      c[i] = hi ? y1 : y0;
    }
    o0 = make_uint4(a[0], a[1], a[2], a[3]);
    o1 = make_uint4(c[0], c[1], c[2], c[3]);
    const int b0 = b & ~31;   // first block of this warp's run
    boff0 = b0 * 32 + 16 * lane;
    boff1 = b0 * 32 + 512 + 16 * lane;
  }
  // four destinations at a time, so that their index loads overlap
  for (int j0 = 0; j0 < k; j0 += 4) {
    int pj[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) pj[q] = j0 + q < k ? __ldg(inv + t * k + j0 + q) : -1;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int p = pj[q];
      if (p < 0 || p >= A_rows) continue;
      uint8_t* row = xq + (size_t)p * cols;
      *(uint4*)(row + boff0) = o0;
      *(uint4*)(row + boff1) = o1;
    }
  }
}

// Token-side scale blocks of the gate/up GEMM, tile-major (tiling.cuh): one CTA per
// group-tile, one thread per row of the tile's scale atoms.  Row n of group-tile gt takes
// the four block scales of K tile kt of its token, xs_tok[perm_tok[row0 + n]][4 kt ..],
// as one word; rows past the tile's valid rows get zero scales.  Each CTA writes its
// k_tiles blocks whole, so no partial sectors reach DRAM.
__global__ void __launch_bounds__(256)
    scale_tiles_kernel(const uint8_t* __restrict__ xs_tok, int nb, const int* __restrict__ perm_tok,
                       const int* __restrict__ counts, const int* __restrict__ offsets,
                       const int* __restrict__ tile_prefix, int E, int k_tiles, uint8_t* __restrict__ xs) {
  griddep_wait();
  griddep_launch_dependents();
  const int gt = blockIdx.x;
  if (gt >= __ldg(tile_prefix + E)) return;
  int lo = 0, hi = E - 1;   // last group whose first tile is <= gt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(tile_prefix + mid) <= gt) lo = mid; else hi = mid - 1;
  }
  const int tp = __ldg(tile_prefix + lo);
  const int ntiles = __ldg(tile_prefix + lo + 1) - tp;
  const int rows = __ldg(counts + lo);
  const int n_per = tile_rows_per(rows, ntiles);
  const int nt = gt - tp;
  const int n_valid = min(n_per, rows - nt * n_per);
  const int atoms = (((n_valid + 15) & ~15) + 127) >> 7;
  const int n = threadIdx.x;
  if (n >= atoms * 128) return;
  const bool valid = n < n_valid;
  const uint8_t* src = xs_tok + (valid ? (size_t)__ldg(perm_tok + __ldg(offsets + lo) + nt * n_per + n) * nb : 0);
  uint8_t* dst = xs + (size_t)gt * k_tiles * SF_TILE_BYTES + sf_atom_offset(n);
  for (int kt = 0; kt < k_tiles; ++kt) {
    const uint32_t v = valid ? __ldg((const uint32_t*)(src + kt * 4)) : 0u;
    *(uint32_t*)(dst + (size_t)kt * SF_TILE_BYTES) = v;
  }
}

// ---------------------------------------------------------------- permutation
// Chunks of TPC tokens (32 per warp); chunk_counts[c][e] = assignments of chunk c to e.
__global__ void perm_histogram_kernel(const int* __restrict__ idx, int T, int k, int E,
                                      int tokens_per_chunk, int* __restrict__ chunk_counts,
                                      unsigned int* status) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ int cnt[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * tokens_per_chunk;
  const int n = min(tokens_per_chunk, T - t0) * k;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = __ldg(idx + (size_t)t0 * k + i);
    if (e < 0 || e >= E) {
      atomicOr(status, MOE_DEV_ERR_BOUNDS);
      continue;
    }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

// Block-wide exclusive scan of n <= 4 * blockDim.x values in place (1024 threads).
__device__ void block_exclusive_scan(int* vals, int n, int* warp_tot) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = threadIdx.x * per;
  int local = 0;
  for (int i = 0; i < per; ++i)
    if (i0 + i < n) local += vals[i0 + i];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    int v = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    warp_tot[lane] = inc - v;
  }
  __syncthreads();
  int run = warp_tot[w] + incl - local;
  for (int i = 0; i < per; ++i)
    if (i0 + i < n) {
      const int v = vals[i0 + i];
      vals[i0 + i] = run;
      run += v;
    }
  __syncthreads();
}

// Single CTA: counts, offsets (exclusive scan), per-chunk bases, and the GEMM tile prefix
// (ceil(count / bn_max) tiles per expert).
__global__ void perm_scan_kernel(int* __restrict__ chunk_counts, int nchunks, int E, int bn_max,
                                 int* __restrict__ counts, int* __restrict__ offsets,
                                 int* __restrict__ tile_prefix) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ int sh[];
  int* s_off = sh;            // E
  int* s_tiles = sh + E;      // E
  int* warp_tot = sh + 2 * E; // 32
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int c = 0; c < nchunks; ++c) {
      int* p = chunk_counts + (size_t)c * E + e;
      const int v = *p;
      *p = run;
      run += v;
    }
    counts[e] = run;
    s_off[e] = run;
    s_tiles[e] = (run + bn_max - 1) / bn_max;
  }
  __syncthreads();
  const int total_rows_last = s_off[E - 1];
  const int total_tiles_last = s_tiles[E - 1];
  __syncthreads();
  block_exclusive_scan(s_off, E, warp_tot);
  block_exclusive_scan(s_tiles, E, warp_tot);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    offsets[e] = s_off[e];
    tile_prefix[e] = s_tiles[e];
    for (int c = 0; c < nchunks; ++c) chunk_counts[(size_t)c * E + e] += s_off[e];
  }
  if (threadIdx.x == 0) {
    offsets[E] = s_off[E - 1] + total_rows_last;
    tile_prefix[E] = s_tiles[E - 1] + total_tiles_last;
  }
}

// Stable placement: position of (t, j) = base of (chunk, expert) + number of earlier
// tokens of the chunk that also chose that expert.  Warp w of a chunk owns tokens
// 32w..32w+31 and builds a per-expert lane mask; ranks come from popcounts.
__global__ void perm_place_kernel(const int* __restrict__ idx, int T, int k, int E,
                                  int tokens_per_chunk, const int* __restrict__ chunk_base,
                                  int* __restrict__ perm_tok, int* __restrict__ inv) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ uint32_t masks[];  // [warps][E]
  const int warps = blockDim.x >> 5;
  for (int i = threadIdx.x; i < warps * E; i += blockDim.x) masks[i] = 0;
  __syncthreads();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * tokens_per_chunk + threadIdx.x;
  const bool valid = threadIdx.x < tokens_per_chunk && t < T;
  if (valid)
    for (int j = 0; j < k; ++j) {
      const int e = __ldg(idx + (size_t)t * k + j);
      if (e >= 0 && e < E) atomicOr(&masks[w * E + e], 1u << lane);
    }
  __syncthreads();
  if (!valid) return;
  const uint32_t lt = (1u << lane) - 1u;
  const int* base = chunk_base + (size_t)blockIdx.x * E;
  for (int j = 0; j < k; ++j) {
    const int e = __ldg(idx + (size_t)t * k + j);
    if (e < 0 || e >= E) {
      inv[(size_t)t * k + j] = -1;
      continue;
    }
    int r = __popc(masks[w * E + e] & lt);
    for (int w2 = 0; w2 < w; ++w2) r += __popc(masks[w2 * E + e]);
    const int p = base[e] + r;
    inv[(size_t)t * k + j] = p;
    perm_tok[p] = t;
  }
}

// ---------------------------------------------------------------- top-k
// fp32 -> uint32 with the same order (negatives flipped whole, positives' sign bit set).
__device__ __forceinline__ uint32_t f32_order_key(float v) {
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float f32_from_order_key(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Top-k selection: the k largest keys in descending order, the lower expert index first
// among equal keys, by warp rounds over per-lane candidate lists.  Each lane holds C (order key, expert index) pairs sorted by key
// descending, lower index first among equal keys; a round takes the warp's best head (a
// redux.sync max of the keys, then a redux.sync min of the indices holding it) and the
// owning lane drops its head.  An empty slot is (0, 0x7fffffff): below every finite key's
// order key, and never chosen while k real candidates remain.
constexpr uint32_t kEmptyIdx = 0x7fffffffu;

template <int C>
__device__ __forceinline__ void lane_sort_desc(uint32_t (&key)[C], uint32_t (&idx)[C]) {
  // odd-even transposition: C passes sort C entries
#pragma unroll
  for (int r = 0; r < C; ++r)
#pragma unroll
    for (int i = r & 1; i + 1 < C; i += 2) {
      const bool sw = key[i] < key[i + 1] || (key[i] == key[i + 1] && idx[i] > idx[i + 1]);
      const uint32_t k0 = sw ? key[i + 1] : key[i], k1 = sw ? key[i] : key[i + 1];
      const uint32_t i0 = sw ? idx[i + 1] : idx[i], i1 = sw ? idx[i] : idx[i + 1];
      key[i] = k0; key[i + 1] = k1;
      idx[i] = i0; idx[i + 1] = i1;
    }
}

// k rounds over sorted per-lane lists; lane r (< k) receives the r-th selection.
template <int C>
__device__ __forceinline__ void warp_select_lists(uint32_t (&key)[C], uint32_t (&idx)[C], int k, int lane,
                                                  uint32_t& my_key, uint32_t& my_idx) {
  my_key = 0;
  my_idx = kEmptyIdx;
  for (int r = 0; r < k; ++r) {
    const uint32_t mu = __reduce_max_sync(0xffffffffu, key[0]);
    const uint32_t bi = __reduce_min_sync(0xffffffffu, key[0] == mu ? idx[0] : 0xffffffffu);
    if (lane == r) { my_key = mu; my_idx = bi; }
    if (key[0] == mu && idx[0] == bi) {   // the winner drops its head
#pragma unroll
      for (int i = 0; i + 1 < C; ++i) { key[i] = key[i + 1]; idx[i] = idx[i + 1]; }
      key[C - 1] = 0;
      idx[C - 1] = kEmptyIdx;
    }
  }
}

// Route selection, one launch after the router GEMM.  A CTA of 8 warps takes `tpc` tokens
// (1 or 8) at a time.
//   Stage 1: warp w owns the expert slice [w * 32C, (w + 1) * 32C), C experts per lane; it
//   forms z (the split partials summed in split order, plus the logit bias, stored; or z
//   as the GEMM stored it) and the selection key (z, or z + b in the select-only mode,
//   fp32) as an order-preserving uint32 in shared memory.
//   Stage 2: warp i selects token i's top k from its E keys.  theta = the k-th largest of
//   the 32 lanes' maxima: k lanes hold a key >= theta, so the k-th largest key is >= theta,
//   and every key of the top k (ties at the k-th included) is >= theta.  Those candidates,
//   about 20 of 896 for spread keys, go into per-lane lists of 4 and k warp rounds pick
//   them in order (key descending, lower index first).  When some lane holds more than 4
//   (heavy ties), the rounds scan the keys in shared memory instead.
//   Then w_j = s_j / sum of the selected s, s = sigmoid(z), the sum in selection order.
// z is not __restrict__: stage 2 reads back what stage 1 stored.
template <int C>
__global__ void __launch_bounds__(256) route_select_kernel(const float* __restrict__ zpart, int ksplit,
                                                           long long plane, const float* __restrict__ bias,
                                                           const float* __restrict__ select_bias, float* z, int T,
                                                           int E, int k, int tpc, int* __restrict__ idx_out,
                                                           float* __restrict__ w_out) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ uint32_t sel_keys[];   // [tpc][E] order keys
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t0 = blockIdx.x * tpc; t0 < T; t0 += gridDim.x * tpc) {
    // ---- stage 1
    for (int i = 0; i < tpc && t0 + i < T; ++i) {
      const size_t row = (size_t)(t0 + i) * E;
      float v[C];
#pragma unroll
      for (int c = 0; c < C; ++c) v[c] = 0.0f;
      if (ksplit > 1) {
        constexpr int S = C >= 8 ? 2 : 8;   // partials in flight per expert
        for (int s0 = 0; s0 < ksplit; s0 += S) {
          float pp[C][S];
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const int e = warp * 32 * C + lane + 32 * c;
#pragma unroll
            for (int q = 0; q < S; ++q)
              pp[c][q] = (e < E && s0 + q < ksplit) ? __ldcg(zpart + (size_t)(s0 + q) * plane + row + e) : 0.0f;
          }
#pragma unroll
          for (int c = 0; c < C; ++c)
#pragma unroll
            for (int q = 0; q < S; ++q)
              if (s0 + q < ksplit) v[c] = (s0 + q == 0) ? pp[c][q] : v[c] + pp[c][q];
        }
      }
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const int e = warp * 32 * C + lane + 32 * c;
        if (e < E) {
          float zv;
          if (ksplit > 1) {
            zv = bias ? v[c] + __ldg(bias + e) : v[c];
            z[row + e] = zv;
          } else {
            zv = z[row + e];
          }
          const float kv = select_bias ? zv + __ldg(select_bias + e) : zv;
          sel_keys[(size_t)i * E + e] = f32_order_key(kv + 0.0f);   // -0 -> +0: equal keys compare equal
        }
      }
    }
    __syncthreads();
    // ---- stage 2
    if (warp < tpc && t0 + warp < T) {
      const int t = t0 + warp;
      uint32_t* kr = sel_keys + (size_t)warp * E;
      uint32_t lmax = 0;
      for (int e = lane; e < E; e += 32) lmax = max(lmax, kr[e]);
      // theta: k rounds of the warp maximum over the lane maxima, one holder removed a round
      uint32_t theta = 0, mk = lmax;
      for (int r = 0; r < k; ++r) {
        const uint32_t mx = __reduce_max_sync(0xffffffffu, mk);
        theta = mx;
        const uint32_t bl = __reduce_min_sync(0xffffffffu, mk == mx ? (uint32_t)lane : 32u);
        if ((uint32_t)lane == bl) mk = 0;
      }
      uint32_t key[4], id[4];
      int cnt = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) { key[j] = 0; id[j] = kEmptyIdx; }
      for (int e = lane; e < E; e += 32) {
        const uint32_t kv = kr[e];
        if (kv >= theta) {
          // append at slot cnt (predicated writes: no dynamic register index)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (j == cnt) { key[j] = kv; id[j] = (uint32_t)e; }
          ++cnt;
        }
      }
      uint32_t sk, si;
      if (__any_sync(0xffffffffu, cnt > 4)) {
        // heavy ties: k rounds over all keys; a taken key becomes 0 (below every real key)
        sk = 0;
        si = kEmptyIdx;
        for (int r = 0; r < k; ++r) {
          uint32_t bv = 0, bi = kEmptyIdx;
          for (int e = lane; e < E; e += 32) {
            const uint32_t kv = kr[e];
            if (kv > bv) { bv = kv; bi = (uint32_t)e; }   // ascending e: the lower index kept
          }
          const uint32_t mu = __reduce_max_sync(0xffffffffu, bv);
          const uint32_t wi = __reduce_min_sync(0xffffffffu, bv == mu ? bi : 0xffffffffu);
          if (lane == r) { sk = mu; si = wi; }
          if (lane == (int)(wi & 31)) kr[wi] = 0;
          __syncwarp();
        }
      } else {
        lane_sort_desc<4>(key, id);
        warp_select_lists<4>(key, id, k, lane, sk, si);
      }
      float sv = 0.0f;
      if (lane < k) {
        // select-only: the weight uses z, which this CTA stored (or the GEMM did)
        const float zsel = select_bias ? z[(size_t)t * E + si] : f32_from_order_key(sk);
        sv = 1.0f / (1.0f + expf(-zsel));
      }
      float ssum = 0.0f;
      for (int r = 0; r < k; ++r) ssum += __shfl_sync(0xffffffffu, sv, r);
      if (lane < k) {
        idx_out[(size_t)t * k + lane] = (int)si;
        w_out[(size_t)t * k + lane] = sv / ssum;
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- combine
// y[t] = bf16( y_shared[t] + sum_j w[t][j] * O[inv[t][j]] ), fp32 sums in slot order.
// Grid (T, ceil(d / 1024)): each thread owns 8 columns of one token; the k expert rows
// are fetched four at a time so that several 16-byte loads are in flight per thread.
constexpr int kCombineThreads = 128;
constexpr int kCombineCols = kCombineThreads * 8;
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const __nv_bfloat16* __restrict__ O, const float* __restrict__ ys,
                   const float* __restrict__ w, const int* __restrict__ inv, int T, int d, int k,
                   __nv_bfloat16* __restrict__ y) {
  griddep_wait();
  griddep_launch_dependents();
  const int t = blockIdx.x;
  extern __shared__ int s_inv[];
  float* s_w = (float*)(s_inv + k);
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    s_inv[j] = __ldg(inv + (size_t)t * k + j);
    s_w[j] = __ldg(w + (size_t)t * k + j);
  }
  __syncthreads();
  const int c = blockIdx.y * kCombineCols + threadIdx.x * 8;
  if (c >= d) return;
  float acc[8];
  if (ys) {
    const float4 a = __ldg((const float4*)(ys + (size_t)t * d + c));
    const float4 b = __ldg((const float4*)(ys + (size_t)t * d + c + 4));
    acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
    acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
  }
  for (int j0 = 0; j0 < k; j0 += 4) {
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int p = j0 + q < k ? s_inv[j0 + q] : -1;
      v[q] = p >= 0 ? __ldg((const uint4*)(O + (size_t)p * d + c)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (j0 + q >= k || s_inv[j0 + q] < 0) continue;
      const uint32_t wv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
      const float wj = s_w[j0 + q];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(wj, __uint_as_float(wv[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(wj, __uint_as_float(wv[i] & 0xFFFF0000u), acc[2 * i + 1]);
      }
    }
  }
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 p2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    o[i] = *(const uint32_t*)&p2;
  }
  *(uint4*)(y + (size_t)t * d + c) = make_uint4(o[0], o[1], o[2], o[3]);
}

// ---------------------------------------------------------------- latent option
// x_n[t] = bf16(x_l[t] / sqrt(mean(x_l[t]^2) + eps) * gamma), one CTA (256 threads) per row;
// the sum of squares in fp32, reduced in a fixed order (per thread, then warp, then CTA).
__global__ void __launch_bounds__(256)
    rmsnorm_bf16_kernel(const float* __restrict__ xl, const float* __restrict__ gamma, int cols, float eps,
                        __nv_bfloat16* __restrict__ xn) {
  griddep_wait();
  griddep_launch_dependents();
  const float* row = xl + (size_t)blockIdx.x * cols;
  float ss = 0.0f;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) ss = fmaf(row[c], row[c], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  __shared__ float part[8];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) tot += part[i];
  const float inv = rsqrtf(tot / (float)cols + eps);
  for (int c = threadIdx.x; c < cols; c += blockDim.x)
    xn[(size_t)blockIdx.x * cols + c] = __float2bfloat16_rn(row[c] * inv * __ldg(gamma + c));
}

// y = bf16(a + b) (b may be NULL), fp32 inputs, 4 elements per thread (n % 4 == 0).
__global__ void add_bf16_kernel(const float* __restrict__ a, const float* __restrict__ b, long long n,
                                __nv_bfloat16* __restrict__ y) {
  griddep_wait();
  griddep_launch_dependents();
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= n) return;
  float4 v = __ldg((const float4*)(a + i));
  if (b) {
    const float4 u = __ldg((const float4*)(b + i));
    v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
  }
  const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 o;
  o.x = *(const uint32_t*)&lo;
  o.y = *(const uint32_t*)&hi;
  *(uint2*)(y + i) = o;
}

// ---------------------------------------------------------------- failure-path probe
// One thread waits on an mbarrier of count 1 that nothing arrives at, with the bounded
// wait of the production kernels; it gives up after the limit and flags the status word.
__global__ void timeout_probe_kernel(unsigned int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, status, (volatile int*)&abort_flag);
  __syncthreads();
}

// ---------------------------------------------------------------- weight packing (setup)
// fp32 rows [R][K] -> E2M1 codes (2 per byte, element 2j in the low nibble) for packed row
// dst_row(r) in the tile-major code layout [m-tile][K/128][256 rows][64 B], and E8M0
// scales into the MMA scale-factor atom layout
// [m_tiles][K/128][2][512]: row rr of a 256-row tile, K-block kb ->
//   ((mt * (K/128) + kb/4) * 2 + half) * 512 + (rr%32)*16 + ((rr%128)/32)*4 + kb%4.
// interleave != 0: rows of two sources (gate, up) go to packed rows
//   256*(r/128) + 128*src + r%128.
__global__ void pack_mxfp4_kernel(const float* __restrict__ src0, const float* __restrict__ src1,
                                  int R, int K, int interleave, uint8_t* __restrict__ wdst,
                                  uint8_t* __restrict__ sdst) {
  const int nb = K >> 5;
  const int nsrc = interleave ? 2 : 1;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)nsrc * R * nb) return;
  const int which = (int)(gid / ((long long)R * nb));
  const long long rem = gid - (long long)which * R * nb;
  const int r = (int)(rem / nb);
  const int b = (int)(rem - (long long)r * nb);
  const float* src = which ? src1 : src0;
  const float4* p = (const float4*)(src + (size_t)r * K + b * 32);
  float v[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 f = __ldg(p + i);
    v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int e = mx_scale_exp(amax, 2);
  const float s = pow2_neg(e);
  uint32_t wds[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t acc = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc |= cvt_e2m1x2(v[8 * i + 2 * j] * s, v[8 * i + 2 * j + 1] * s) << (8 * j);
    wds[i] = acc;
  }
  const int pr = interleave ? 256 * (r >> 7) + 128 * which + (r & 127) : r;
  // tile-major codes: [m-tile][k-tile][256 rows][64 B]; block b is 16 B of its row's 64 B
  const size_t wo = ((size_t)((pr >> 8) * (K >> 7) + (b >> 2)) * 256 + (pr & 255)) * 64 + (b & 3) * 16;
  *(uint4*)(wdst + wo) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  const int mt = pr >> 8, half = (pr >> 7) & 1, rr = pr & 127;
  const size_t so = ((size_t)(mt * (K >> 7) + (b >> 2)) * 2 + half) * 512 + (rr & 31) * 16 +
                    (rr >> 5) * 4 + (b & 3);
  sdst[so] = (uint8_t)(e + 127);
}

// Router weights W_r fp32 [d][E] -> three bf16 planes W^T [E][3d] with
// W = hi + mid + lo exactly (hi = bf16(W), mid = bf16(W - hi), lo = bf16(W - hi - mid)).
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ W, int d, int E,
                                                           __nv_bfloat16* __restrict__ planes) {
  griddep_wait();
  griddep_launch_dependents();
  // block: 32 experts x 64 rows of W; coalesced 128-byte row reads, then per expert 64
  // consecutive K elements of each plane as bf16 pairs (128-byte warp stores)
  __shared__ float tile[64][33];
  const int e0 = blockIdx.x * 32, i0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 8 warps
  for (int r = ty; r < 64; r += 8) {
    const int i = i0 + r, e = e0 + tx;
    tile[r][tx] = (i < d && e < E) ? W[(size_t)i * E + e] : 0.0f;
  }
  __syncthreads();
  for (int c = ty; c < 32; c += 8) {
    const int e = e0 + c, i = i0 + 2 * tx;
    if (e >= E || i >= d) continue;   // d is even (a multiple of 128)
    __nv_bfloat162 p[3];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float w = tile[2 * tx + u][c];
      const __nv_bfloat16 hi = __float2bfloat16_rn(w);
      const float r1 = w - __bfloat162float(hi);
      const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
      const float r2 = r1 - __bfloat162float(mid);
      const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
      if (u == 0) { p[0].x = hi; p[1].x = mid; p[2].x = lo; }
      else        { p[0].y = hi; p[1].y = mid; p[2].y = lo; }
    }
    __nv_bfloat16* row = planes + (size_t)e * 3 * d;
#pragma unroll
    for (int q = 0; q < 3; ++q) *(__nv_bfloat162*)(row + (size_t)q * d + i) = p[q];
  }
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------- Quantile Balancing inputs
// Routing margin m[t][e] = key[t][e] - theta[t], with key = z (+ b in the select-only
// mode, formed in fp32) and theta[t] the token's k-th largest key; the per-expert quantile
// at level q is the order statistic of rank j = clamp(ceil(q T), 1, T) of m[:, e].

// One warp per token: theta[t] = the k-th largest key (k rounds of a warp arg-max, lower
// index first on equal keys, as in the selection).
__global__ void kth_key_kernel(const float* __restrict__ z, const float* __restrict__ select_bias, int T,
                               int E, int k, float* __restrict__ theta) {
  extern __shared__ float keys[];  // [warps][E]
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + w;
  if (t >= T) return;
  float* row = keys + (size_t)w * E;
  for (int e = lane; e < E; e += 32)
    row[e] = select_bias ? __ldg(z + (size_t)t * E + e) + __ldg(select_bias + e) : __ldg(z + (size_t)t * E + e);
  __syncwarp();
  float bv = -INFINITY;
  for (int r = 0; r < k; ++r) {
    bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float v = row[e];
      if (v > bv) { bv = v; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) row[bi] = -INFINITY;
    __syncwarp();
  }
  if (lane == 0) theta[t] = bv;
}

// Exact order statistics of the margins by radix select, 8 bits a pass from the top.
// CTA (group g, level l): experts 32 g .. 32 g + 31 (lane = expert within the group), rank
// ranks[l].  256 threads; each warp walks tokens w, w + 8, ... and reads one 128-byte run
// of a token's logits per step.
constexpr int kQuantThreads = 256;
constexpr int kMaxQuantLevels = 16;
struct QuantRanks {
  int r[kMaxQuantLevels];   // 1-based ranks, one per level
};
__global__ void __launch_bounds__(kQuantThreads)
    margin_quantile_kernel(const float* __restrict__ z, const float* __restrict__ select_bias,
                           const float* __restrict__ theta, int T, int E, const QuantRanks ranks,
                           float* __restrict__ out) {
  __shared__ uint32_t hist[32][257];
  __shared__ uint32_t s_prefix[32], s_rank[32];
  const int g = blockIdx.x, lvl = blockIdx.y;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = g * 32 + lane;
  const bool e_ok = e < E;
  const float b = (select_bias && e_ok) ? __ldg(select_bias + e) : 0.0f;
  if (threadIdx.x < 32) {
    s_prefix[threadIdx.x] = 0u;
    s_rank[threadIdx.x] = (uint32_t)ranks.r[lvl];   // 1-based rank within the column
  }
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 32 * 257; i += blockDim.x) (&hist[0][0])[i] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix[lane];
    const uint32_t hi_mask = pass == 0 ? 0u : (0xffffffffu << (32 - 8 * pass));
    if (e_ok) {
      for (int t = w; t < T; t += blockDim.x >> 5) {
        const float key = select_bias ? __ldg(z + (size_t)t * E + e) + b : __ldg(z + (size_t)t * E + e);
        const uint32_t u = f32_order_key(key - __ldg(theta + t));
        if ((u & hi_mask) == prefix) atomicAdd(&hist[lane][(u >> shift) & 255u], 1u);
      }
    }
    __syncthreads();
    if (threadIdx.x < 32 && g * 32 + (int)threadIdx.x < E) {
      uint32_t r = s_rank[threadIdx.x], digit = 0;
      for (; digit < 255; ++digit) {
        const uint32_t c = hist[threadIdx.x][digit];
        if (r <= c) break;
        r -= c;
      }
      s_rank[threadIdx.x] = r;
      s_prefix[threadIdx.x] |= digit << shift;
    }
    __syncthreads();
  }
  if (threadIdx.x < 32 && g * 32 + (int)threadIdx.x < E)
    out[(size_t)lvl * E + g * 32 + threadIdx.x] = f32_from_order_key(s_prefix[threadIdx.x]);
}

}  // namespace moe
