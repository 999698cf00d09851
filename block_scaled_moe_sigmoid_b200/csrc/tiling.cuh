// Token-tile bookkeeping shared by the grouped GEMMs and the kernels that write their
// token-side scale factors.
//
// Rows of one group (expert) are split into ntiles = ceil(rows / BN) tiles of
// n_per = round_up(ceil(rows / ntiles), 16) rows; tile_prefix[g] is the first group-tile
// index of group g.  Token-side scale factors are stored tile-major: for group-tile gt and
// K tile kt, a 1 KB block holds two 512-byte scale-factor atoms in the layout the tensor
// core reads (row n of the tile -> atom n/128, byte (n%32)*16 + ((n%128)/32)*4 + kb, with
// kb the 32-element block inside the 128-element K tile).  A GEMM stage then fetches its
// token scales with one bulk copy.
#pragma once

namespace moe {

constexpr int SF_TILE_BYTES = 1024;

__host__ __device__ __forceinline__ int sf_atom_offset(int n) {
  return (n >> 7) * 512 + (n & 31) * 16 + ((n & 127) >> 5) * 4;
}

__host__ __device__ __forceinline__ int tile_rows_per(int rows, int ntiles) {
  const int n = (rows + ntiles - 1) / ntiles;
  return (n + 15) & ~15;
}

// Group-tile index and row-in-tile of row p (global row) of group e.
__device__ __forceinline__ void row_tile(const int* counts, const int* offsets, const int* tile_prefix,
                                         int e, int p, int& gt, int& n) {
  const int tp = __ldg(tile_prefix + e);
  const int ntiles = __ldg(tile_prefix + e + 1) - tp;
  const int n_per = tile_rows_per(__ldg(counts + e), ntiles);
  const int r = p - __ldg(offsets + e);
  const int nt = r / n_per;
  gt = tp + nt;
  n = r - nt * n_per;
}

}  // namespace moe
