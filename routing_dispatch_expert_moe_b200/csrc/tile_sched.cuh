// Device-side tile scheduler for the grouped expert GEMMs.
//
// Expert e owns rows [offsets[e], offsets[e+1]) of the permuted activations; the row
// counts are known only on the device (no host synchronisation).  Every CTA of a
// persistent grid rebuilds, in shared memory, the exclusive prefix
//   tile_start[e] = sum_{e' < e} ceil(rows_e' / BM) * n_tiles
// and walks the virtual tile sequence blockIdx.x, blockIdx.x + gridDim.x, ...; a tile
// index maps back to its expert by binary search (empty experts own no tile).
// Uneven groups without padding: "Mixture of Experts Explained" (zh), section
// "更多关于高效训练的内容" (block-sparse handling of uneven expert loads).
#pragma once

#include "common.cuh"

namespace moe {

struct TileCoord {
  int e;          // expert
  int row0;       // first row of the tile (global row index into the permuted buffers)
  int rows;       // valid rows in this tile (1..BM)
  int n_tile;     // tile index along the output columns
};

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024).
__device__ __forceinline__ int block_excl_scan(int v, int* sh32, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += n;
  }
  __syncthreads();
  if (lane == 31 || threadIdx.x == blockDim.x - 1) sh32[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? sh32[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    sh32[lane] = w;
  }
  __syncthreads();
  *total = sh32[nw - 1];
  return (warp > 0 ? sh32[warp - 1] : 0) + x - v;
}

// Fills tile_start[0..E] (shared memory).  Row counts are clamped to [0, rows_max];
// a bad offsets array records MOE_DEVERR_ROW and yields fewer tiles, never a bad access.
__device__ __forceinline__ void build_tile_starts(const int32_t* __restrict__ offsets, int E, int BM,
                                                  int n_tiles, long long rows_max, int* tile_start,
                                                  int* sh32, int* err) {
  const int nt = blockDim.x;
  const int per = (E + nt - 1) / nt;
  const int e0 = min(E, (int)threadIdx.x * per), e1 = min(E, e0 + per);
  int local = 0;
  for (int e = e0; e < e1; ++e) {
    long long a = __ldg(offsets + e), b = __ldg(offsets + e + 1);
    if (a < 0 || b < a || b > rows_max) {
      record_error(err, MOE_DEVERR_ROW);
      continue;
    }
    local += (int)((b - a + BM - 1) / BM) * n_tiles;
  }
  int total;
  int run = block_excl_scan(local, sh32, &total);
  for (int e = e0; e < e1; ++e) {
    tile_start[e] = run;
    long long a = __ldg(offsets + e), b = __ldg(offsets + e + 1);
    if (a < 0 || b < a || b > rows_max) continue;
    run += (int)((b - a + BM - 1) / BM) * n_tiles;
  }
  if (threadIdx.x == 0) tile_start[E] = total;
  __syncthreads();
}

// Tile index -> coordinates: m fastest inside an expert, then n, so that the CTAs working
// at one time share each weight tile (the large operand of the expert GEMMs).
__device__ __forceinline__ TileCoord tile_coord(const int* tile_start, const int32_t* __restrict__ offsets,
                                                int E, int BM, int tile) {
  int lo = 0, hi = E;  // find last e with tile_start[e] <= tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_start[mid] <= tile) lo = mid; else hi = mid;
  }
  // skip experts that own no tile (equal starts): the last e with start <= tile owns it
  TileCoord c;
  c.e = lo;
  const int a = __ldg(offsets + lo), b = __ldg(offsets + lo + 1);
  const int mt = (b - a + BM - 1) / BM;
  const int local = tile - tile_start[lo];
  c.n_tile = local / mt;
  const int m = local - c.n_tile * mt;
  c.row0 = a + m * BM;
  c.rows = min(BM, b - c.row0);
  return c;
}

}  // namespace moe
