// Fractal flattening and its inverse: a row permutation along the token axis
// (NABLA technical summary, "Metodologia: NABLA", item 1).  Grid order
// s = (t*H + h)*W + w; flattened order
// f = t*H*W + ((h/P)*(W/P) + w/P)*P*P + (h%P)*P + (w%P).
//
// HBM-bound copy: one warp moves one destination row with 16-byte vector
// loads and stores (a row is row_bytes = Hh*D*2 bytes, a multiple of 16), so
// every warp request covers 512 contiguous bytes.  Reads are streamed
// (evict-first); the grid is a multiple of the SM count and loops.
#pragma once

#include "common.cuh"

namespace nabla {

struct GridShape {
  int T, H, W, P;
};

// Flattened index -> grid index.
__device__ __forceinline__ int64_t flat_to_grid(int64_t f, const GridShape g) {
  const int64_t hw = static_cast<int64_t>(g.H) * g.W;
  const int64_t t = f / hw;
  const int rem = static_cast<int>(f - t * hw);
  const int pp = g.P * g.P;
  const int blk = rem / pp;
  const int within = rem - blk * pp;
  const int nbw = g.W / g.P;
  const int bh = blk / nbw, bw = blk - (blk / nbw) * nbw;
  const int h = bh * g.P + within / g.P;
  const int w = bw * g.P + within % g.P;
  return (t * g.H + h) * g.W + w;
}

// Grid index -> flattened index.
__device__ __forceinline__ int64_t grid_to_flat(int64_t s, const GridShape g) {
  const int64_t hw = static_cast<int64_t>(g.H) * g.W;
  const int64_t t = s / hw;
  const int rem = static_cast<int>(s - t * hw);
  const int h = rem / g.W, w = rem - (rem / g.W) * g.W;
  const int nbw = g.W / g.P;
  return t * hw + static_cast<int64_t>((h / g.P) * nbw + w / g.P) * g.P * g.P + (h % g.P) * g.P + (w % g.P);
}

// dst row r (of B*S rows) receives src row map(r).  inverse = false: dst is
// flattened (flatten); inverse = true: dst is grid order (unflatten).
template <bool kInverse>
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          int64_t rows, int64_t S, GridShape g, int chunks) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; r < rows; r += warps_total) {
    const int64_t b = r / S;
    const int64_t d = r - b * S;
    const int64_t s = kInverse ? grid_to_flat(d, g) : flat_to_grid(d, g);
    const uint4* sp = src + (b * S + s) * chunks;
    uint4* dp = dst + r * chunks;
    int c = lane;
    for (; c + 96 < chunks; c += 128) {
      uint4 v0 = __ldcs(sp + c), v1 = __ldcs(sp + c + 32), v2 = __ldcs(sp + c + 64), v3 = __ldcs(sp + c + 96);
      dp[c] = v0;
      dp[c + 32] = v1;
      dp[c + 64] = v2;
      dp[c + 96] = v3;
    }
    for (; c < chunks; c += 32) dp[c] = __ldcs(sp + c);
  }
}

}  // namespace nabla
