// AB-Attention sampling plan (news page "AB-Attention acelera a geracao de
// video em ate 2,23x e pula 92% da atencao", section "Os tres recursos do
// AB-Attention"), on tensors in their original (grid) order:
//
// ab_key_means_kernel  mean key of every 4-token block, written transposed
//                      kbar^T [B][Hh][D][NKB] for the centroid logits;
// ab_kmeans_kernel     IBCS: 8 clusters per 128-query block (Lloyd's
//                      iterations from the queries at 0, 16, ..., 112),
//                      centroids transposed cent^T [B][Hh][D][NQB*8] and
//                      counts [B][Hh][NQB][8];
// (score_tile_kernel)  centroid logits l = cent . kbar * scale, [NQB*8][NKB]
//                      per (b, head), the same fp32 chain as the oracle;
// ab_select_kernel     per query block: block scores
//                      s_J = sum_c (n_c/128) softmax_J(l_c)_J, inclusion
//                      probabilities pi = min(1, lambda s) with sum(pi) =
//                      budget (water-filling), the sample u < pi with its
//                      logit shifts -log(pi), compacted ascending.
// The arithmetic of the means, the clustering and the logits is the oracle's
// operation for operation (bit-identical); the scores use expf and fp32/fp64
// sums in the GPU's order, so pi agrees with the oracle's to ~1e-7 and the
// sampling decisions to within that band.
#pragma once

#include "common.cuh"
#include "mask.cuh"

namespace nabla {

constexpr int kABQBlock = 128;
constexpr int kABClusters = 8;
constexpr int kABKBlock = 4;

// grid (NKB / 8, B): CTA = 8 consecutive key blocks (32 tokens); thread c
// sums elements 8c..8c+7 of the 4 token rows of each block in fp32, rows
// ascending, times 0.25, and writes them transposed.
__global__ void __launch_bounds__(256) ab_key_means_kernel(const __nv_bfloat16* __restrict__ k,
                                                           float* __restrict__ kbarT, int S, int Hh, int D) {
  const int J0 = blockIdx.x * 8, b = blockIdx.y;
  const int nkb = S / kABKBlock;
  const int chunks = (Hh * D) >> 3;
  const uint4* base = reinterpret_cast<const uint4*>(k) + (static_cast<int64_t>(b) * S + J0 * kABKBlock) * chunks;
  for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
    float out[8][8];  // [element][block]
#pragma unroll
    for (int jb = 0; jb < 8; ++jb) {
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int r = 0; r < kABKBlock; ++r) {
        const uint4 v = __ldg(base + static_cast<int64_t>(jb * kABKBlock + r) * chunks + c);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          acc[2 * e] = __fadd_rn(acc[2 * e], f.x);
          acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], f.y);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) out[e][jb] = acc[e] * 0.25f;
    }
    const int col = c * 8, h = col / D, d = col - h * D;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float4* o = reinterpret_cast<float4*>(kbarT + ((static_cast<int64_t>(b) * Hh + h) * D + d + e) * nkb + J0);
      o[0] = make_float4(out[e][0], out[e][1], out[e][2], out[e][3]);
      o[1] = make_float4(out[e][4], out[e][5], out[e][6], out[e][7]);
    }
  }
}

// grid (NQB, Hh, B), 256 threads.  Shared memory: the block's 128 queries
// as fp32 rows of D + 1 floats (the padding spreads a column over the
// banks), the 8 centroids, the assignment.  Per iteration:
//   assignment: thread (t, half) = (tid / 2, tid % 2) computes the squared
//     distances of query t to centroids 4*half .. 4*half+3 (diff rounded to
//     fp32, then an fmaf chain over d ascending), keeps the nearest (ties to
//     the lower index) and settles with its partner lane;
//   members: one warp lists each cluster's queries in ascending token order
//     (ballots over 32 queries at a time);
//   update: thread owns (c, d) pairs; the fp32 sum over the cluster's
//     listed queries in that order, one division by the count; an empty
//     cluster keeps its centroid.
__global__ void __launch_bounds__(256) ab_kmeans_kernel(const __nv_bfloat16* __restrict__ q,
                                                        float* __restrict__ centT, int32_t* __restrict__ counts,
                                                        int S, int Hh, int D, int iters) {
  extern __shared__ __align__(16) float ksm[];
  const int I = blockIdx.x, hd = blockIdx.y, b = blockIdx.z;
  const int nqb = S / kABQBlock;
  const int ld = D + 1;
  float* x = ksm;                         // [128][D + 1]
  float* mu = x + kABQBlock * ld;         // [8][D]
  int* asg = reinterpret_cast<int*>(mu + kABClusters * D);  // [128]
  int* cnt = asg + kABQBlock;             // [8]
  int* mem = cnt + kABClusters;           // [8][128]: each cluster's queries, ascending
  int* mcount = mem + kABClusters * kABQBlock;  // [8]
  const int tid = threadIdx.x;
  const int chunks = D >> 3;  // 16-byte chunks of one head's slice of a token row
  for (int u = tid; u < kABQBlock * chunks; u += blockDim.x) {
    const int t = u / chunks, c = u - t * chunks;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(
                              q + ((static_cast<int64_t>(b) * S + static_cast<int64_t>(I) * kABQBlock + t) * Hh + hd) * D) +
                          c);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      x[t * ld + c * 8 + 2 * e] = f.x;
      x[t * ld + c * 8 + 2 * e + 1] = f.y;
    }
  }
  __syncthreads();
  for (int u = tid; u < kABClusters * D; u += blockDim.x) {
    const int c = u / D, d = u - c * D;
    mu[u] = x[(c * (kABQBlock / kABClusters)) * ld + d];
  }
  if (tid < kABClusters) cnt[tid] = 0;
  __syncthreads();
  const int t = tid >> 1, half = tid & 1;
  for (int it = 0; it < iters; ++it) {
    // assignment
    float dist[4];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) dist[cc] = 0.f;
    const float* xt = x + t * ld;
    const float* m0 = mu + (4 * half) * D;
    for (int d = 0; d < D; ++d) {
      const float xv = xt[d];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const float diff = __fsub_rn(xv, m0[cc * D + d]);
        dist[cc] = __fmaf_rn(diff, diff, dist[cc]);
      }
    }
    int best = 4 * half;
    float bd = dist[0];
#pragma unroll
    for (int cc = 1; cc < 4; ++cc)
      if (dist[cc] < bd) {
        bd = dist[cc];
        best = 4 * half + cc;
      }
    const float obd = __shfl_xor_sync(0xffffffffu, bd, 1);
    const int obest = __shfl_xor_sync(0xffffffffu, best, 1);
    // the lower half's candidate has the lower index: it wins ties
    if (half == 0) asg[t] = (obd < bd) ? obest : best;
    __syncthreads();
    // members of each cluster, ascending
    if (tid < 32) {
      const int lane = tid;
      int nb[kABClusters];
#pragma unroll
      for (int c = 0; c < kABClusters; ++c) nb[c] = 0;
      for (int s0 = 0; s0 < kABQBlock; s0 += 32) {
        const int a_s = asg[s0 + lane];
#pragma unroll
        for (int c = 0; c < kABClusters; ++c) {
          const unsigned bal = __ballot_sync(0xffffffffu, a_s == c);
          if (a_s == c) mem[c * kABQBlock + nb[c] + __popc(bal & ((1u << lane) - 1u))] = s0 + lane;
          nb[c] += __popc(bal);
        }
      }
#pragma unroll
      for (int c = 0; c < kABClusters; ++c)
        if (lane == c) mcount[c] = nb[c];
    }
    __syncthreads();
    // update: pairs (c, d), c = u / D (one c per warp: D >= 32)
    for (int u = tid; u < kABClusters * D; u += blockDim.x) {
      const int c = u / D, d = u - c * D;
      const int n = mcount[c];
      const int* mc = mem + c * kABQBlock;
      float acc = 0.f;
      for (int e = 0; e < n; ++e) acc = __fadd_rn(acc, x[mc[e] * ld + d]);
      if (n > 0) mu[u] = __fdiv_rn(acc, static_cast<float>(n));
      if (d == 0) cnt[c] = n;
    }
    __syncthreads();
  }
  const int64_t bh = static_cast<int64_t>(b) * Hh + hd;
  const int R = nqb * kABClusters;
  for (int u = tid; u < kABClusters * D; u += blockDim.x) {
    const int c = u / D, d = u - c * D;
    centT[(bh * D + d) * R + I * kABClusters + c] = mu[u];
  }
  if (tid < kABClusters) counts[(bh * nqb + I) * kABClusters + tid] = cnt[tid];
}

inline size_t ab_kmeans_smem(int D) {
  return (static_cast<size_t>(kABQBlock) * (D + 1) + kABClusters * D) * 4 + kABQBlock * 4 + kABClusters * 4 +
         kABClusters * kABQBlock * 4 + kABClusters * 4;
}

struct ABSelectArgs {
  const float* logits;   // [B*Hh][NQB*8][NKB]
  const int32_t* counts; // [B*Hh][NQB][8]
  const float* u;        // [B*Hh][NQB][NKB] uniforms in [0, 1)
  int32_t* kcount;       // [B*Hh][NQB]
  int32_t* kidx;         // [B*Hh][NQB][NKB]
  float* kshift;         // [B*Hh][NQB][NKB]
  int nqb, nkb;
  double budget;
};

__device__ __forceinline__ double block_sum_f64(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += red[w];
  return t;
}
__device__ __forceinline__ int block_sum_int(int v, double* red) {
  return static_cast<int>(block_sum_f64(static_cast<double>(v), red));
}

// grid (NQB, B*Hh), 256 threads (8 warps).  Shared memory: the row's block
// scores (NKB fp32), per-warp partial maxima and sums, reductions.  The row's
// 8 x NKB centroid logits are read twice, as float4 with the 8 centroids'
// loads independent (NKB is a multiple of 32):
//   1. one pass for every centroid's max and normaliser: each thread keeps a
//      running max m and sum z = sum_J exp(l_cJ - m) (expf terms, fp64 sum),
//      rescaled by exp(m_old - m_new) when m grows; the partial (m, z) pairs
//      are merged over the warp, then over the CTA, the same way;
//   2. s_J = sum_c (n_c / 128) exp(l_cJ - max_c) / Z_c, and sum_J s_J;
//   3. lambda by water-filling: start from lambda = budget / sum(s), then
//      repeatedly cap the blocks with lambda s >= 1 and set lambda =
//      (budget - capped) / (sum of the uncapped scores) until the capped
//      set stops growing (it only grows; at most 64 rounds);
//   4. block J is sampled iff u_J < min(1, lambda s_J); each warp owns a
//      contiguous range of J, counts its sample, and after one exchange of
//      the counts writes it ascending with its shifts -log(pi).
constexpr int kABSelectWarps = 8;
__global__ void __launch_bounds__(kABSelectWarps * 32, 3) ab_select_kernel(const ABSelectArgs a) {
  extern __shared__ __align__(16) float sel_sm[];
  float* sc = sel_sm;                                                // [NKB]
  double* red = reinterpret_cast<double*>(sc + ((a.nkb + 3) & ~3));  // [8]
  double* wsum = red + 8;                                            // [warps][8]
  float* cmax = reinterpret_cast<float*>(wsum + kABSelectWarps * kABClusters);  // [8]
  float* cinv = cmax + 8;                                            // [8]: (n_c / 128) / Z_c
  float* wmax = cinv + 8;                                            // [warps][8]
  int* woff = reinterpret_cast<int*>(wmax + kABSelectWarps * kABClusters);  // [warps]
  const int I = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nkb = a.nkb, nkb4 = nkb >> 2;
  const int64_t row = bh * a.nqb + I;
  const float* lg = a.logits + (bh * a.nqb * kABClusters + static_cast<int64_t>(I) * kABClusters) * nkb;
  const float4* lg4 = reinterpret_cast<const float4*>(lg);
  // 1. max and normaliser of every centroid's row
  {
    float m[kABClusters];
    double z[kABClusters];
#pragma unroll
    for (int c = 0; c < kABClusters; ++c) {
      m[c] = -INFINITY;
      z[c] = 0.0;
    }
    for (int J4 = tid; J4 < nkb4; J4 += blockDim.x) {
      float4 x[kABClusters];
#pragma unroll
      for (int c = 0; c < kABClusters; ++c) x[c] = __ldg(lg4 + static_cast<int64_t>(c) * nkb4 + J4);
#pragma unroll
      for (int c = 0; c < kABClusters; ++c) {
        const float mn = fmaxf(m[c], fmaxf(fmaxf(x[c].x, x[c].y), fmaxf(x[c].z, x[c].w)));
        double zc = mn > m[c] ? z[c] * static_cast<double>(expf(m[c] - mn)) : z[c];
        zc += static_cast<double>(expf(x[c].x - mn));
        zc += static_cast<double>(expf(x[c].y - mn));
        zc += static_cast<double>(expf(x[c].z - mn));
        zc += static_cast<double>(expf(x[c].w - mn));
        z[c] = zc;
        m[c] = mn;
      }
    }
#pragma unroll
    for (int c = 0; c < kABClusters; ++c) {
      float mw = m[c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, o));
      // a lane that saw no element (m = -inf) adds nothing
      double t = m[c] == -INFINITY ? 0.0 : z[c] * static_cast<double>(expf(m[c] - mw));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) {
        wmax[warp * kABClusters + c] = mw;
        wsum[warp * kABClusters + c] = t;
      }
    }
  }
  __syncthreads();
  if (tid < kABClusters) {
    const int c = tid;
    float M = -INFINITY;
    for (int w = 0; w < kABSelectWarps; ++w) M = fmaxf(M, wmax[w * kABClusters + c]);
    double Z = 0.0;
    for (int w = 0; w < kABSelectWarps; ++w) {
      const float mw = wmax[w * kABClusters + c];
      if (mw != -INFINITY) Z += wsum[w * kABClusters + c] * static_cast<double>(expf(mw - M));
    }
    const int n = a.counts[row * kABClusters + c];
    cmax[c] = M;
    cinv[c] = n > 0 ? static_cast<float>(static_cast<double>(n) / kABQBlock / Z) : 0.f;
  }
  __syncthreads();
  // 2. block scores
  float mloc[kABClusters], wloc[kABClusters];
#pragma unroll
  for (int c = 0; c < kABClusters; ++c) {
    mloc[c] = cmax[c];
    wloc[c] = cinv[c];
  }
  double tot = 0.0;
  float4* sc4 = reinterpret_cast<float4*>(sc);
  for (int J4 = tid; J4 < nkb4; J4 += blockDim.x) {
    float4 x[kABClusters];
#pragma unroll
    for (int c = 0; c < kABClusters; ++c) x[c] = __ldg(lg4 + static_cast<int64_t>(c) * nkb4 + J4);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < kABClusters; ++c)
      if (wloc[c] > 0.f) {
        s.x = __fmaf_rn(wloc[c], expf(x[c].x - mloc[c]), s.x);
        s.y = __fmaf_rn(wloc[c], expf(x[c].y - mloc[c]), s.y);
        s.z = __fmaf_rn(wloc[c], expf(x[c].z - mloc[c]), s.z);
        s.w = __fmaf_rn(wloc[c], expf(x[c].w - mloc[c]), s.w);
      }
    sc4[J4] = s;
    tot += s.x;
    tot += s.y;
    tot += s.z;
    tot += s.w;
  }
  tot = block_sum_f64(tot, red);  // begins with a barrier: every score is written
  int npos = 0;
  for (int J = tid; J < nkb; J += blockDim.x) npos += sc[J] > 0.f;
  npos = block_sum_int(npos, red);
  // 3. water-filling
  double lambda = INFINITY;
  if (a.budget < static_cast<double>(npos) && tot > 0.0) {
    lambda = a.budget / tot;
    int capped = 0;
    for (int round = 0; round < 64; ++round) {
      int c1 = 0;
      double rest = 0.0;
      for (int J = tid; J < nkb; J += blockDim.x) {
        const double s = sc[J];
        if (lambda * s >= 1.0)
          ++c1;
        else
          rest += s;
      }
      c1 = block_sum_int(c1, red);
      rest = block_sum_f64(rest, red);
      if (c1 == capped && round > 0) break;
      capped = c1;
      if (rest <= 0.0 || c1 >= npos) {
        lambda = INFINITY;
        break;
      }
      lambda = (a.budget - c1) / rest;
    }
  }
  // 4. sampling and compaction: warp w owns J in [w * seg, (w + 1) * seg)
  const float* u = a.u + row * nkb;
  int32_t* oidx = a.kidx + row * nkb;
  float* osh = a.kshift + row * nkb;
  const int seg = (nkb + kABSelectWarps * 32 - 1) / (kABSelectWarps * 32) * 32;
  const int j0 = warp * seg, j1 = min(nkb, j0 + seg);
  auto sampled = [&](int J, double& pi) {
    const double s = sc[J];
    pi = s <= 0.0 ? 0.0 : fmin(1.0, lambda * s);
    return static_cast<double>(u[J]) < pi;
  };
  int mine = 0;
  for (int b0 = j0; b0 < j1; b0 += 32) {
    const int J = b0 + lane;
    double pi = 0.0;
    const bool inc = J < j1 && sampled(J, pi);
    mine += __popc(__ballot_sync(0xffffffffu, inc));
  }
  if (lane == 0) woff[warp] = mine;
  __syncthreads();
  int base = 0, total = 0;
  for (int w = 0; w < kABSelectWarps; ++w) {
    base += w < warp ? woff[w] : 0;
    total += woff[w];
  }
  for (int b0 = j0; b0 < j1; b0 += 32) {
    const int J = b0 + lane;
    double pi = 0.0;
    const bool inc = J < j1 && sampled(J, pi);
    const unsigned bal = __ballot_sync(0xffffffffu, inc);
    if (inc) {
      const int pos = base + __popc(bal & ((1u << lane) - 1u));
      oidx[pos] = J;
      osh[pos] = static_cast<float>(-log(pi));
    }
    base += __popc(bal);
  }
  if (tid == 0) a.kcount[row] = total;
}

inline size_t ab_select_smem(int nkb) {
  return static_cast<size_t>((nkb + 3) & ~3) * 4 + 8 * 8 + kABSelectWarps * kABClusters * 8 + 8 * 4 * 2 +
         kABSelectWarps * kABClusters * 4 + kABSelectWarps * 4;
}

}  // namespace nabla
