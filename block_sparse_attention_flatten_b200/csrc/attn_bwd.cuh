// Backward pass of the block-sparse attention, the parts around the tensor-
// core kernels of attn_bwd_tc.cuh: the transposed (column) block lists the
// key-block walk needs, and Delta = rowsum(dO * O) (the summary's "Aceleracao
// de Dupla Fase": NABLA speeds up pre-training and fine-tuning, which run
// this pass).  For query token a and every token c of its row's kept
// blocks, with P = softmax of the scaled logits (recomputed from the
// forward's LSE):
//   dP = dO_a . v_c,   dS = P (dP - Delta_a),   Delta_a = dO_a . O_a,
//   dV_c += P dO_a,    dQ_a += scale dS k_c,    dK_c += scale dS q_a.
#pragma once

#include "common.cuh"

namespace nabla {

// ------------------------------------------------------- transposed lists
// Column lists: for key block j of (b, head), the query blocks i whose row
// lists j, ascending.  Block counts above kTransposeMaxNb: one warp per key
// block; lane l tests rows base + l by
// a binary search of the row's (ascending) list, and a ballot compacts the
// hits in order.  Rows whose count is out of range are treated as empty and
// reported.
__global__ void __launch_bounds__(256) transpose_lists_kernel(const int32_t* __restrict__ kv_count,
                                                              const int32_t* __restrict__ kv_idx,
                                                              int32_t* __restrict__ q_count,
                                                              int32_t* __restrict__ q_idx, int Nb) {
  const int lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (j >= Nb) return;
  const int64_t bh = blockIdx.y;
  const int32_t* cnt = kv_count + bh * Nb;
  const int32_t* lists = kv_idx + bh * static_cast<int64_t>(Nb) * Nb;
  int32_t* out = q_idx + (bh * Nb + j) * static_cast<int64_t>(Nb);
  int n = 0;
  for (int base = 0; base < Nb; base += 32) {
    const int i = base + lane;
    bool hit = false;
    if (i < Nb) {
      int c = cnt[i];
      if (c < 0 || c > Nb) {
        if (j == 0) report(NABLA_ERR_DEVICE_BOUNDS);
        c = 0;
      }
      const int32_t* l = lists + static_cast<int64_t>(i) * Nb;
      int lo = 0, hi = c;  // first entry >= j in [lo, hi)
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (l[mid] < j) lo = mid + 1; else hi = mid;
      }
      hit = lo < c && l[lo] == j;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    if (hit) out[n + __popc(bal & ((1u << lane) - 1u))] = i;
    n += __popc(bal);
  }
  if (lane == 0) q_count[bh * Nb + j] = n;
}

// Column lists by 32 x 32 bit-tile transposes: one CTA per (32 key blocks
// j0 .. j0+31, b, head).  Each thread takes rows i = tid, tid + 256, ...:
// a binary search for the first entry >= j0 of the row's list, then the
// entries below j0 + 32 set bits of a 32-bit row mask (shared memory, one
// word per row).  Then warp w builds columns j0 + w, j0 + w + 8, ...: per
// group of 32 rows, lane l holds row 32g + l's mask, a ballot of bit (j -
// j0) gives the group's hits in row order, and their indices are written
// ascending.  One binary search per (row, 32 columns) instead of per (row,
// column).  Shared memory: Nb words.
constexpr int kTransposeMaxNb = 49152;  // 192 KB of row masks
__global__ void __launch_bounds__(256) transpose_lists_tiled_kernel(const int32_t* __restrict__ kv_count,
                                                                    const int32_t* __restrict__ kv_idx,
                                                                    int32_t* __restrict__ q_count,
                                                                    int32_t* __restrict__ q_idx, int Nb) {
  extern __shared__ uint32_t rowmask[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j0 = blockIdx.x * 32;
  const int64_t bh = blockIdx.y;
  const int32_t* cnt = kv_count + bh * Nb;
  const int32_t* lists = kv_idx + bh * static_cast<int64_t>(Nb) * Nb;
  for (int i = threadIdx.x; i < Nb; i += blockDim.x) {
    int c = __ldg(cnt + i);
    if (c < 0 || c > Nb) {
      if (j0 == 0) report(NABLA_ERR_DEVICE_BOUNDS);
      c = 0;
    }
    const int32_t* l = lists + static_cast<int64_t>(i) * Nb;
    int lo = 0, hi = c;  // first entry >= j0 in [lo, hi)
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(l + mid) < j0) lo = mid + 1; else hi = mid;
    }
    uint32_t m = 0u;
    for (; lo < c; ++lo) {
      const int j = __ldg(l + lo);
      if (j >= j0 + 32 || j >= Nb) break;
      if (j >= j0) m |= 1u << (j - j0);
    }
    rowmask[i] = m;
  }
  __syncthreads();
  for (int b = warp; b < 32; b += blockDim.x >> 5) {
    const int j = j0 + b;
    if (j >= Nb) break;
    int32_t* out = q_idx + (bh * Nb + j) * static_cast<int64_t>(Nb);
    int n = 0;
    for (int base = 0; base < Nb; base += 32) {
      const int i = base + lane;
      const bool hit = i < Nb && ((rowmask[i] >> b) & 1u);
      const unsigned bal = __ballot_sync(0xffffffffu, hit);
      if (hit) out[n + __popc(bal & ((1u << lane) - 1u))] = i;
      n += __popc(bal);
    }
    if (lane == 0) q_count[bh * Nb + j] = n;
  }
}

// ------------------------------------------------------------------ Delta
// Delta[b][hd][a] = sum_d dO[b,a,hd,d] * O[b,a,hd,d] (fp32, d ascending in
// chunks of 8 then a butterfly over the head's chunks).  One warp per token
// row; a head's D/8 chunks (8 or 16) sit on consecutive lanes.
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ dout,
                                                        float* __restrict__ delta, int64_t rows, int S, int Hh,
                                                        int D) {
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int chunks = Hh * D / 8, cph = D / 8;
  const uint4* po = reinterpret_cast<const uint4*>(o) + r * chunks;
  const uint4* pg = reinterpret_cast<const uint4*>(dout) + r * chunks;
  const int64_t b = r / S, a = r - b * S;
  for (int base = 0; base < chunks; base += 32) {
    const int c = base + lane;
    float acc = 0.f;
    if (c < chunks) {
      const uint4 x = __ldg(po + c), y = __ldg(pg + c);
      const __nv_bfloat162* hx = reinterpret_cast<const __nv_bfloat162*>(&x);
      const __nv_bfloat162* hy = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fx = __bfloat1622float2(hx[e]), fy = __bfloat1622float2(hy[e]);
        acc = fmaf(fx.x, fy.x, acc);
        acc = fmaf(fx.y, fy.y, acc);
      }
    }
    for (int off = cph >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (c < chunks && (c & (cph - 1)) == 0) {
      const int hd = c / cph;
      delta[(b * Hh + hd) * S + a] = acc;
    }
  }
}

struct BwdArgs {
  const __nv_bfloat16 *q, *k, *v, *dout;  // [B][S][Hh][D], flattened order
  const float* lse;                       // [B][Hh][S] (natural log)
  const float* delta;                     // [B][Hh][S]
  const int32_t *kv_count, *kv_idx;       // row lists
  const int32_t *q_count, *q_idx;         // column lists
  __nv_bfloat16 *dq, *dk, *dv;            // [B][S][Hh][D]
  int S, Hh, Nb;
  float scale, scale_log2;                // scale, scale * log2(e)
  // grid order (W > 0): tensors, LSE and Delta indexed by grid rows of a
  // T x H x W grid; W = 0: flattened order
  int H, W, nbw, per_t;
};

}  // namespace nabla
