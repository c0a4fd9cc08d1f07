// Backward pass of the block-sparse attention: the gradients dQ, dK, dV of
// the attention on the kept 64 x 64 tiles, over the same block lists as the
// forward (the summary's "Aceleracao de Dupla Fase": NABLA speeds up
// pre-training and fine-tuning too, which run this pass).  For query token a
// and every token c of its row's kept blocks, with P = softmax of the scaled
// logits (recomputed from the forward's LSE):
//   dP = dO_a . v_c,   dS = P (dP - Delta_a),   Delta_a = dO_a . O_a,
//   dV_c += P dO_a,    dQ_a += scale dS k_c,    dK_c += scale dS q_a.
//
// Three kernels, each output element written by exactly one CTA (no atomics,
// deterministic):
//   bwd_delta_kernel  Delta = rowsum(dO * O) per token and head (fp32);
//   bwd_dq_kernel     one CTA per query block: walks the row's kept key
//                     blocks, dQ accumulated in registers;
//   bwd_dkdv_kernel   one CTA per key block: walks the query blocks that keep
//                     it (the transposed lists of transpose_lists_kernel),
//                     dK and dV accumulated in registers.
// The tile products use the warp-level bf16 tensor-core MMA (m16n8k16, fp32
// accumulation) on operands staged in padded shared memory: four warps, 16
// rows of the 64-row block each, operand fragments loaded by ldmatrix.  P
// and dS are rounded to bf16 for the products, as the forward rounds P.  No thread ever waits on another
// except at __syncthreads.
#pragma once

#include "common.cuh"

namespace nabla {

constexpr int kBwdThreads = 128;

// ------------------------------------------------------- transposed lists
// Column lists: for key block j of (b, head), the query blocks i whose row
// lists j, ascending.  One warp per key block; lane l tests rows base + l by
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

// ------------------------------------------------------------ MMA helpers
// D = A * B + D for one m16n8k16 tile: A 16 x 16 row-major, B 16 x 8
// column-major, bf16, fp32 accumulators.  Fragment ownership (g = lane / 4,
// t = lane % 4): a0 (row g, k 2t..2t+1), a1 (row g+8, same k), a2 (row g,
// k 2t+8..), a3 (row g+8, k 2t+8..); b0 (k 2t..2t+1, col g), b1 (k 2t+8..,
// col g); c0, c1 (row g, cols 2t, 2t+1), c2, c3 (row g+8, same cols).  Each
// 32-bit register holds its lower-index element in the low half.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Four 8 x 8 bf16 matrices from shared memory; lanes 8m..8m+7 give the row
// addresses of matrix m (16-byte aligned) and register m receives it:
// without .trans lane (g, t) gets row g, columns 2t and 2t+1 (an A or a
// row-indexed B fragment); with .trans it gets rows 2t and 2t+1 of column g
// (a B fragment of a matrix stored with k along rows).
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const __nv_bfloat16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const __nv_bfloat16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

// Shared-memory row stride of a staged 64 x D tile: D + 8 elements, so rows
// start 16 bytes apart modulo 128 and the eight 16-byte rows of every
// ldmatrix matrix fall in distinct banks.
template <int D>
struct BwdTile {
  static constexpr int kStride = D + 8;
  // dynamic shared memory of the dQ and dK/dV kernels: the CTA's own two
  // tiles, two buffers of the two tiles it walks over, then two buffers of
  // the 64 LSE and Delta values of the dK/dV kernel
  static constexpr size_t kSmemBytes = 6u * 64u * kStride * 2u + 2u * 2u * 64u * 4u;
};

// Row of the r-th token (flattened order inside the block) of a block,
// relative to the block's first token: r itself for flattened tensors; for
// tensors in grid order (W > 0) row r/8 of the 8 x 8 patch, column r%8.
__device__ __forceinline__ int64_t block_row(int r, int W) {
  return W > 0 ? static_cast<int64_t>(r >> 3) * W + (r & 7) : r;
}

// stage_tile with asynchronous copies.
template <int D>
__device__ __forceinline__ void stage_tile_async(__nv_bfloat16* dst, const __nv_bfloat16* src_row0, int row_elems,
                                                 int W) {
  constexpr int kChunks = D / 8;
  for (int x = threadIdx.x; x < 64 * kChunks; x += kBwdThreads) {
    const int r = x / kChunks, c = x - r * kChunks;
    cp_async16(dst + r * BwdTile<D>::kStride + c * 8,
               reinterpret_cast<const uint4*>(src_row0 + block_row(r, W) * row_elems) + c);
  }
}

// Copies a 64-token x D tile of one head (rows of Hh*D elements; first token
// at src_row0) into shared memory with 16-byte loads.
template <int D>
__device__ __forceinline__ void stage_tile(__nv_bfloat16* dst, const __nv_bfloat16* src_row0, int row_elems, int W) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  for (int x = threadIdx.x; x < 64 * kChunks; x += kBwdThreads) {
    const int r = x / kChunks, c = x - r * kChunks;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src_row0 + block_row(r, W) * row_elems) + c);
    *reinterpret_cast<uint4*>(dst + r * BwdTile<D>::kStride + c * 8) = v;
  }
}

// acc[n][.] (16 rows of this warp x 64 columns) = A_w (16 x D, rows of sa
// from row0) times B^T where B is the 64 x D tile sb (column n of the result
// is row n of sb): the "row . row" product used for S = Q K^T and dP = dO V^T
// and their transposes.
// Fragment loads by ldmatrix (lane l, m = l / 8, r = l % 8): A's matrices
// are (rows lo, k lo), (rows hi, k lo), (rows lo, k hi), (rows hi, k hi); a
// B pair covers two column tiles, each (k lo), (k hi).
template <int D>
__device__ __forceinline__ void mma_rows_rows(float (&acc)[8][4], const __nv_bfloat16* sa, int row0,
                                              const __nv_bfloat16* sb, int lane) {
  constexpr int ST = BwdTile<D>::kStride;
  const int m = lane >> 3, r = lane & 7;
#pragma unroll
  for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a[4];
    ldsm_x4(a, sa + (row0 + r + 8 * (m & 1)) * ST + ks * 16 + 8 * (m >> 1));
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t bb[4];
      ldsm_x4(bb, sb + ((2 * np + (m >> 1)) * 8 + r) * ST + ks * 16 + 8 * (m & 1));
      mma_bf16_16816(acc[2 * np], a[0], a[1], a[2], a[3], bb[0], bb[1]);
      mma_bf16_16816(acc[2 * np + 1], a[0], a[1], a[2], a[3], bb[2], bb[3]);
    }
  }
}

// out[n][.] (16 x D) += P (16 x 64, given as fp32 accumulator fragments of
// the 8 column tiles, rounded to bf16 here) times the 64 x D tile sb.
template <int D>
__device__ __forceinline__ void mma_p_tile(float (&out)[D / 8][4], const float (&p)[8][4],
                                           const __nv_bfloat16* sb, int lane) {
  constexpr int ST = BwdTile<D>::kStride;
  const int m = lane >> 3, r = lane & 7;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {  // 16 of the 64 columns of P per step
    const uint32_t a0 = pack2_bf16(p[2 * ks][0], p[2 * ks][1]);
    const uint32_t a1 = pack2_bf16(p[2 * ks][2], p[2 * ks][3]);
    const uint32_t a2 = pack2_bf16(p[2 * ks + 1][0], p[2 * ks + 1][1]);
    const uint32_t a3 = pack2_bf16(p[2 * ks + 1][2], p[2 * ks + 1][3]);
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      uint32_t bb[4];
      ldsm_x4_trans(bb, sb + (ks * 16 + r + 8 * (m & 1)) * ST + (2 * np + (m >> 1)) * 8);
      mma_bf16_16816(out[2 * np], a0, a1, a2, a3, bb[0], bb[1]);
      mma_bf16_16816(out[2 * np + 1], a0, a1, a2, a3, bb[2], bb[3]);
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

// First token (within its batch) of block j.
__device__ __forceinline__ int64_t block_first_token(const BwdArgs& a, int j) {
  if (a.W == 0) return static_cast<int64_t>(j) * 64;
  const int t = j / a.per_t, rem = j - t * a.per_t, bh = rem / a.nbw, bw = rem - bh * a.nbw;
  return (static_cast<int64_t>(t) * a.H + bh * 8) * a.W + bw * 8;
}

// ---------------------------------------------------------------- dQ
// CTA (i, hd, b): query block i.  Warp w owns query rows 16w..16w+15; thread
// (g, t) rows g and g+8 of them.
template <int D>
__global__ void __launch_bounds__(kBwdThreads) bwd_dq_kernel(const BwdArgs a) {
  constexpr int ST = BwdTile<D>::kStride;
  extern __shared__ __align__(16) unsigned char bwd_smem[];
  __nv_bfloat16* sq = reinterpret_cast<__nv_bfloat16*>(bwd_smem);
  __nv_bfloat16* sdo = sq + 64 * ST;
  __nv_bfloat16* skv = sdo + 64 * ST;  // two buffers of (K, V)
  const int i = blockIdx.x, hd = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int row_elems = a.Hh * D;
  const int64_t bh = static_cast<int64_t>(b) * a.Hh + hd;
  const int64_t first = block_first_token(a, i);
  const int64_t tok0 = static_cast<int64_t>(b) * a.S + first;
  stage_tile<D>(sq, a.q + tok0 * row_elems + hd * D, row_elems, a.W);
  stage_tile<D>(sdo, a.dout + tok0 * row_elems + hd * D, row_elems, a.W);
  const int r0 = warp * 16 + g;  // this thread's rows inside the block: r0, r0 + 8
  const int64_t o0 = block_row(r0, a.W), o1 = block_row(r0 + 8, a.W);
  const int64_t lrow = bh * a.S + first;
  const float l0 = a.lse[lrow + o0], l1 = a.lse[lrow + o1];
  const float L0 = l0 == -INFINITY ? INFINITY : l0 * 1.4426950408889634f;
  const float L1 = l1 == -INFINITY ? INFINITY : l1 * 1.4426950408889634f;
  const float d0 = a.delta[lrow + o0], d1 = a.delta[lrow + o1];
  int cnt = a.kv_count[bh * a.Nb + i];
  if (cnt < 0 || cnt > a.Nb) {
    if (threadIdx.x == 0) report(NABLA_ERR_DEVICE_BOUNDS);
    cnt = 0;
  }
  const int32_t* list = a.kv_idx + (bh * a.Nb + i) * static_cast<int64_t>(a.Nb);
  float dq[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;
  // K, V of list entry e go to buffer e & 1: the copies of entry e + 1 are
  // in flight while entry e is multiplied.  A bad entry is reported, not
  // fetched and skipped.
  auto fetch = [&](int e) -> bool {
    const int j = list[e];
    if (j < 0 || j >= a.Nb) {
      if (threadIdx.x == 0) report(NABLA_ERR_DEVICE_BOUNDS);
      return false;
    }
    const int64_t ktok = static_cast<int64_t>(b) * a.S + block_first_token(a, j);
    __nv_bfloat16* bk = skv + (e & 1) * 2 * 64 * ST;
    stage_tile_async<D>(bk, a.k + ktok * row_elems + hd * D, row_elems, a.W);
    stage_tile_async<D>(bk + 64 * ST, a.v + ktok * row_elems + hd * D, row_elems, a.W);
    return true;
  };
  bool ok = cnt > 0 && fetch(0);
  cp_async_commit();
  for (int e = 0; e < cnt; ++e) {
    const bool ok_next = e + 1 < cnt && fetch(e + 1);
    cp_async_commit();
    cp_async_wait_one();  // entry e's copies have landed
    __syncthreads();
    if (!ok) {
      __syncthreads();
      ok = ok_next;
      continue;
    }
    const __nv_bfloat16* sk = skv + (e & 1) * 2 * 64 * ST;
    const __nv_bfloat16* sv = sk + 64 * ST;
    float s[8][4], dp[8][4];
    mma_rows_rows<D>(s, sq, warp * 16, sk, lane);   // S = Q K^T
    mma_rows_rows<D>(dp, sdo, warp * 16, sv, lane);  // dP = dO V^T
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float p0 = exp2f(s[n][0] * a.scale_log2 - L0), p1 = exp2f(s[n][1] * a.scale_log2 - L0);
      const float p2 = exp2f(s[n][2] * a.scale_log2 - L1), p3 = exp2f(s[n][3] * a.scale_log2 - L1);
      s[n][0] = p0 * (dp[n][0] - d0);  // dS
      s[n][1] = p1 * (dp[n][1] - d0);
      s[n][2] = p2 * (dp[n][2] - d1);
      s[n][3] = p3 * (dp[n][3] - d1);
    }
    mma_p_tile<D>(dq, s, sk, lane);  // dQ += dS K
    __syncthreads();  // every warp is done with buffer e & 1 before entry e + 2 is fetched into it
    ok = ok_next;
  }
  __nv_bfloat16* out0 = a.dq + (tok0 + o0) * row_elems + hd * D;
  __nv_bfloat16* out1 = a.dq + (tok0 + o1) * row_elems + hd * D;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int c = n * 8 + 2 * t;
    *reinterpret_cast<uint32_t*>(out0 + c) = pack2_bf16(dq[n][0] * a.scale, dq[n][1] * a.scale);
    *reinterpret_cast<uint32_t*>(out1 + c) = pack2_bf16(dq[n][2] * a.scale, dq[n][3] * a.scale);
  }
}

// -------------------------------------------------------------- dK, dV
// CTA (j, hd, b): key block j.  Warp w owns key rows 16w..16w+15 and works
// on the transposed products (keys as rows): S^T = K Q^T, dP^T = V dO^T,
// dV += P^T dO, dK += dS^T Q.
template <int D>
__global__ void __launch_bounds__(kBwdThreads) bwd_dkdv_kernel(const BwdArgs a) {
  constexpr int ST = BwdTile<D>::kStride;
  extern __shared__ __align__(16) unsigned char bwd_smem[];
  __nv_bfloat16* sk = reinterpret_cast<__nv_bfloat16*>(bwd_smem);
  __nv_bfloat16* sv = sk + 64 * ST;
  __nv_bfloat16* sqdo = sv + 64 * ST;  // two buffers of (Q, dO)
  float* s_ld = reinterpret_cast<float*>(sqdo + 4 * 64 * ST);  // two buffers of (LSE, Delta), raw
  const int j = blockIdx.x, hd = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int row_elems = a.Hh * D;
  const int64_t bh = static_cast<int64_t>(b) * a.Hh + hd;
  const int64_t tok0 = static_cast<int64_t>(b) * a.S + block_first_token(a, j);
  stage_tile<D>(sk, a.k + tok0 * row_elems + hd * D, row_elems, a.W);
  stage_tile<D>(sv, a.v + tok0 * row_elems + hd * D, row_elems, a.W);
  int cnt = a.q_count[bh * a.Nb + j];
  if (cnt < 0 || cnt > a.Nb) {
    if (threadIdx.x == 0) report(NABLA_ERR_DEVICE_BOUNDS);
    cnt = 0;
  }
  const int32_t* list = a.q_idx + (bh * a.Nb + j) * static_cast<int64_t>(a.Nb);
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    dk[n][0] = dk[n][1] = dk[n][2] = dk[n][3] = 0.f;
    dv[n][0] = dv[n][1] = dv[n][2] = dv[n][3] = 0.f;
  }
  // Q, dO, LSE and Delta of list entry e go to buffer e & 1 (as in the dQ
  // kernel, the next entry's copies overlap this entry's products).
  auto fetch = [&](int e) -> bool {
    const int i = list[e];
    if (i < 0 || i >= a.Nb) {
      if (threadIdx.x == 0) report(NABLA_ERR_DEVICE_BOUNDS);
      return false;
    }
    const int64_t qfirst = block_first_token(a, i);
    const int64_t qtok = static_cast<int64_t>(b) * a.S + qfirst;
    __nv_bfloat16* bq = sqdo + (e & 1) * 2 * 64 * ST;
    stage_tile_async<D>(bq, a.q + qtok * row_elems + hd * D, row_elems, a.W);
    stage_tile_async<D>(bq + 64 * ST, a.dout + qtok * row_elems + hd * D, row_elems, a.W);
    const int x = threadIdx.x & 63;  // threads 0-63 copy the LSE, 64-127 Delta
    const int64_t lr = bh * a.S + qfirst + block_row(x, a.W);
    cp_async4(s_ld + (e & 1) * 128 + threadIdx.x, threadIdx.x < 64 ? a.lse + lr : a.delta + lr);
    return true;
  };
  bool ok = cnt > 0 && fetch(0);
  cp_async_commit();
  for (int e = 0; e < cnt; ++e) {
    const bool ok_next = e + 1 < cnt && fetch(e + 1);
    cp_async_commit();
    cp_async_wait_one();  // entry e's copies have landed
    __syncthreads();
    if (!ok) {
      __syncthreads();
      ok = ok_next;
      continue;
    }
    const __nv_bfloat16* sq = sqdo + (e & 1) * 2 * 64 * ST;
    const __nv_bfloat16* sdo = sq + 64 * ST;
    const float* s_l = s_ld + (e & 1) * 128;
    const float* s_d = s_l + 64;
    float s[8][4], dp[8][4];
    mma_rows_rows<D>(s, sk, warp * 16, sq, lane);   // S^T = K Q^T
    mma_rows_rows<D>(dp, sv, warp * 16, sdo, lane);  // dP^T = V dO^T
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int c = n * 8 + 2 * t;  // query columns c, c+1
      const float l0 = s_l[c], l1 = s_l[c + 1], d0 = s_d[c], d1 = s_d[c + 1];
      const float L0 = l0 == -INFINITY ? INFINITY : l0 * 1.4426950408889634f;
      const float L1 = l1 == -INFINITY ? INFINITY : l1 * 1.4426950408889634f;
      const float p0 = exp2f(s[n][0] * a.scale_log2 - L0), p1 = exp2f(s[n][1] * a.scale_log2 - L1);
      const float p2 = exp2f(s[n][2] * a.scale_log2 - L0), p3 = exp2f(s[n][3] * a.scale_log2 - L1);
      s[n][0] = p0;
      s[n][1] = p1;
      s[n][2] = p2;
      s[n][3] = p3;
      dp[n][0] = p0 * (dp[n][0] - d0);  // dS^T
      dp[n][1] = p1 * (dp[n][1] - d1);
      dp[n][2] = p2 * (dp[n][2] - d0);
      dp[n][3] = p3 * (dp[n][3] - d1);
    }
    mma_p_tile<D>(dv, s, sdo, lane);  // dV += P^T dO
    mma_p_tile<D>(dk, dp, sq, lane);  // dK += dS^T Q
    __syncthreads();  // every warp is done with buffer e & 1 before entry e + 2 is fetched into it
    ok = ok_next;
  }
  const int r0 = warp * 16 + g;
  const int64_t o0 = (tok0 + block_row(r0, a.W)) * row_elems + hd * D;
  const int64_t o1 = (tok0 + block_row(r0 + 8, a.W)) * row_elems + hd * D;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int c = n * 8 + 2 * t;
    *reinterpret_cast<uint32_t*>(a.dk + o0 + c) = pack2_bf16(dk[n][0] * a.scale, dk[n][1] * a.scale);
    *reinterpret_cast<uint32_t*>(a.dk + o1 + c) = pack2_bf16(dk[n][2] * a.scale, dk[n][3] * a.scale);
    *reinterpret_cast<uint32_t*>(a.dv + o0 + c) = pack2_bf16(dv[n][0], dv[n][1]);
    *reinterpret_cast<uint32_t*>(a.dv + o1 + c) = pack2_bf16(dv[n][2], dv[n][3]);
  }
}

}  // namespace nabla
