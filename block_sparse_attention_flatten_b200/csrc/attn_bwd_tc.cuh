// Backward pass of the block-sparse attention on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory, operands by TMA): the same
// gradients as attn_bwd.cuh (the summary's "Aceleracao de Dupla Fase": NABLA
// speeds up pre-training and fine-tuning, which run this pass), with
// P = softmax of the scaled logits recomputed from the forward's LSE:
//   dP = dO . v,  dS = P (dP - Delta),  dV += P^T dO,  dQ += dS K,
//   dK += dS^T Q  (dQ and dK times the scale).
//
// bwd_dq_tc_kernel    one CTA per pair of query blocks (128 rows, M = 128),
//                     walking the union of their row lists (a key block
//                     listed by one half is masked for the other half's
//                     rows): S = Q K^T and dP = dO V^T into tensor memory,
//                     P and dS by 16 elementwise warps, dQ += dS K.
// bwd_dkdv_tc_kernel  one CTA per pair of key blocks (128 key rows),
//                     walking the union of their column lists:
//                     S^T = K Q^T, dP^T = V dO^T, P^T and dS^T elementwise,
//                     dV += P^T dO and dK += dS^T Q, both accumulated in
//                     tensor memory across the walk.
// Unlike the forward's softmax the elementwise step has no row reduction
// (the LSE is known), so four threads share a row: warps w, w + 4, w + 8,
// w + 12 read the same 32 tensor-memory lanes (rows), columns 16q .. 16q+15
// for quarter q = w / 4.  Their bf16 results go back into the first 8 of
// the columns they read, which the next MMA reads as its A operand (K = 16
// keys per step = one quarter, so the quarters need not be adjacent).
// Sixteen elementwise warps keep four per scheduler, so one warp's wait on
// a tensor-memory load hides behind the others' arithmetic.
// Warp roles (608 threads, one CTA per SM: 512 tensor-memory columns):
//   warps 0-15 elementwise, then the epilogue (row r = 32 (w % 4) + lane,
//              column quarter w / 4);
//   warp 16    TMA producer (one thread; dK/dV kernel: the warp, for the LSE
//              and Delta values it copies);
//   warp 17    MMA issuer of the two products of a tile (S and dP);
//   warp 18    MMA issuer of the accumulating products (dQ; dV and dK).
// Every wait is bounded (see common.cuh); a timeout raises the CTA's abort
// flag, every role drains and the tensor memory is freed.
#pragma once

#include "attn_bwd.cuh"
#include "attn_fwd.cuh"
#include "common.cuh"

namespace nabla {

constexpr int kBwdTcThreads = 608;
constexpr int kBwdTcElemThreads = 512;  // warps 0-15

struct BwdTcArgs {
  const int32_t* row_count;  // lists walked by the CTA: dQ kernel the row lists, dK/dV the column lists
  const int32_t* row_idx;
  const float* lse;    // [B][Hh][S] (natural log)
  const float* delta;  // [B][Hh][S]
  __nv_bfloat16* out0;  // dQ (dQ kernel) or dK (dK/dV kernel), [B][S][Hh][D]
  __nv_bfloat16* out1;  // dV (dK/dV kernel)
  int S, Hh, Nb;
  int grid_H, grid_W;   // > 0: tensors in grid order of a T x H x W grid
  int in_T, in_nbw, in_per_t;
  float scale, scale_log2;
};

// Token row (flattened order inside block j; grid order when grid_W > 0) of
// row r of block j.
__device__ __forceinline__ int64_t bwd_tc_row(const BwdTcArgs& a, int j, int r) {
  if (a.grid_W <= 0) return static_cast<int64_t>(j) * 64 + r;
  const int nbw = a.grid_W >> 3, per_t = (a.grid_H >> 3) * nbw;
  const int t = j / per_t, rem = j - t * per_t, bh = rem / nbw, bw = rem - bh * nbw;
  return (static_cast<int64_t>(t) * a.grid_H + bh * 8 + (r >> 3)) * a.grid_W + bw * 8 + (r & 7);
}

template <int D, int WS>
struct BwdTcSmem {
  static constexpr int kChunks = D / 64;
  static constexpr int kPairBytes = 128 * 128 * kChunks;  // 128 rows x D
  static constexpr int kBlkBytes = 64 * 128 * kChunks;    // 64 rows x D
  // fixed pair tiles: (Q, dO) in the dQ kernel, (K, V) in the dK/dV kernel
  static constexpr int kA = 0;
  static constexpr int kB = kA + kPairBytes;
  // kWS stages of the walked blocks: (K, V) or (Q, dO), each 64 rows.  A
  // stage is held from its load until the tile's accumulating MMAs are
  // done, so with two stages the load of tile n + 2 waited for the whole
  // chain of tile n (products, elementwise step, accumulation) and its copy
  // latency sat on the critical path; four stages keep the copies three
  // tiles ahead (192 KB of shared memory at D = 128, one CTA per SM); the
  // launcher falls back to two where the block lists leave no room for four.
  static constexpr int kWS = WS;
  static constexpr int kW0 = kB + kPairBytes;
  static constexpr int kW1 = kW0 + kWS * kBlkBytes;
  // dK/dV: per elementwise warp two slots of its 16 columns' LSE (log2
  // units) and Delta, [16 warps][2][32] fp32
  static constexpr int kLD = kW1 + kWS * kBlkBytes;
  static constexpr int kBars = kLD + 16 * 64 * 4;
  // fixed_full, w_full[kWS], w0_empty[kWS], w1_empty[kWS], s_full[2], e_full[2], acc_done[2], drain
  static constexpr int kNumBars = 1 + 3 * kWS + 2 + 2 + 2 + 1;
  static constexpr int kMisc = kBars + 8 * kNumBars;
  static constexpr int kList = kMisc + 32;
  __host__ __device__ static size_t list_bytes(int Nb) { return (static_cast<size_t>(Nb) * 2 + 15) & ~size_t(15); }
  static size_t bytes(int Nb) {
    const int words = (Nb + 31) / 32;
    return 1024 + kList + list_bytes(Nb) + 2 * static_cast<size_t>(words) * 4;
  }
};

// kDq = true: the dQ kernel; false: the dK/dV kernel.  tmA/tmB are the maps
// of the CTA's fixed pair tiles (Q, dO or K, V), tmC/tmD those of the
// walked blocks (K, V or Q, dO).
template <int D, bool kDq, int WS>
__global__ void __launch_bounds__(kBwdTcThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmD,
                  const BwdTcArgs a) {
  using L = BwdTcSmem<D, WS>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* fixed_full = bars;
  constexpr int kWS = L::kWS;
  uint64_t* w_full = bars + 1;               // [kWS] walked stage landed
  uint64_t* w0_empty = w_full + kWS;         // [kWS] first walked tile (K or Q) free
  uint64_t* w1_empty = w0_empty + kWS;       // [kWS] second walked tile (V or dO) free
  uint64_t* s_full = w1_empty + kWS;         // [2] the tile's two products are in tensor memory
  uint64_t* e_full = s_full + 2;             // [2] elementwise results written (one arrival per warp)
  uint64_t* acc_done = e_full + 2;           // [2] the accumulating products of the tile are done
  uint64_t* drain = acc_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMisc + 4);
  int* list_len = reinterpret_cast<int*>(sm + L::kMisc + 8);
  uint16_t* list = reinterpret_cast<uint16_t*>(sm + L::kList);
  const int Nb = a.Nb;
  const int words = (Nb + 31) >> 5;
  uint32_t* bm = reinterpret_cast<uint32_t*>(sm + L::kList + L::list_bytes(Nb));  // [2][words]
  float* ld_s = reinterpret_cast<float*>(sm + L::kLD);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p = blockIdx.x, hd = blockIdx.y, b = blockIdx.z;
  const int64_t bh = static_cast<int64_t>(b) * a.Hh + hd;
  const int blk0 = 2 * p, blk1 = 2 * p + 1 < Nb ? 2 * p + 1 : -1;

  auto load_block = [&](unsigned char* dst, const CUtensorMap* map, uint64_t* bar, int j, int chunk_stride) {
    if (a.in_nbw > 0) {
      const int t = j / a.in_per_t, rem = j - t * a.in_per_t, bhh = rem / a.in_nbw, bww = rem - bhh * a.in_nbw;
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_5d(dst + c * chunk_stride, map, bar, c * 64, hd, bww * 8, bhh * 8, b * a.in_T + t);
    } else {
      for (int c = 0; c < L::kChunks; ++c) tma_load_4d(dst + c * chunk_stride, map, bar, c * 64, hd, j * 64, b);
    }
  };

  // ---- set-up: barriers, tensor memory, the fixed pair tiles, merged list
  if (tid == 0) {
    mbar_init(fixed_full, 1);
    for (int s = 0; s < kWS; ++s) {
      mbar_init(w_full + s, 1);
      mbar_init(w0_empty + s, 1);
      mbar_init(w1_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(e_full + s, kBwdTcElemThreads / 32);  // one arrival per warp
      mbar_init(acc_done + s, 1);
    }
    mbar_init(drain, 2);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    mbar_arrive_expect_tx(fixed_full, 2 * L::kPairBytes);
    const int b1 = blk1 >= 0 ? blk1 : blk0;  // a missing second block loads the first again (never stored)
    load_block(sm + L::kA, &tmA, fixed_full, blk0, 128 * 128);
    load_block(sm + L::kA + 64 * 128, &tmA, fixed_full, b1, 128 * 128);
    load_block(sm + L::kB, &tmB, fixed_full, blk0, 128 * 128);
    load_block(sm + L::kB + 64 * 128, &tmB, fixed_full, b1, 128 * 128);
  }
  if (warp == 16) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
    if (lane == 0) {
      tma_prefetch_desc(&tmC);
      tma_prefetch_desc(&tmD);
    }
  }
  for (int w = tid; w < 2 * words; w += kBwdTcThreads) bm[w] = 0u;
  __syncthreads();
  // bitmaps of the two lists (bad entries reported and skipped)
  for (int h = 0; h < 2; ++h) {
    const int blk = h == 0 ? blk0 : blk1;
    if (blk < 0) continue;
    int c = __ldg(a.row_count + bh * Nb + blk);
    if (c < 0 || c > Nb) {
      if (tid == 0) report(NABLA_ERR_DEVICE_BOUNDS);
      c = c < 0 ? 0 : Nb;
    }
    const int32_t* src = a.row_idx + (bh * Nb + blk) * static_cast<int64_t>(Nb);
    for (int e = tid; e < c; e += kBwdTcThreads) {
      const int j = __ldg(src + e);
      if (j < 0 || j >= Nb) {
        report(NABLA_ERR_DEVICE_BOUNDS);
        continue;
      }
      atomicOr(bm + h * words + (j >> 5), 1u << (j & 31));
    }
  }
  __syncthreads();
  if (warp == 0) {
    // merged list, ascending; bit 14: listed by the first block of the pair,
    // bit 15: by the second
    int base = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t x0 = w < words ? bm[w] : 0u, x1 = w < words ? bm[words + w] : 0u;
      uint32_t u = x0 | x1;
      const int n = __popc(u);
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int pos = base + incl - n;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        const uint32_t m = 1u << bit;
        list[pos++] = static_cast<uint16_t>((w * 32 + bit) | ((x0 & m) ? 0x4000u : 0u) | ((x1 & m) ? 0x8000u : 0u));
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *list_len = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int L_n = *list_len;
  // tensor memory: products X[2] (S or S^T), Y[2] (dP or dP^T), then the
  // accumulators: dQ (dQ kernel) or dV, dK
  const uint32_t tX0 = tmem, tY0 = tmem + 128, tAcc0 = tmem + 256, tAcc1 = tmem + 384;
  constexpr uint32_t kIdescXY = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, false, true);
  const uint32_t sA = smem_u32(sm + L::kA), sB = smem_u32(sm + L::kB);
  const uint32_t sW0 = smem_u32(sm + L::kW0), sW1 = smem_u32(sm + L::kW1);

  if (warp == 16) {
    // ------------------------------------------------------------ producer
    // dQ: walked (K, V) of each key block; dK/dV: (Q, dO) of each query
    // block.  (The elementwise warps load the walked query blocks' LSE and
    // Delta themselves: in this thread's loop the loads' latency held the
    // copies back to about one block ahead of the MMAs.)
    int issued = 0;
    bool ok = true;
    for (int n = 0; ok && n < L_n; ++n) {
      const int s = n % kWS;
      if (n >= kWS) {
        const bool w0 = mbar_wait(w0_empty + s, ((n / kWS) - 1) & 1, abort_flag);
        const bool w1 = mbar_wait(w1_empty + s, ((n / kWS) - 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, w0 && w1)) {
          ok = false;
          break;
        }
      }
      const int j = static_cast<int>(list[n] & 0x3FFFu);
      if (lane == 0) {
        mbar_arrive_expect_tx(w_full + s, 2 * L::kBlkBytes);
        load_block(sm + L::kW0 + s * L::kBlkBytes, &tmC, w_full + s, j, 64 * 128);
        load_block(sm + L::kW1 + s * L::kBlkBytes, &tmD, w_full + s, j, 64 * 128);
      }
      issued = n + 1;
    }
    if (lane == 0) {
      for (int n = (issued > kWS ? issued - kWS : 0); n < issued; ++n)
        mbar_wait_drain(w_full + n % kWS, (n / kWS) & 1);
      mbar_wait_drain(fixed_full, 0);
    }
  } else if (warp == 17) {
    // -------------------------------------------- the two products of a tile
    // dQ: S = Q K^T (A = Q pair, B = K block), dP = dO V^T.
    // dK/dV: S^T = K Q^T (A = K pair, B = Q block), dP^T = V dO^T.
    if (lane == 0 && L_n > 0) {
      bool ok = mbar_wait(fixed_full, 0, abort_flag);
      tc_fence_after();
      for (int n = 0; ok && n < L_n; ++n) {
        const int s = n & 1, ws = n % kWS;
        if (!mbar_wait(w_full + ws, (n / kWS) & 1, abort_flag)) { ok = false; break; }
        // buffers s hold the previous use's bf16 results until the
        // accumulating MMAs of tile n - 2 have read them
        if (n >= 2 && !mbar_wait(acc_done + s, ((n - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t w0b = sW0 + ws * L::kBlkBytes, w1b = sW1 + ws * L::kBlkBytes;
        const uint32_t tX = tX0 + s * 64, tY = tY0 + s * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t ad = smem_desc_sw128(sA + c * 128 * 128 + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(w0b + c * 64 * 128 + off, 16, 1024);
          umma_bf16_ss(tX, ad, bd, kIdescXY, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t ad = smem_desc_sw128(sB + c * 128 * 128 + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(w1b + c * 64 * 128 + off, 16, 1024);
          umma_bf16_ss(tY, ad, bd, kIdescXY, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full + s);
        // dQ kernel: V is read only here; dK/dV: dO is read again by dV
        if (kDq) umma_commit(w1_empty + ws);
      }
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp == 18) {
    // ------------------------------------------ the accumulating products
    // A operands from tensor memory (bf16 pairs: the 16 key/query columns
    // of quarter q in the buffer's columns 16q .. 16q+7), B operands
    // MN-major from the walked stage.
    if (lane == 0 && L_n > 0) {
      bool ok = true;
      for (int n = 0; ok && n < L_n; ++n) {
        const int s = n & 1, ws = n % kWS;
        if (!mbar_wait(e_full + s, (n >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tX = tX0 + s * 64, tY = tY0 + s * 64;
        const uint32_t w0b = sW0 + ws * L::kBlkBytes, w1b = sW1 + ws * L::kBlkBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t col = kk * 16;
          if (kDq) {
            // dQ += dS K
            const uint64_t bd = smem_desc_sw128(w0b + kk * 16 * 128, 64 * 128, 1024);
            umma_bf16_ts(tAcc0, tX + col, bd, kIdescAcc, (n > 0 || kk > 0) ? 1u : 0u);
          } else {
            // dV += P^T dO, dK += dS^T Q
            const uint64_t bdo = smem_desc_sw128(w1b + kk * 16 * 128, 64 * 128, 1024);
            const uint64_t bq = smem_desc_sw128(w0b + kk * 16 * 128, 64 * 128, 1024);
            umma_bf16_ts(tAcc0, tX + col, bdo, kIdescAcc, (n > 0 || kk > 0) ? 1u : 0u);
            umma_bf16_ts(tAcc1, tY + col, bq, kIdescAcc, (n > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(acc_done + s);
        umma_commit(w0_empty + ws);
        if (!kDq) umma_commit(w1_empty + ws);
      }
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else {
    // ----------------------------------------------------------- elementwise (warps 0-15)
    const int r = 32 * (warp & 3) + lane;  // tensor-memory lane = row of the pair tile
    const int ch = warp >> 2;              // column quarter
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t flag = 0x4000u << (r >> 6);
    // dQ kernel: this row's LSE (log2 units, -inf -> +inf) and Delta
    float L2row = 0.f, drow = 0.f;
    const int myblk = (r >> 6) == 0 ? blk0 : blk1;
    if (kDq && myblk >= 0) {
      const int64_t row = bh * a.S + bwd_tc_row(a, myblk, r & 63);
      const float l = __ldg(a.lse + row);
      L2row = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
      drow = __ldg(a.delta + row);
    }
    // dK/dV: the LSE (log2 units; -inf -> +inf, so P = 0) and Delta of this
    // warp's 16 columns, one walked block ahead: lanes 0-15 load the LSE of
    // columns 16 ch + lane, lanes 16-31 the Delta, into a register; the
    // value is published to the warp's shared slot at the next step
    float* wslot = ld_s + warp * 64;  // [2][32]
    float pre = 0.f;
    auto fetch = [&](int n) {
      if (kDq || n >= L_n) return;
      const int j = static_cast<int>(list[n] & 0x3FFFu);
      const int64_t row = bh * a.S + bwd_tc_row(a, j, ch * 16 + (lane & 15));
      pre = __ldg((lane < 16 ? a.lse : a.delta) + row);
    };
    fetch(0);
    bool ok = true;
    for (int n = 0; n < L_n; ++n) {
      const int s = n & 1;
      if (!kDq) {
        wslot[(n & 1) * 32 + lane] = lane < 16 ? (pre == -INFINITY ? INFINITY : pre * 1.4426950408889634f) : pre;
        __syncwarp();
        fetch(n + 1);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(s_full + s, (n >> 1) & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      const uint32_t tX = tX0 + s * 64 + ch * 16 + lane_off, tY = tY0 + s * 64 + ch * 16 + lane_off;
      uint32_t xv[1][16], yv[1][16];  // this quarter's 16 columns of X and Y
      tmem_ld16(tX, xv[0]);
      tmem_ld16(tY, yv[0]);
      tmem_ld_wait();
      reg_fence16(xv[0]);
      reg_fence16(yv[0]);
      const bool inc = (static_cast<uint32_t>(list[n]) & flag) != 0u;
      const float* lq = wslot + (n & 1) * 32;  // dK/dV: the 16 columns' LSE, then their Delta
      uint32_t pk[8], dk[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        float p0 = 0.f, p1 = 0.f, d0, d1, L0, L1;
        if (kDq) {
          L0 = L1 = L2row;
          d0 = d1 = drow;
        } else {
          L0 = lq[e];
          L1 = lq[e + 1];
          d0 = lq[16 + e];
          d1 = lq[16 + e + 1];
        }
        if (inc) {
          p0 = ex2_approx(fmaf(__uint_as_float(xv[e >> 4][e & 15]), a.scale_log2, -L0));
          p1 = ex2_approx(fmaf(__uint_as_float(xv[e >> 4][(e + 1) & 15]), a.scale_log2, -L1));
        }
        const float ds0 = p0 * (__uint_as_float(yv[e >> 4][e & 15]) - d0);
        const float ds1 = p1 * (__uint_as_float(yv[e >> 4][(e + 1) & 15]) - d1);
        pk[e >> 1] = pack_bf16x2(p0, p1);
        dk[e >> 1] = pack_bf16x2(ds0, ds1);
      }
      if (kDq) {
        tmem_st8(tX, dk);  // dS into the S buffer
      } else {
        tmem_st8(tX, pk);  // P^T into the S^T buffer
        tmem_st8(tY, dk);  // dS^T into the dP^T buffer
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(e_full + s);
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && L_n > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(acc_done + ((L_n - 1) & 1), ((L_n - 1) >> 1) & 1, abort_flag));
    tc_fence_after();
    __syncwarp();
    const bool valid = myblk >= 0;
    const int64_t trow = static_cast<int64_t>(b) * a.S + (valid ? bwd_tc_row(a, myblk, r & 63) : 0);
    const int nacc = kDq ? 1 : 2;
    for (int which = 0; which < nacc; ++which) {
      const uint32_t tacc = (which == 0 ? tAcc0 : tAcc1) + lane_off + ch * (D / 4);
      // dQ kernel: dQ (scaled); dK/dV kernel: which 0 = dV, 1 = dK (scaled)
      const float f = kDq ? a.scale : (which == 0 ? 1.f : a.scale);
      __nv_bfloat16* orow = (kDq ? a.out0 : (which == 0 ? a.out1 : a.out0)) + (trow * a.Hh + hd) * D + ch * (D / 4);
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t ov[16];
        if (ok && L_n > 0) {
          tmem_ld16(tacc + c * 16, ov);
          tmem_ld_wait();
          reg_fence16(ov);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = 0u;
        }
        uint4 w0, w1;
        w0.x = pack_bf16x2(__uint_as_float(ov[0]) * f, __uint_as_float(ov[1]) * f);
        w0.y = pack_bf16x2(__uint_as_float(ov[2]) * f, __uint_as_float(ov[3]) * f);
        w0.z = pack_bf16x2(__uint_as_float(ov[4]) * f, __uint_as_float(ov[5]) * f);
        w0.w = pack_bf16x2(__uint_as_float(ov[6]) * f, __uint_as_float(ov[7]) * f);
        w1.x = pack_bf16x2(__uint_as_float(ov[8]) * f, __uint_as_float(ov[9]) * f);
        w1.y = pack_bf16x2(__uint_as_float(ov[10]) * f, __uint_as_float(ov[11]) * f);
        w1.z = pack_bf16x2(__uint_as_float(ov[12]) * f, __uint_as_float(ov[13]) * f);
        w1.w = pack_bf16x2(__uint_as_float(ov[14]) * f, __uint_as_float(ov[15]) * f);
        if (valid) {
          reinterpret_cast<uint4*>(orow + c * 16)[0] = w0;
          reinterpret_cast<uint4*>(orow + c * 16)[1] = w1;
        }
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 16) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace nabla
