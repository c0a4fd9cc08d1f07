// AB-Attention forward on the sampled 4-token key blocks (news page
// "AB-Attention acelera a geracao de video em ate 2,23x e pula 92% da
// atencao", section "Os tres recursos do AB-Attention": the kernel gathers
// the chosen 4-token blocks by index into full tensor-core tiles, tokens are
// not permuted, and each sampled block's logits are shifted by -log(pi), its
// Horvitz-Thompson weight).
//
// One CTA per 128-query block of one (batch, head) (the page's query block
// is the full M = 128 of tcgen05.mma).  A tile of keys is 16 sampled blocks
// = 64 keys; tile n holds sample entries 16n .. 16n+15, the last one padded
// with zero rows whose shift is -inf (probability 0).
// Warp roles (256 threads, two CTAs per SM):
//   warps 0-3  softmax: thread t = query row t = TMEM lane t; scores of the
//              tile plus the keys' shifts, online max/sum with the lazy O
//              rescale, bf16 P written back into the score buffer's TMEM;
//              epilogue O / l and the LSE.
//   warp 4     K gather (all 32 lanes): each lane copies 16-byte pieces of
//              the tile's K rows with cp.async into the 128-byte-swizzled
//              layout a TMA box would produce, then waits for its copies,
//              fences them for the tensor core's (async) proxy and arrives
//              on the K stage's full barrier.
//   warp 7     V gather, the same for V, and the tile's shifts.
//   warp 5     QK^T issuer (one thread): S = Q K^T (M 128, N 64, K = D).
//   warp 6     PV issuer (one thread): O += P V (M 128, N = D, K 64).
// K and V have rings of their own: a K stage is refilled as soon as its
// QK^T is done, so the gather of tile n+2's keys runs while tile n is in
// the softmax; a V stage (with the tile's shifts, which the softmax reads)
// is refilled once its PV is done.
// Tensor memory per CTA: S0 | S1 (64 columns each, P in their first 32) |
// O (D columns).  Every wait is bounded; see attn_fwd.cuh.
#pragma once

#include "common.cuh"

namespace nabla {

constexpr int kABAttnThreads = 256;

template <int D>
struct ABAttnSmem {
  static constexpr int kChunks = D / 64;
  static constexpr int kStages = 2;
  static constexpr int kQBytes = 128 * 128 * kChunks;
  static constexpr int kKVBytes = 64 * 128 * kChunks;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + kStages * kKVBytes;
  static constexpr int kShift = kV + kStages * kKVBytes;  // [stages][64] fp32, log2 units (with V)
  static constexpr int kBars = kShift + kStages * 64 * 4;
  // q_full, k_full[stages], k_empty[stages], v_full[stages], v_empty[stages],
  // s_full[2], p_full[2], pv_done[2], mma_drain
  static constexpr int kNumBars = 1 + 4 * kStages + 6 + 1;
  static constexpr int kMisc = kBars + 8 * kNumBars;
  static constexpr size_t kBytes = 1024 + kMisc + 32;
};

struct ABAttnArgs {
  const __nv_bfloat16* k;  // [B][S][Hh][D], grid order
  const __nv_bfloat16* v;
  const int32_t* kcount;   // [B][Hh][NQB]
  const int32_t* kidx;     // [B][Hh][NQB][NKB]
  const float* kshift;     // [B][Hh][NQB][NKB], natural log
  __nv_bfloat16* out;      // [B][S][Hh][D]
  float* lse;              // [B][Hh][S] or null
  int S, Hh, nkb;
  float scale_log2;
};

template <int D>
__global__ void __launch_bounds__(kABAttnThreads, 2)
    ab_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const ABAttnArgs a) {
  using L = ABAttnSmem<D>;
  constexpr int kStages = L::kStages;
  constexpr int kRowChunks = D / 8;  // 16-byte pieces of one token's head slice
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kStages;
  uint64_t* v_full = k_empty + kStages;
  uint64_t* v_empty = v_full + kStages;
  uint64_t* s_full = v_empty + kStages;  // [2]
  uint64_t* p_full = s_full + 2;          // [2]
  uint64_t* pv_done = p_full + 2;         // [2]
  uint64_t* mma_drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMisc + 4);
  float* shift_s = reinterpret_cast<float*>(sm + L::kShift);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int I = blockIdx.x, hd = blockIdx.y, b = blockIdx.z;
  const int nqb = a.S / 128;
  const int64_t row = (static_cast<int64_t>(b) * a.Hh + hd) * nqb + I;
  int cnt = __ldg(a.kcount + row);
  if (cnt < 0 || cnt > a.nkb) {
    if (tid == 0) report(NABLA_ERR_DEVICE_BOUNDS);
    cnt = cnt < 0 ? 0 : a.nkb;
  }
  const int n_tiles = (cnt + 15) >> 4;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full + s, 32);  // one arrival per gathering lane
      mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 32);
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 4);  // one arrival per softmax warp
      mbar_init(pv_done + s, 1);
    }
    mbar_init(mma_drain, 2);
    *abort_flag = 0;
    fence_mbar_init();
    if (n_tiles > 0) {
      tma_prefetch_desc(&tmQ);
      mbar_arrive_expect_tx(q_full, L::kQBytes);
      for (int c = 0; c < L::kChunks; ++c) tma_load_4d(sm + L::kQ + c * 128 * 128, &tmQ, q_full, c * 64, hd, I * 128, b);
    }
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem, tS1 = tmem + 64, tO = tmem + 128;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
  const uint32_t sQ = smem_u32(sm + L::kQ), sK = smem_u32(sm + L::kK), sV = smem_u32(sm + L::kV);

  if (warp == 4 || warp == 7) {
    // ------------------------------------------------------ K or V gather
    const bool is_v = warp == 7;
    const int32_t* lst = a.kidx + row * a.nkb;
    const float* shl = a.kshift + row * a.nkb;
    const int64_t tok_stride = static_cast<int64_t>(a.Hh) * D;  // elements between consecutive tokens
    const __nv_bfloat16* base = (is_v ? a.v : a.k) + (static_cast<int64_t>(b) * a.S * a.Hh + hd) * D;
    uint64_t* full = is_v ? v_full : k_full;
    uint64_t* empty = is_v ? v_empty : k_empty;
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % kStages;
      if (n >= kStages && !__all_sync(0xffffffffu, mbar_wait(empty + s, ((n / kStages) - 1) & 1, abort_flag)))
        break;
      int j = -1;
      if (lane < 16) {
        const int e = 16 * n + lane;
        float sh = -INFINITY;
        if (e < cnt) {
          const int jj = __ldg(lst + e);
          if (jj < 0 || jj >= a.nkb) {
            if (!is_v) report(NABLA_ERR_DEVICE_BOUNDS);
          } else {
            j = jj;
            sh = __ldg(shl + e) * 1.4426950408889634f;
          }
        }
        if (is_v) {
          float* sd = shift_s + s * 64 + 4 * lane;
          const float w = j >= 0 ? sh : -INFINITY;
          sd[0] = w;
          sd[1] = w;
          sd[2] = w;
          sd[3] = w;
        }
      }
      unsigned char* dstage = sm + (is_v ? L::kV : L::kK) + s * L::kKVBytes;
      for (int x = lane; x < 64 * kRowChunks; x += 32) {
        const int kr = x / kRowChunks, cc = x - kr * kRowChunks;
        const int jj = __shfl_sync(0xffffffffu, j, kr >> 2);
        const bool valid = jj >= 0;
        const int64_t off = valid ? (static_cast<int64_t>(jj) * 4 + (kr & 3)) * tok_stride + cc * 8 : 0;
        const int dst = (cc >> 3) * (64 * 128) + kr * 128 + (((cc & 7) ^ (kr & 7)) << 4);
        cp_async16_zfill(dstage + dst, base + off, valid);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(full + s);
    }
    cp_async_wait<0>();
  } else if (warp == 5) {
    // ---------------------------------------------------------- QK^T issue
    if (lane == 0 && n_tiles > 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag);
      tc_fence_after();
      for (int n = 0; ok && n < n_tiles; ++n) {
        const int s = n % kStages;
        if (!mbar_wait(k_full + s, (n / kStages) & 1, abort_flag)) { ok = false; break; }
        if (n >= 2 && !mbar_wait(pv_done + (n & 1), ((n - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = sK + s * L::kKVBytes;
        const uint32_t tS = (n & 1) ? tS1 : tS0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t ad = smem_desc_sw128(sQ + c * 128 * 128 + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(kb + c * 64 * 128 + off, 16, 1024);
          umma_bf16_ss(tS, ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full + (n & 1));
        umma_commit(k_empty + s);
      }
      umma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0);
    }
    if (lane == 0 && n_tiles > 0) mbar_wait_drain(q_full, 0);
  } else if (warp == 6) {
    // ------------------------------------------------------------- PV issue
    if (lane == 0 && n_tiles > 0) {
      bool ok = true;
      for (int m = 0; ok && m < n_tiles; ++m) {
        const int s = m % kStages;
        if (!mbar_wait(p_full + (m & 1), (m >> 1) & 1, abort_flag)) { ok = false; break; }
        if (!mbar_wait(v_full + s, (m / kStages) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t pa = (m & 1) ? tS1 : tS0;
        const uint32_t vb = sV + s * L::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = smem_desc_sw128(vb + kk * 16 * 128, 64 * 128, 1024);
          umma_bf16_ts(tO, pa + kk * 8, bd, kIdescPV, (m > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(pv_done + (m & 1));
        umma_commit(v_empty + s);
      }
      umma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0);
    }
  } else {
    // --------------------------------------------------------------- softmax (warps 0-3)
    const int r = tid;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % kStages;
      // the shifts of this tile are published with its V stage's full
      // barrier (that stage is refilled only after this tile's PV, so the
      // barrier cannot run a phase ahead of this wait)
      if (!__all_sync(0xffffffffu, mbar_wait(v_full + s, (n / kStages) & 1, abort_flag) &&
                                       mbar_wait(s_full + (n & 1), (n >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[4][16];
      const uint32_t tS = ((n & 1) ? tS1 : tS0) + lane_off;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16(tS + c * 16, sv[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence16(sv[c]);
      // logits in log2 units plus the keys' shifts, in place, two columns
      // per two-lane FMA
      const float* shs = shift_s + s * 64;
      const unsigned long long sc2 = f2_pack(a.scale_log2, a.scale_log2);
      float mc[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        mc[c] = -INFINITY;
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const unsigned long long sh2 = *reinterpret_cast<const unsigned long long*>(shs + c * 16 + e);
          const unsigned long long x2 = f2_fma((static_cast<unsigned long long>(sv[c][e + 1]) << 32) | sv[c][e], sc2, sh2);
          sv[c][e] = static_cast<uint32_t>(x2);
          sv[c][e + 1] = static_cast<uint32_t>(x2 >> 32);
          mc[c] = fmax3(mc[c], f2_lo(x2), f2_hi(x2));
        }
      }
      const float mx = fmax3(fmaxf(mc[0], mc[1]), mc[2], mc[3]);
      float factor = 1.f;
      bool need = false;
      if (mx > m_run + 8.f) {  // also true while m_run is -inf (unless mx is -inf too)
        factor = ex2_approx(m_run - mx);
        need = (n > 0) && (l_run > 0.f);
        m_run = mx;
      }
      // a row that so far saw only padding keys has m_run = -inf: its
      // probabilities are 0, not exp(-inf - -inf)
      const float mref = m_run == -INFINITY ? 0.f : m_run;
      unsigned long long rs2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[2][16];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float p0 = ex2_approx(__uint_as_float(sv[c][e]) - mref);
          const float p1 = ex2_approx(__uint_as_float(sv[c][e + 1]) - mref);
          rs2[c] = f2_add(rs2[c], f2_pack(p0, p1));
          const int k = c * 8 + e / 2;
          pk[k >> 4][k & 15] = pack_bf16x2(p0, p1);
        }
      const unsigned long long rall = f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3]));
      l_run = l_run * factor + (f2_lo(rall) + f2_hi(rall));
      __syncwarp();
      if (__any_sync(0xffffffffu, need)) {
        if (!__all_sync(0xffffffffu, mbar_wait(pv_done + ((n - 1) & 1), ((n - 1) >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float f = need ? factor : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          uint32_t ov[16];
          tmem_ld16(tO + lane_off + c * 16, ov);
          tmem_ld_wait();
          reg_fence16(ov);
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st16(tO + lane_off + c * 16, ov);
        }
      }
      tmem_st16(tS, pk[0]);
      tmem_st16(tS + 16, pk[1]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + (n & 1));
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && n_tiles > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(pv_done + ((n_tiles - 1) & 1), ((n_tiles - 1) >> 1) & 1, abort_flag));
    tc_fence_after();
    __syncwarp();
    const int64_t tok = static_cast<int64_t>(I) * 128 + r;
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    __nv_bfloat16* orow = a.out + ((static_cast<int64_t>(b) * a.S + tok) * a.Hh + hd) * D;
#pragma unroll 1
    for (int c = 0; c < D / 16; ++c) {
      uint32_t ov[16];
      if (ok && n_tiles > 0) {
        tmem_ld16(tO + lane_off + c * 16, ov);
        tmem_ld_wait();
        reg_fence16(ov);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) ov[e] = 0u;
      }
      uint4 w0, w1;
      w0.x = pack_bf16x2(__uint_as_float(ov[0]) * inv_l, __uint_as_float(ov[1]) * inv_l);
      w0.y = pack_bf16x2(__uint_as_float(ov[2]) * inv_l, __uint_as_float(ov[3]) * inv_l);
      w0.z = pack_bf16x2(__uint_as_float(ov[4]) * inv_l, __uint_as_float(ov[5]) * inv_l);
      w0.w = pack_bf16x2(__uint_as_float(ov[6]) * inv_l, __uint_as_float(ov[7]) * inv_l);
      w1.x = pack_bf16x2(__uint_as_float(ov[8]) * inv_l, __uint_as_float(ov[9]) * inv_l);
      w1.y = pack_bf16x2(__uint_as_float(ov[10]) * inv_l, __uint_as_float(ov[11]) * inv_l);
      w1.z = pack_bf16x2(__uint_as_float(ov[12]) * inv_l, __uint_as_float(ov[13]) * inv_l);
      w1.w = pack_bf16x2(__uint_as_float(ov[14]) * inv_l, __uint_as_float(ov[15]) * inv_l);
      reinterpret_cast<uint4*>(orow + c * 16)[0] = w0;
      reinterpret_cast<uint4*>(orow + c * 16)[1] = w1;
    }
    if (a.lse != nullptr)
      a.lse[(static_cast<int64_t>(b) * a.Hh + hd) * a.S + tok] =
          l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace nabla
