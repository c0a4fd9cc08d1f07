// Adaptive block mask (NABLA technical summary, "Metodologia: NABLA", item 2
// "Construcao de Mascara Adaptativa" and item 3 "Integracao Hibrida com STA").
//
// pool_kernel       Downsampling: per 64-token block the fp32 mean of the
//                   flattened queries and keys (Q and K read once from HBM),
//                   optionally fused with their fractal flattening.
// mask_rows_kernel  Reduced attention, CDF threshold, STA union and block-CSR
//                   compaction, R query-block rows per CTA:
//   1. scores s_ij = (qbar_i . kbar_j) * scale (fp32 FMA chain over d) into
//      shared memory, one row of Nb scores per query block;
//   2. softmax numerators per row (one warp per row): max, e = expf(s - max);
//      p = e / sum(e) is never formed: the order of e is the order of p, and
//      the masses are integers e * 2^40, so every partial sum is exact and
//      independent of summation order;
//   3. the CDF rule "keep where the ascending cumulative mass exceeds 1 - thr"
//      without a full sort: a search over the fp32 bit patterns of e, two
//      bits per pass, with warp-summed exact masses finds the boundary
//      element (e*, j*) of the ascending (e, j) order (shared-memory
//      histograms with atomics serialise on the few bins most masses fall
//      into);
//   4. keep = (e, j) >= (e*, j*)  OR arg-max  OR STA window, compacted with
//      warp ballots into ascending kv_idx and kv_count.
#pragma once

#include "common.cuh"

namespace nabla {

// ------------------------------------------------------------------ pooling
// grid (Nb, B, 2): z = 0 pools Q into qbar [B][Hh][Nb][D], z = 1 pools K
// into kbar^T [B][Hh][D][Nbp] (Nbp = Nb rounded up to a multiple of 4; the
// padding columns are never written).
// Thread c handles elements 8c..8c+7 of a token row (Hh*D elements), summing
// the block's 64 rows in ascending flattened order in fp32.
// kFlatten = false: q, k are already flattened.  kFlatten = true: q, k are in
// grid order and the block's 64 rows are gathered in flattened order; if
// qf_out / kf_out are given the kernel also writes them there (fractal
// flattening fused with the pooling, so Q and K are read once).  Flattened rows 8u..8u+7 of a block are one run of 8
// consecutive grid rows (patch row u).
template <bool kFlatten>
__global__ void __launch_bounds__(384) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, __nv_bfloat16* qf_out,
                                                   __nv_bfloat16* kf_out, float* __restrict__ qbar,
                                                   float* __restrict__ kbar, int S, int Hh, int D, int H, int W) {
  const int i = blockIdx.x, b = blockIdx.y;
  const int Nb = S >> 6;
  const __nv_bfloat16* x = blockIdx.z == 0 ? q : k;
  float* out = blockIdx.z == 0 ? qbar : kbar;
  const int row = Hh * D;
  const int chunks = row >> 3;
  const int64_t batch_rows = static_cast<int64_t>(b) * S;
  // first grid row of the block's patch (kFlatten) or first flattened row
  int64_t src0 = batch_rows + static_cast<int64_t>(i) * 64;
  if (kFlatten) {
    const int nbw = W >> 3, per_t = (H >> 3) * nbw;
    const int t = i / per_t, rem = i - t * per_t, bh = rem / nbw, bw = rem - bh * nbw;
    src0 = batch_rows + (static_cast<int64_t>(t) * H + bh * 8) * W + bw * 8;
  }
  const uint4* base = reinterpret_cast<const uint4*>(x) + src0 * chunks;
  __nv_bfloat16* flat_out = blockIdx.z == 0 ? qf_out : kf_out;
  uint4* dst = (kFlatten && flat_out != nullptr)
                   ? reinterpret_cast<uint4*>(flat_out) + (batch_rows + static_cast<int64_t>(i) * 64) * chunks
                   : nullptr;
  for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 1
    for (int r0 = 0; r0 < 64; r0 += 8) {
      // rows r0..r0+7: flattened order; in grid order one run of 8 along w
      const int64_t src_row = kFlatten ? static_cast<int64_t>(r0 >> 3) * W : r0;
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = kFlatten ? __ldcs(base + (src_row + u) * chunks + c) : __ldg(base + (src_row + u) * chunks + c);
      if (kFlatten && dst != nullptr) {
#pragma unroll
        for (int u = 0; u < 8; ++u) dst[static_cast<int64_t>(r0 + u) * chunks + c] = v[u];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(h2[e]);
          acc[2 * e] = __fadd_rn(acc[2 * e], f.x);
          acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], f.y);
        }
      }
    }
    const int col = c * 8;
    const int h = col / D, d = col - h * D;
    if (blockIdx.z == 0) {
      float4* o = reinterpret_cast<float4*>(out + ((static_cast<int64_t>(b) * Hh + h) * Nb + i) * D + d);
      o[0] = make_float4(acc[0] * (1.f / 64.f), acc[1] * (1.f / 64.f), acc[2] * (1.f / 64.f), acc[3] * (1.f / 64.f));
      o[1] = make_float4(acc[4] * (1.f / 64.f), acc[5] * (1.f / 64.f), acc[6] * (1.f / 64.f), acc[7] * (1.f / 64.f));
    } else {
      // keys transposed: kbar^T [B][Hh][D][Nbp], so the score phase reads
      // them coalesced along the key blocks
      const int Nbp = (Nb + 3) & ~3;
      float* o = out + ((static_cast<int64_t>(b) * Hh + h) * D + d) * Nbp + i;
#pragma unroll
      for (int e = 0; e < 8; ++e) o[static_cast<int64_t>(e) * Nbp] = acc[e] * (1.f / 64.f);
    }
  }
}

// -------------------------------------------------------------- mask rows
struct MaskArgs {
  const float* qbar;  // [B][Hh][Nb][D]
  const float* kbar;
  int32_t* kv_count;  // [B][Hh][Nb]
  int32_t* kv_idx;    // [B][Hh][Nb][Nb]
  int Hh, Nb, D;
  int nbh, nbw;       // blocks per frame row / column
  int sta_rt, sta_rh, sta_rw;  // STA half-widths; sta_on = 0 disables
  int sta_on;
  int keep_all;       // thr >= 1
  float scale;
  double tau;         // 1 - thr (exact in double)
};

constexpr int kMaskThreads = 256;
constexpr int kMaskWarps = kMaskThreads / 32;
constexpr int kMaskCols = 4;  // adjacent key blocks per thread in the score phase

// Column count of the transposed pooled keys kbar^T [D][Nbp]: Nb rounded up
// to a multiple of 4 so every thread's four columns are an aligned 16-byte
// load.
__host__ __device__ inline int kbar_cols(int Nb) { return (Nb + 3) & ~3; }

// d = a * b + d on two fp32 lanes at once; each lane is one fmaf (round to
// nearest even), so a lane's chain of these equals the scalar fmaf chain.
__device__ __forceinline__ void ffma2(unsigned long long& d, unsigned long long a, unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

// Integer mass of an unnormalised probability e in [0, 1], from its bit
// pattern u: floor(e * 2^40) (exact for e >= 2^-16; smaller masses lose
// < 2^-40 each).  The row's CDF rule "cumulative p > 1 - thr" becomes, with
// p = e / sum(e), "cumulative mass > floor((1 - thr) * total mass)" in exact
// integers, independent of summation order.
__device__ __forceinline__ unsigned long long mass_bits(uint32_t u) {
  const int sh = static_cast<int>(u >> 23) - 110;  // biased exponent - (150 - 40)
  const unsigned long long m24 = (u & 0x7FFFFFu) | 0x800000u;
  return sh >= 0 ? (m24 << sh) : (sh > -24 ? (m24 >> -sh) : 0ull);
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// R query-block rows per CTA, 256 threads.  Shared memory: q pairs [D][R]
// (each fp32 qbar value twice, the second operand of a two-lane FMA), score
// rows [R][Nb], per-warp candidate slots.
template <int R>
__global__ void __launch_bounds__(kMaskThreads, 2) mask_rows_kernel(const MaskArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int D = a.D, Nb = a.Nb, Nbp = kbar_cols(Nb);
  unsigned long long* qd = reinterpret_cast<unsigned long long*>(smem_raw);          // [D][R]
  float* rows = reinterpret_cast<float*>(qd + static_cast<size_t>(R) * D);          // [R][Nb]
  int* cand_all = reinterpret_cast<int*>(rows + static_cast<size_t>(R) * Nb);      // [warps][32]

  const int i0 = blockIdx.x * R;
  const int hd = blockIdx.y, b = blockIdx.z;
  const int64_t bh = static_cast<int64_t>(b) * a.Hh + hd;
  const float* qb = a.qbar + (bh * Nb + i0) * D;
  const float* kt = a.kbar + bh * static_cast<int64_t>(D) * Nbp;  // kbar^T [D][Nbp]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int e = tid; e < R * D; e += kMaskThreads) {
    const int r = e / D, d = e - r * D;
    const uint32_t u = __float_as_uint((i0 + r < Nb) ? qb[e] : 0.f);
    qd[d * R + r] = (static_cast<unsigned long long>(u) << 32) | u;
  }
  __syncthreads();

  // 1. scores: thread owns key blocks j..j+3 and all R rows; per (row, block)
  //    one fused multiply-add chain over d ascending (the oracle's order),
  //    two blocks per instruction.  kbar^T rows are read coalesced (16 bytes
  //    a thread), two or four d ahead of use; each q pair loaded from shared memory
  //    feeds four two-lane FMAs.
  for (int j = tid * kMaskCols; j < Nb; j += kMaskThreads * kMaskCols) {
    unsigned long long acc[R][2];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r][0] = acc[r][1] = 0ull;
    const ulonglong2* kp = reinterpret_cast<const ulonglong2*>(kt + j);
    const int kstride = Nbp / 4;  // in groups of four columns
    constexpr int PF = R >= 16 ? 2 : 4;  // d rows loaded ahead (registers allowing)
    ulonglong2 kv[PF];
#pragma unroll
    for (int u = 0; u < PF; ++u) kv[u] = __ldg(kp + static_cast<int64_t>(u) * kstride);
    for (int d0 = 0; d0 < D; d0 += PF) {
      ulonglong2 kn[PF];
      const bool more = d0 + PF < D;
#pragma unroll
      for (int u = 0; u < PF; ++u)
        kn[u] = more ? __ldg(kp + static_cast<int64_t>(d0 + PF + u) * kstride) : make_ulonglong2(0ull, 0ull);
#pragma unroll
      for (int u = 0; u < PF; ++u) {
        const ulonglong2* qrow = reinterpret_cast<const ulonglong2*>(qd + (d0 + u) * R);
#pragma unroll
        for (int r2 = 0; r2 < R / 2; ++r2) {
          const ulonglong2 qq = qrow[r2];
          ffma2(acc[2 * r2][0], kv[u].x, qq.x);
          ffma2(acc[2 * r2][1], kv[u].y, qq.x);
          ffma2(acc[2 * r2 + 1][0], kv[u].x, qq.y);
          ffma2(acc[2 * r2 + 1][1], kv[u].y, qq.y);
        }
      }
#pragma unroll
      for (int u = 0; u < PF; ++u) kv[u] = kn[u];
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float* row = rows + static_cast<size_t>(r) * Nb;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const unsigned long long v = acc[r][c >> 1];
        if (j + c < Nb) row[j + c] = __uint_as_float(static_cast<uint32_t>(c & 1 ? v >> 32 : v)) * a.scale;
      }
    }
  }
  __syncthreads();

  int* cand = cand_all + warp * 32;
  for (int r = warp; r < R; r += kMaskWarps) {
    const int i = i0 + r;
    if (i >= Nb) break;
    float* row = rows + static_cast<size_t>(r) * Nb;

    // 2. softmax numerators e = exp(s - max) (<= 1), their total integer
    //    mass and the arg-max, in one pass
    float m = -INFINITY;
    for (int j = lane; j < Nb; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    unsigned long long best = 0;  // (bits(e) << 32) | j; max = arg-max, ties to the larger j
    unsigned long long total = 0;
    int n_tiny = 0;  // blocks with e < 2^-63
    // first pass of the boundary search (step 3), on the way: masses and
    // counts of the quarters [2^-63, 2^-47), [2^-47, 2^-31), [2^-31, 2^-15)
    // of the starting range [2^-63, 2)
    unsigned long long fm0 = 0, fm1 = 0, fm2 = 0;
    int fc0 = 0, fc1 = 0, fc2 = 0;
    for (int j = lane; j < Nb; j += 32) {
      const float e = expf(row[j] - m);
      row[j] = e;
      const uint32_t u = __float_as_uint(e);
      const unsigned long long key = (static_cast<unsigned long long>(u) << 32) | static_cast<unsigned>(j);
      best = key > best ? key : best;
      const unsigned long long w = mass_bits(u);
      total += w;
      n_tiny += u < 0x20000000u;
      const uint32_t q = (u - 0x20000000u) >> 27;  // 0..3 for u in [0x20000000, 0x40000000)
      fm0 += q == 0 ? w : 0ull;
      fm1 += q == 1 ? w : 0ull;
      fm2 += q == 2 ? w : 0ull;
      fc0 += q == 0;
      fc1 += q == 1;
      fc2 += q == 2;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long ob = __shfl_xor_sync(0xffffffffu, best, o);
      best = ob > best ? ob : best;
    }
    total = warp_sum_u64(total);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n_tiny += __shfl_xor_sync(0xffffffffu, n_tiny, o);
    const int argmax = static_cast<int>(best & 0xffffffffu);
    const unsigned long long tau_m =
        static_cast<unsigned long long>(floor(a.tau * static_cast<double>(total)));

    // 3. CDF boundary: the element (e*, j*) of the ascending (e, j) order at
    //    which the cumulative mass first exceeds tau_m; keep (e, j) >= it.
    //    bits(e*) is the largest bit pattern x with mass(bits(e) < x) <= tau_m
    //    (positive floats order like their bit patterns).  It is narrowed
    //    inside a range [prefix, prefix + 2^span), two bits per pass: a pass
    //    sums, per quarter of the range, the exact masses and counts of the
    //    blocks in it (warp sums, no atomics; blocks outside the range cost a
    //    compare).  As soon as at most 32 blocks remain in the range they are
    //    sorted by a warp bitonic sort and the boundary is read off their
    //    prefix sums.  Every block with positive mass has e >= 2^-40, so e*
    //    does too and the search starts at [2^-63, 2): bits(e*) has bit 29
    //    set and bit 30 clear, and nothing below 2^-63 carries mass.
    //    When no finite element qualifies (thr = 0: the mass never exceeds
    //    tau_m = total) the boundary is the smallest key of an STA-marked
    //    block, +inf: the CDF then keeps nothing but the arg-max, and the
    //    window is still kept.
    unsigned long long kstar = 0x7F800000ull << 32;
    if (!a.keep_all && total > tau_m) {
      uint32_t prefix = 0x20000000u;
      int span = 29;
      unsigned long long below = 0;  // mass(bits(e) < prefix)
      int n_lo = n_tiny, n_hi = Nb;  // blocks below prefix, below prefix + 2^span
      // Narrows [prefix, prefix + 2^span) to the quarter (of width 2^lo) that
      // holds bits(e*), given the masses and counts of its first three
      // quarters.
      auto narrow = [&](unsigned long long m0, unsigned long long m1, unsigned long long m2, int c0, int c1, int c2,
                        int lo) {
        const unsigned long long s1 = below + m0, s2 = s1 + m1, s3 = s2 + m2;
        if (s3 <= tau_m) {
          prefix += 3u << lo;
          below = s3;
          n_lo += c0 + c1 + c2;
        } else if (s2 <= tau_m) {
          prefix += 2u << lo;
          below = s2;
          n_lo += c0 + c1;
          n_hi = n_lo + c2;
        } else if (s1 <= tau_m) {
          prefix += 1u << lo;
          below = s1;
          n_lo += c0;
          n_hi = n_lo + c1;
        } else {
          n_hi = n_lo + c0;
        }
        span = lo;
      };
      if (n_hi - n_lo > 32) {
        // the first pass was done with the exponentials
        fm0 = warp_sum_u64(fm0);
        fm1 = warp_sum_u64(fm1);
        fm2 = warp_sum_u64(fm2);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          fc0 += __shfl_xor_sync(0xffffffffu, fc0, o);
          fc1 += __shfl_xor_sync(0xffffffffu, fc1, o);
          fc2 += __shfl_xor_sync(0xffffffffu, fc2, o);
        }
        narrow(fm0, fm1, fm2, fc0, fc1, fc2, 27);
      }
      while (span > 0 && n_hi - n_lo > 32) {
        const int lo = span > 2 ? span - 2 : 0;
        const uint32_t range = 1u << span;
        unsigned long long m0 = 0, m1 = 0, m2 = 0;
        int c0 = 0, c1 = 0, c2 = 0;
        for (int j = lane; j < Nb; j += 32) {
          const uint32_t u = __float_as_uint(row[j]);
          const uint32_t d = u - prefix;
          if (d < range) {
            const uint32_t q = d >> lo;
            const unsigned long long w = mass_bits(u);
            m0 += q == 0 ? w : 0ull;
            m1 += q == 1 ? w : 0ull;
            m2 += q == 2 ? w : 0ull;
            c0 += q == 0;
            c1 += q == 1;
            c2 += q == 2;
          }
        }
        m0 = warp_sum_u64(m0);
        m1 = warp_sum_u64(m1);
        m2 = warp_sum_u64(m2);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          c0 += __shfl_xor_sync(0xffffffffu, c0, o);
          c1 += __shfl_xor_sync(0xffffffffu, c1, o);
          c2 += __shfl_xor_sync(0xffffffffu, c2, o);
        }
        narrow(m0, m1, m2, c0, c1, c2, lo);
      }
      const uint32_t range = 1u << span;
      if (n_hi - n_lo <= 32) {
        // gather the blocks of the range (ascending j), then sort them
        int ncand = 0;
        for (int base = 0; base < Nb && ncand < n_hi - n_lo; base += 32) {
          const int j = base + lane;
          const bool hit = j < Nb && __float_as_uint(row[j]) - prefix < range;
          const unsigned bal = __ballot_sync(0xffffffffu, hit);
          const int pos = ncand + __popc(bal & ((1u << lane) - 1u));
          if (hit && pos < 32) cand[pos] = j;
          ncand += __popc(bal);
        }
        __syncwarp();
        unsigned long long key = ~0ull, w = 0ull;
        if (lane < ncand) {
          const int j = cand[lane];
          const uint32_t u = __float_as_uint(row[j]);
          key = (static_cast<unsigned long long>(u) << 32) | static_cast<unsigned>(j);
          w = mass_bits(u);
        }
        // bitonic sort of (key, w) ascending by key across the warp
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
          for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const unsigned long long okey = __shfl_xor_sync(0xffffffffu, key, stride);
            const unsigned long long ow = __shfl_xor_sync(0xffffffffu, w, stride);
            const bool up = (lane & size) == 0;
            const bool lower = (lane & stride) == 0;
            if (lower == up ? (okey < key) : (okey > key)) {
              key = okey;
              w = ow;
            }
          }
        }
        unsigned long long cw = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long v = __shfl_up_sync(0xffffffffu, cw, o);
          if (lane >= o) cw += v;
        }
        // below + (mass of the whole range) > tau_m, so some lane qualifies
        const unsigned hitb = __ballot_sync(0xffffffffu, lane < ncand && below + cw > tau_m);
        kstar = __shfl_sync(0xffffffffu, key, __ffs(hitb) - 1);
      } else {
        // More than 32 blocks share the value e* = prefix: the boundary is
        // the need-th smallest index among them.
        const unsigned long long wstar = mass_bits(prefix);
        const unsigned long long need = (tau_m - below) / wstar + 1ull;
        unsigned long long seen = 0;
        int jstar = Nb;
        for (int base = 0; base < Nb; base += 32) {
          const int j = base + lane;
          const bool hit = j < Nb && __float_as_uint(row[j]) == prefix;
          const unsigned bal = __ballot_sync(0xffffffffu, hit);
          const unsigned c = __popc(bal);
          if (seen + c >= need) {
            unsigned bb = bal;
            for (unsigned long long t = seen + 1; t < need; ++t) bb &= bb - 1;  // drop lower hits
            jstar = base + __ffs(bb) - 1;
            break;
          }
          seen += c;
        }
        kstar = (static_cast<unsigned long long>(prefix) << 32) | static_cast<unsigned>(jstar);
      }
      __syncwarp();
    }

    // 4. union with the STA window: the window's blocks get e = +inf, which
    //    orders above every kept key; then compaction of keep = (e, j) >=
    //    (e*, j*) or arg-max, ascending j
    if (a.sta_on) {
      const int per_t = a.nbh * a.nbw;
      const int nbt = Nb / per_t;
      const int ti = i / per_t, hi = (i - ti * per_t) / a.nbw, wi = i - ti * per_t - hi * a.nbw;
      const int wh = 2 * a.sta_rh + 1, ww = 2 * a.sta_rw + 1, plane = wh * ww;
      const int nwin = (2 * a.sta_rt + 1) * plane;
      for (int e = lane; e < nwin; e += 32) {
        const int et = e / plane, ehw = e - et * plane, eh = ehw / ww;
        const int tj = ti + et - a.sta_rt, hj = hi + eh - a.sta_rh, wj = wi + (ehw - eh * ww) - a.sta_rw;
        if (tj >= 0 && tj < nbt && hj >= 0 && hj < a.nbh && wj >= 0 && wj < a.nbw)
          row[tj * per_t + hj * a.nbw + wj] = __uint_as_float(0x7F800000u);
      }
      __syncwarp();
    }
    int32_t* out = a.kv_idx + (bh * Nb + i) * static_cast<int64_t>(Nb);
    int count = 0;
    for (int base = 0; base < Nb; base += 32) {
      const int j = base + lane;
      bool keep = false;
      if (j < Nb) {
        const unsigned long long key = (static_cast<unsigned long long>(__float_as_uint(row[j])) << 32) | static_cast<unsigned>(j);
        keep = a.keep_all || key >= kstar || j == argmax;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if (keep) out[count + __popc(bal & ((1u << lane) - 1u))] = j;
      count += __popc(bal);
    }
    if (lane == 0) a.kv_count[bh * Nb + i] = count;
  }
}

// ------------------------------------------------ static sliding-tile lists
// The window mask M_STA on its own ("Integracao Hibrida com STA" without the
// content-adaptive term): row i lists the blocks of the window centred on
// block i and truncated at the grid border, ascending.  The truncated window
// is a box [t0,t1] x [h0,h1] x [w0,w1] of block coordinates, and walking it
// frame, patch row, patch column in nested order visits the flattened
// indices (t*nbh + h)*nbw + w in ascending order, so entry e of the list is
// the box's e-th block.  Nothing depends on the data: one warp computes row
// i and writes it into every (b, head) copy blockIdx.y, blockIdx.y +
// gridDim.y, ...; lane e writes entries e, e + 32, ... (coalesced).
__global__ void __launch_bounds__(256) sta_lists_kernel(int32_t* __restrict__ kv_count,
                                                        int32_t* __restrict__ kv_idx, int copies, int Nb,
                                                        int nbh, int nbw, int rt, int rh, int rw) {
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (i >= Nb) return;
  const int per_t = nbh * nbw;
  const int nbt = Nb / per_t;
  const int ti = i / per_t, hi = (i - ti * per_t) / nbw, wi = i - ti * per_t - hi * nbw;
  const int t0 = max(ti - rt, 0), t1 = min(ti + rt, nbt - 1);
  const int h0 = max(hi - rh, 0), h1 = min(hi + rh, nbh - 1);
  const int w0 = max(wi - rw, 0), w1 = min(wi + rw, nbw - 1);
  const int nh = h1 - h0 + 1, nw = w1 - w0 + 1, plane = nh * nw;
  const int count = (t1 - t0 + 1) * plane;
  for (int c = blockIdx.y; c < copies; c += gridDim.y) {
    int32_t* out = kv_idx + (static_cast<int64_t>(c) * Nb + i) * Nb;
    for (int e = lane; e < count; e += 32) {
      const int et = e / plane, r = e - et * plane, eh = r / nw;
      out[e] = ((t0 + et) * nbh + h0 + eh) * nbw + w0 + (r - eh * nw);
    }
    if (lane == 0) kv_count[static_cast<int64_t>(c) * Nb + i] = count;
  }
}

// --------------------------------------------------------- mask validation
__global__ void validate_mask_kernel(const int32_t* __restrict__ kv_count, const int32_t* __restrict__ kv_idx,
                                     int64_t rows, int Nb, int32_t* bad_rows) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const int c = kv_count[r];
  bool bad = c < 1 || c > Nb;
  if (!bad) {
    const int32_t* l = kv_idx + r * Nb;
    int prev = -1;
    for (int e = 0; e < c; ++e) {
      const int j = l[e];
      if (j <= prev || j >= Nb) {
        bad = true;
        break;
      }
      prev = j;
    }
  }
  if (bad) atomicAdd(bad_rows, 1);
}

}  // namespace nabla
