// Adaptive block mask (NABLA technical summary, "Metodologia: NABLA", item 2
// "Construcao de Mascara Adaptativa" and item 3 "Integracao Hibrida com STA").
//
// pool_kernel         Downsampling: per 64-token block the fp32 mean of the
//                     flattened queries and keys (Q and K read once from
//                     HBM), optionally fused with their fractal flattening.
// score_tile_kernel   Reduced attention scores s_ij = (qbar_i . kbar_j) *
//                     scale as a tiled fp32 GEMM (128 x 128 tiles, the
//                     oracle's FMA chain per entry) into a score scratch.
// select_rows_kernel  Per row (one warp): softmax numerators, the CDF
//                     threshold, STA union and block-CSR compaction.
// mask_rows_smem_kernel  Both stages in one kernel with the score rows in
//                     shared memory (no scratch), for callers without one.
// sta_lists_kernel, radial_lists_kernel  The static windows alone as lists.
// The selection (select_row) never forms p = e / sum(e) and never sorts the
// row: the order of e is the order of p, the masses are the e themselves
// summed in fp64 in a fixed order, and the boundary element (e*, j*) of the
// ascending (e, j) order is found by threshold masses (register-only
// predicated sums) narrowing an interval of bit patterns whose elements are
// compacted into a shrinking candidate set, then a warp sort of the last
// <= 32; keep = (e, j) >= (e*, j*) OR arg-max OR a static window.
#pragma once

#include "common.cuh"

namespace nabla {

// ------------------------------------------------------------------ pooling
// grid (Nb, B, 2 * slices), kPoolThreads threads: z & 1 = 0 pools Q into
// qbar^T, 1 pools K into kbar^T, both [B][Hh][D][Nbp] (Nbp = Nb rounded up
// to a multiple of 4; the padding columns are never written); z >> 1 is the
// CTA's slice of kPoolThreads 16-byte chunks of a token row.  Thread c of
// the row handles elements 8c..8c+7 (Hh*D elements), summing the block's 64
// rows in ascending flattened order in fp32, with the next 8 rows' loads
// in flight during each 8 rows' sums.  Small CTAs keep many of them per SM
// (the loads in flight set the bandwidth) and split a layer into enough
// CTAs that the last wave is a small fraction.
// kFlatten = false: q, k are already flattened.  kFlatten = true: q, k are in
// grid order and the block's 64 rows are gathered in flattened order; if
// qf_out / kf_out are given the kernel also writes them there (fractal
// flattening fused with the pooling, so Q and K are read once).  Flattened rows 8u..8u+7 of a block are one run of 8
// consecutive grid rows (patch row u).
constexpr int kPoolThreads = 64;
template <bool kFlatten>
__global__ void __launch_bounds__(kPoolThreads, 8) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, __nv_bfloat16* qf_out,
                                                   __nv_bfloat16* kf_out, float* __restrict__ qbar,
                                                   float* __restrict__ kbar, int S, int Hh, int D, int H, int W) {
  const int i = blockIdx.x, b = blockIdx.y;
  const int Nb = S >> 6;
  const int which = blockIdx.z & 1;
  const __nv_bfloat16* x = which == 0 ? q : k;
  float* out = which == 0 ? qbar : kbar;
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
  __nv_bfloat16* flat_out = which == 0 ? qf_out : kf_out;
  uint4* dst = (kFlatten && flat_out != nullptr)
                   ? reinterpret_cast<uint4*>(flat_out) + (batch_rows + static_cast<int64_t>(i) * 64) * chunks
                   : nullptr;
  // rows r0..r0+7: flattened order; in grid order one run of 8 along w
  auto load8 = [&](uint4 (&v)[8], int r0, int c) {
    const int64_t src_row = kFlatten ? static_cast<int64_t>(r0 >> 3) * W : r0;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = kFlatten ? __ldcs(base + (src_row + u) * chunks + c) : __ldg(base + (src_row + u) * chunks + c);
  };
  {
    const int c = (blockIdx.z >> 1) * kPoolThreads + threadIdx.x;
    if (c >= chunks) return;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    // two groups of 8 rows in flight: the next group's loads are issued
    // before this group's sums (the sums stay in ascending row order)
    auto consume = [&](const uint4 (&v)[8], int g) {
      if (kFlatten && dst != nullptr) {
#pragma unroll
        for (int u = 0; u < 8; ++u) dst[static_cast<int64_t>(8 * g + u) * chunks + c] = v[u];
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
    };
    uint4 va[8], vb[8];
    load8(va, 0, c);
#pragma unroll 1
    for (int g = 0; g < 8; g += 2) {
      load8(vb, 8 * (g + 1), c);
      consume(va, g);
      if (g + 2 < 8) load8(va, 8 * (g + 2), c);
      consume(vb, g + 1);
    }
    // transposed, xbar^T [B][Hh][D][Nbp]: the score stages read a d-slice of
    // consecutive blocks as one contiguous run
    const int col = c * 8;
    const int h = col / D, d = col - h * D;
    const int Nbp = (Nb + 3) & ~3;
    float* o = out + ((static_cast<int64_t>(b) * Hh + h) * D + d) * Nbp + i;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[static_cast<int64_t>(e) * Nbp] = acc[e] * (1.f / 64.f);
  }
}

// -------------------------------------------------------------- mask rows
struct MaskArgs {
  const float* qbar;  // pooled queries, transposed: [B][Hh][D][Nbp]
  const float* kbar;  // pooled keys, transposed:    [B][Hh][D][Nbp]
  int32_t* kv_count;  // [B][Hh][Nb]
  int32_t* kv_idx;    // [B][Hh][Nb][Nb]
  int Hh, Nb, D;
  int nbh, nbw;       // blocks per frame row / column
  int sta_rt, sta_rh, sta_rw;  // STA half-widths; sta_on = 0 disables
  int sta_on;
  int radial_r0;      // radial window half-width at temporal distance 0; 0 disables
  int keep_all;       // thr >= 1
  float scale;
  double tau;         // 1 - thr (exact in double)
};

// Temporal band of the radial window: floor(log2(dt + 1)); its spatial
// half-width is r0 >> band (the window halves each time dt + 1 doubles).
__host__ __device__ __forceinline__ int radial_band(int dt) {
  int r = 0;
  while ((dt + 1) >> (r + 1)) ++r;
  return r;
}

// Calls f(j, pos) for every block j of the radial window of block i (frame
// ti, patch row hi, column wi), pos = its position in the ascending list:
// per frame tj the box of half-width r0 >> radial_band(|ti - tj|) around
// (hi, wi), clipped to the grid, entries in (row, column) order.  One warp:
// lane l takes frames l, l + 32, ... (most boxes far from ti are a single
// block, so a frame per lane keeps the lanes busy), the boxes' sizes give
// the positions by a warp prefix sum.  Returns the window's size (every
// lane).
template <class F>
__device__ __forceinline__ int radial_for_each(int ti, int hi, int wi, int nbt, int nbh, int nbw, int r0, int lane,
                                              const F& f) {
  int n = 0;
  for (int t0 = 0; t0 < nbt; t0 += 32) {
    const int tj = t0 + lane;
    int cnt = 0, h0 = 0, w0 = 0, nw = 1;
    if (tj < nbt) {
      const int rho = r0 >> radial_band(abs(ti - tj));
      h0 = max(hi - rho, 0);
      w0 = max(wi - rho, 0);
      const int h1 = min(hi + rho, nbh - 1), w1 = min(wi + rho, nbw - 1);
      nw = w1 - w0 + 1;
      cnt = (h1 - h0 + 1) * nw;
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int pos = n + incl - cnt;
    for (int e = 0, eh = 0, ew = 0; e < cnt; ++e) {
      f((tj * nbh + h0 + eh) * nbw + w0 + ew, pos + e);
      if (++ew == nw) {
        ew = 0;
        ++eh;
      }
    }
    n += __shfl_sync(0xffffffffu, incl, 31);
  }
  return n;
}

constexpr int kMaskThreads = 256;
constexpr int kMaskWarps = kMaskThreads / 32;
constexpr int kMaskCols = 4;  // adjacent key blocks per thread in the in-shared-memory score phase

// Columns of the transposed pooled vectors and row stride of the score
// scratch: Nb rounded up to a multiple of 4, so every row starts 16-byte
// aligned and is read and written as float4.
__host__ __device__ inline int kbar_cols(int Nb) { return (Nb + 3) & ~3; }


// d = a * b + d on two fp32 lanes at once; each lane is one fmaf (round to
// nearest even), so a lane's chain of these equals the scalar fmaf chain.
__device__ __forceinline__ void ffma2(unsigned long long& d, unsigned long long a, unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}
__device__ __forceinline__ unsigned long long dup2(float x) {
  const unsigned long long u = __float_as_uint(x);
  return (u << 32) | u;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The softmax numerator exp(x) correctly rounded to fp32 (evaluated in
// fp64, then rounded once), as the mask's reading of the method defines it.
// CUDA's expf is within 2 ulp of it; the selection below uses expf and
// switches to this value wherever 2 ulp could change a decision.
__device__ __forceinline__ float exp_rounded(float x) { return __double2float_rn(exp(static_cast<double>(x))); }

constexpr uint32_t kOneBits = 0x3F800000u;         // 1.0f
constexpr uint32_t kNearOneBits = kOneBits - 8u;  // within 8 ulp below 1.0
constexpr int kWindowUlps = 8;                    // > 2 ulp (expf) on either side, with margin
constexpr unsigned long long kInfKey = 0x7F800000ull << 32;
constexpr int kSelCap = 1024;                     // candidate slots per warp
// First-pass thresholds: the numerators 2^-1, 2^-2, 2^-4, 2^-7, 2^-11, 2^-16
// (bit patterns descending).
constexpr int kNThr = 6;
__host__ __device__ constexpr uint32_t thr_bits(int k) {
  return static_cast<uint32_t>(127 - (k == 0 ? 1 : k == 1 ? 2 : k == 2 ? 4 : k == 3 ? 7 : k == 4 ? 11 : 16)) << 23;
}

// Shared memory one warp needs to select one row: candidate slots (int32),
// 32 more for the window, the row (Nbp floats).
__host__ __device__ inline size_t select_warp_bytes(int Nb) {
  return kSelCap * 4 + 32 * 4 + static_cast<size_t>(kbar_cols(Nb)) * 4;
}

// Ascending warp bitonic sort of up to 32 (key, mass) pairs (lanes past the
// data hold key ~0), then the key of the first lane whose cumulative mass,
// on top of `base`, exceeds tau_m (~0 if none).
__device__ __forceinline__ unsigned long long sort_and_cross(unsigned long long key, double w, int lane, double base,
                                                             double tau_m, unsigned long long* lane_key,
                                                             double* lane_w) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const unsigned long long okey = __shfl_xor_sync(0xffffffffu, key, stride);
      const double ow = __shfl_xor_sync(0xffffffffu, w, stride);
      const bool up = (lane & size) == 0;
      const bool lower = (lane & stride) == 0;
      if (lower == up ? (okey < key) : (okey > key)) {
        key = okey;
        w = ow;
      }
    }
  }
  double cw = w;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double v = __shfl_up_sync(0xffffffffu, cw, o);
    if (lane >= o) cw += v;
  }
  *lane_key = key;
  *lane_w = w;
  const unsigned hit = __ballot_sync(0xffffffffu, key != ~0ull && base + cw > tau_m);
  return hit ? __shfl_sync(0xffffffffu, key, __ffs(hit) - 1) : ~0ull;
}

// Numerator pass: row[j] <- e_j = exp(s_j - m) for j < Nbp (padding scores
// are -inf, so their e is 0), with the total mass and the masses of the
// numerators at or above each first-pass threshold, all in fp64 in a fixed
// order.  Per element only register arithmetic (predicated adds, no memory
// read-modify-write, no divergence in the common case).  kExact: every e
// is the correctly rounded value, the scores read through score_of (the
// row already holds numerators); otherwise e = expf, except within 8 ulp of
// 1 where the correctly rounded value is used, so the blocks with e == 1
// (the arg-max ties) are exact.  Returns the arg-max (largest j, e == 1).
template <bool kExact, class ScoreFn>
__device__ __forceinline__ int numerator_pass(float* row, int Nb, int Nbp, float m, const ScoreFn& score_of,
                                              double& total, double (&above)[kNThr]) {
  const int lane = threadIdx.x & 31;
  float4* row4 = reinterpret_cast<float4*>(row);
  total = 0.0;
#pragma unroll
  for (int k = 0; k < kNThr; ++k) above[k] = 0.0;
  int amax = -1;
  for (int c = lane; c < (Nbp >> 2); c += 32) {
    float ev[4];
    if (kExact) {
#pragma unroll
      for (int t = 0; t < 4; ++t) ev[t] = 4 * c + t < Nb ? score_of(4 * c + t) : -INFINITY;
    } else {
      const float4 v = row4[c];
      ev[0] = v.x;
      ev[1] = v.y;
      ev[2] = v.z;
      ev[3] = v.w;
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float x = __fsub_rn(ev[t], m);
      float e = kExact ? exp_rounded(x) : expf(x);
      uint32_t u = __float_as_uint(e);
      if (!kExact && u >= kNearOneBits) {
        e = exp_rounded(x);
        u = __float_as_uint(e);
      }
      ev[t] = e;
      amax = u == kOneBits ? 4 * c + t : amax;
      const double w = static_cast<double>(e);
      total += w;
      // selects, not branches: lanes disagree on every comparison
#pragma unroll
      for (int k = 0; k < kNThr; ++k) above[k] += u >= thr_bits(k) ? w : 0.0;
    }
    row4[c] = make_float4(ev[0], ev[1], ev[2], ev[3]);
  }
  total = warp_sum_f64(total);
#pragma unroll
  for (int k = 0; k < kNThr; ++k) above[k] = warp_sum_f64(above[k]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __syncwarp();
  return amax;
}

// Writes, in ascending j, the indices of the elements whose bit pattern lies
// in [lo, hi) to cbuf (first kSelCap of them) and returns their count.
// `from_row`: scan the whole row; otherwise cbuf[0..n) (compacted in place:
// a write never overtakes the reads of its chunk).
__device__ __forceinline__ int compact_range(const float* row, int* cbuf, int Nbp, bool from_row, int n, uint32_t lo,
                                             uint32_t hi) {
  const int lane = threadIdx.x & 31;
  int out = 0;
  if (from_row) {
    // four 32-element chunks per step, lane l taking element 32u + l of
    // chunk u: ballots give the ascending positions, the chunks' loads are
    // independent and only the running count links the steps
    const unsigned below_me = (1u << lane) - 1u;
    for (int base = 0; base < Nbp; base += 128) {
      bool in[4];
      unsigned bal[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = base + 32 * u + lane;
        const uint32_t v = j < Nbp ? __float_as_uint(row[j]) : 0u;
        in[u] = j < Nbp && v >= lo && v < hi;
        bal[u] = __ballot_sync(0xffffffffu, in[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int pos = out + __popc(bal[u] & below_me);
        if (in[u] && pos < kSelCap) cbuf[pos] = base + 32 * u + lane;
        out += __popc(bal[u]);
      }
    }
  } else {
    for (int base = 0; base < n; base += 32) {
      const int x = base + lane;
      int j = -1;
      if (x < n) j = cbuf[x];
      const uint32_t u = j >= 0 ? __float_as_uint(row[j]) : 0u;
      const bool in = j >= 0 && u >= lo && u < hi;
      const unsigned bal = __ballot_sync(0xffffffffu, in);
      __syncwarp();  // every lane has read its slot before any is overwritten
      if (in) cbuf[out + __popc(bal & ((1u << lane) - 1u))] = j;
      out += __popc(bal);
      __syncwarp();
    }
  }
  __syncwarp();
  return out;
}

// The CDF boundary of a row of numerators: the element (e*, j*) of the
// ascending (e, j) order at which the cumulative mass first exceeds tau_m
// (keep (e, j) >= (e*, j*)); returns its key (bits(e) << 32 | j).  The
// first pass's threshold masses give an interval [lo, hi) of bit patterns
// holding bits(e*); its elements are compacted into cbuf, and the interval
// is narrowed by 8 each round (masses and counts of 7 interior thresholds
// over the candidates, then compaction) until at most 32 remain, which are
// sorted in the warp.  More than 32 equal values: the boundary is the
// need-th smallest index among them.  Requires tau_m < total.  On return
// [*rlo, *rhi) is the last interval, *rbelow the mass below it, and when at
// most 32 candidates remained the lanes hold them sorted (lane_key, lane_w).
__device__ __forceinline__ unsigned long long cdf_boundary(const float* row, int* cbuf, int Nbp, double total,
                                                           const double (&above)[kNThr], double tau_m, uint32_t* rlo,
                                                           uint32_t* rhi, double* rbelow, bool* sorted,
                                                           unsigned long long* lane_key, double* lane_w) {
  const int lane = threadIdx.x & 31;
  // the highest threshold with mass below <= tau_m (masses below grow as the
  // threshold falls: the qualifying thresholds are the lowest ones)
  uint32_t lo = 0u, hi = thr_bits(kNThr - 1);
  double below = 0.0;
  bool found = false;
#pragma unroll
  for (int k = 0; k < kNThr; ++k) {
    const double bl = total - above[k];
    if (!found && bl <= tau_m) {
      found = true;
      lo = thr_bits(k);
      below = bl;
      hi = k == 0 ? 0x7F800000u : thr_bits(k > 0 ? k - 1 : 0);
    }
  }
  bool from_row = true;
  int n = compact_range(row, cbuf, Nbp, true, 0, lo, hi);
  from_row = n > kSelCap;
  while (n > 32 && hi - lo > 1u) {
    // masses and counts at or above 7 interior thresholds of [lo, hi)
    const uint32_t width = hi - lo;
    uint32_t th[7];
#pragma unroll
    for (int k = 0; k < 7; ++k)
      th[k] = lo + static_cast<uint32_t>((static_cast<uint64_t>(width) * (k + 1)) >> 3);
    double ab[7], mi = 0.0;
    int cab[7], ci = 0;
#pragma unroll
    for (int k = 0; k < 7; ++k) {
      ab[k] = 0.0;
      cab[k] = 0;
    }
    const int items = from_row ? Nbp : n;
    for (int x = lane; x < items; x += 32) {
      const int j = from_row ? x : cbuf[x];
      const float e = row[j];
      const uint32_t u = __float_as_uint(e);
      const bool in = u >= lo && u < hi;
      const double w = in ? static_cast<double>(e) : 0.0;
      mi += w;
      ci += in;
#pragma unroll
      for (int k = 0; k < 7; ++k) {
        const bool ge = u >= th[k];
        ab[k] += ge ? w : 0.0;
        cab[k] += (in && ge) ? 1 : 0;
      }
    }
    const double mass_in = warp_sum_f64(mi);  // the interval's mass and count
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ci += __shfl_xor_sync(0xffffffffu, ci, o);
    const int cnt_in = ci;
#pragma unroll
    for (int k = 0; k < 7; ++k) {
      ab[k] = warp_sum_f64(ab[k]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cab[k] += __shfl_xor_sync(0xffffffffu, cab[k], o);
    }
    // the highest threshold whose mass below stays <= tau_m (mass below
    // grows with the threshold, so the qualifying ones are a prefix); none:
    // the first sub-interval [lo, th[0])
    uint32_t nlo = lo, nhi = th[0];
    double nbelow = below;
    int ncnt = cnt_in - cab[0];
#pragma unroll
    for (int k = 0; k < 7; ++k) {
      const double bl = below + (mass_in - ab[k]);
      if (bl <= tau_m) {
        nlo = th[k];
        nbelow = bl;
        ncnt = cab[k] - (k < 6 ? cab[k < 6 ? k + 1 : 6] : 0);
        nhi = k < 6 ? th[k < 6 ? k + 1 : 6] : hi;
      }
    }
    lo = nlo;
    hi = nhi;
    below = nbelow;
    if (from_row && ncnt <= kSelCap) {
      n = compact_range(row, cbuf, Nbp, true, 0, lo, hi);
      from_row = false;
    } else if (!from_row) {
      n = compact_range(row, cbuf, Nbp, false, n, lo, hi);
    } else {
      n = ncnt;
    }
  }
  *rlo = lo;
  *rhi = hi;
  *rbelow = below;
  *sorted = n <= 32;
  if (n <= 32) {
    unsigned long long key = ~0ull;
    double w = 0.0;
    if (lane < n) {
      const int j = cbuf[lane];
      const float e = row[j];
      key = (static_cast<unsigned long long>(__float_as_uint(e)) << 32) | static_cast<unsigned>(j);
      w = static_cast<double>(e);
    }
    __syncwarp();
    return sort_and_cross(key, w, lane, below, tau_m, lane_key, lane_w);
  }
  // more than 32 elements share the value lo: the boundary is the need-th
  // smallest index among them (ascending in cbuf when it holds them)
  *lane_key = ~0ull;
  *lane_w = 0.0;
  const double wstar = static_cast<double>(__uint_as_float(lo));
  double needd = floor((tau_m - below) / wstar) + 1.0;
  const int need = needd < 1.0 ? 1 : (needd > static_cast<double>(n) ? n : static_cast<int>(needd));
  int jstar = -1;
  if (!from_row) {
    jstar = cbuf[need - 1];
  } else {
    int seen = 0;
    for (int base = 0; base < Nbp && jstar < 0; base += 32) {
      const int j = base + lane;
      const bool hit = j < Nbp && __float_as_uint(row[j]) == lo;
      const unsigned bal = __ballot_sync(0xffffffffu, hit);
      const int c = __popc(bal);
      if (seen + c >= need) {
        unsigned bb = bal;
        for (int t = seen + 1; t < need; ++t) bb &= bb - 1;  // drop lower hits
        jstar = base + __ffs(bb) - 1;
      }
      seen += c;
    }
  }
  return (static_cast<unsigned long long>(lo) << 32) | static_cast<unsigned>(jstar);
}

// Selects the kept blocks of query block i from its scores, one warp:
//   1. m = max_j s_j;
//   2. e_j = exp(s_j - m) (numerator_pass), their total and threshold
//      masses in fp64; the arg-max;
//   3. the CDF boundary (cdf_boundary) on these e;
//   4. exactness: e_j differs from the correctly rounded value by at most
//      2 ulp, so the order statistics shift by at most 2 ulp and only blocks
//      within 8 ulp of the boundary value B can be ordered differently.
//      Those (taken from the last interval, or by one more pass) get the
//      correctly rounded e (scores re-read through score_of) and are sorted
//      again on top of the mass below B - 8 ulp: the boundary is then the
//      one of the exact order.  (More than 32 such blocks: the whole row is
//      recomputed exactly and searched again.)
//   5. static windows (STA, radial) marked +inf, then keep = (e, j) >=
//      (e*, j*), the arg-max, or a window, compacted ascending with ballots.
// row: Nbp scores in shared memory, -inf past Nb; overwritten.  cbuf:
// kSelCap candidate slots; cand: 32 slots.
template <class ScoreFn>
__device__ __forceinline__ void select_row(float* row, int* cbuf, int* cand, int Nb, int i, const MaskArgs& a,
                                           int32_t* out, int32_t* count_out, const ScoreFn& score_of) {
  const int lane = threadIdx.x & 31;
  const int Nbp = kbar_cols(Nb);
  const float4* row4 = reinterpret_cast<const float4*>(row);
  float m = -INFINITY;
  for (int c = lane; c < (Nbp >> 2); c += 32) {
    const float4 v = row4[c];
    m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

  double total, above[kNThr];
  int argmax = numerator_pass<false>(row, Nb, Nbp, m, score_of, total, above);
  double tau_m = a.tau * total;
  unsigned long long kstar = kInfKey;  // thr = 0: the CDF keeps nothing but the arg-max
  if (!a.keep_all && total > tau_m) {
    uint32_t lo, hi;
    double below, lw;
    bool sorted;
    unsigned long long lkey;
    const unsigned long long kfast =
        cdf_boundary(row, cbuf, Nbp, total, above, tau_m, &lo, &hi, &below, &sorted, &lkey, &lw);
    const uint32_t B = static_cast<uint32_t>(kfast >> 32);
    const uint32_t wlo = B - kWindowUlps, whi = B + kWindowUlps;
    double base = 0.0;
    int nw = 0;
    unsigned long long wkey = ~0ull;
    if (kfast != ~0ull) {
      if (sorted && wlo >= lo && whi < hi) {
        // the last interval held every block of the window, sorted in lkey/lw
        const uint32_t u = static_cast<uint32_t>(lkey >> 32);
        const bool inw = lkey != ~0ull && u >= wlo && u <= whi;
        base = below + warp_sum_f64(lkey != ~0ull && u < wlo ? lw : 0.0);
        const unsigned bal = __ballot_sync(0xffffffffu, inw);
        nw = __popc(bal);
        if (inw) cand[__popc(bal & ((1u << lane) - 1u))] = static_cast<int>(lkey & 0xffffffffu);
      } else {
        double ml = 0.0;
        for (int base_j = 0; base_j < Nbp; base_j += 32) {
          const int j = base_j + lane;
          const float e = j < Nbp ? row[j] : 0.f;
          const uint32_t u = __float_as_uint(e);
          if (u < wlo) ml += static_cast<double>(e);
          const bool inw = j < Nbp && u >= wlo && u <= whi;
          const unsigned bal = __ballot_sync(0xffffffffu, inw);
          if (inw && nw + __popc(bal & ((1u << lane) - 1u)) < 32) cand[nw + __popc(bal & ((1u << lane) - 1u))] = j;
          nw += __popc(bal);
        }
        base = warp_sum_f64(ml);
      }
    }
    __syncwarp();
    if (kfast == ~0ull) {
      // fp64 rounding put the crossing just past the last candidate (a band
      // case): keep what lies above the interval
      kstar = static_cast<unsigned long long>(hi) << 32;
    } else if (nw <= 32) {
      double w = 0.0;
      if (lane < nw) {
        const int j = cand[lane];
        const float e = j < Nb ? exp_rounded(__fsub_rn(score_of(j), m)) : 0.f;  // padding stays 0
        row[j] = e;
        const uint32_t u = __float_as_uint(e);
        wkey = (static_cast<unsigned long long>(u) << 32) | static_cast<unsigned>(j);
        w = static_cast<double>(e);
      }
      __syncwarp();
      unsigned long long k2;
      double w2;
      kstar = sort_and_cross(wkey, w, lane, base, tau_m, &k2, &w2);
      if (kstar == ~0ull) kstar = kfast;  // crossing outside the window: a band block, either is allowed
    } else {
      // many blocks within a few ulp of the boundary: exact numerators for the
      // whole row, then the search again (no window step needed)
      argmax = numerator_pass<true>(row, Nb, Nbp, m, score_of, total, above);
      tau_m = a.tau * total;
      kstar = kInfKey;
      if (total > tau_m) {
        kstar = cdf_boundary(row, cbuf, Nbp, total, above, tau_m, &lo, &hi, &below, &sorted, &lkey, &lw);
        if (kstar == ~0ull) kstar = static_cast<unsigned long long>(hi) << 32;
      }
    }
    __syncwarp();
  }

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
  if (a.radial_r0 > 0) {
    const int per_t = a.nbh * a.nbw;
    const int ti = i / per_t, hi = (i - ti * per_t) / a.nbw, wi = i - ti * per_t - hi * a.nbw;
    radial_for_each(ti, hi, wi, Nb / per_t, a.nbh, a.nbw, a.radial_r0, lane,
                    [row](int j, int) { row[j] = __uint_as_float(0x7F800000u); });
    __syncwarp();
  }
  // four 32-block chunks per step: their loads and ballots are independent,
  // only the running count links the steps
  int count = 0;
  const unsigned below_me = (1u << lane) - 1u;
  for (int base_j = 0; base_j < Nb; base_j += 128) {
    bool keep[4];
    unsigned bal[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = base_j + 32 * u + lane;
      keep[u] = false;
      if (j < Nb) {
        const unsigned long long key =
            (static_cast<unsigned long long>(__float_as_uint(row[j])) << 32) | static_cast<unsigned>(j);
        keep[u] = a.keep_all || key >= kstar || j == argmax;
      }
      bal[u] = __ballot_sync(0xffffffffu, keep[u]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (keep[u]) out[count + __popc(bal[u] & below_me)] = base_j + 32 * u + lane;
      count += __popc(bal[u]);
    }
  }
  if (lane == 0) *count_out = count;
  __syncwarp();
}

// ------------------------------------------------- scores as a tiled GEMM
// s_ij = (qbar_i . kbar_j) * scale for a 128 x 128 tile of one (b, head), in
// the oracle's arithmetic: per (i, j) one fp32 fused multiply-add chain over
// d ascending (two lanes per fma.rn.f32x2, each rounding like fmaf), then one
// fp32 multiply.  256 threads; thread (ty, tx) = (tid / 16, tid % 16) owns
// rows {4ty..4ty+3, 64+4ty..64+4ty+3} and columns {4tx..4tx+3,
// 64+4tx..64+4tx+3}.  32-deep slices of qbar^T and kbar^T are staged in
// shared memory by cp.async (two stages, zero fill past Nbp); each d step
// reads 4 x 16 bytes of shared memory per thread for 64 multiply-adds.
// Scores go to the scratch, per (b, head) [nrows][out_ld]; for the mask
// [Nb][Nbp] (columns Nb..Nbp are padding).
constexpr int kScoreTile = 128;
constexpr int kScoreKc = 32;
constexpr int kScoreThreads = 256;
constexpr int kScoreStageFloats = 2 * kScoreKc * kScoreTile;
constexpr size_t kScoreSmemBytes = 2 * kScoreStageFloats * sizeof(float);

// Shapes of one score GEMM: rows of A = qT columns, rows of B = kT
// columns; both operands transposed ([D][ld] per (b, head)), the output
// [nrows][out_ld] per (b, head).  Leading dimensions are multiples of 4.
struct ScoreShape {
  int nrows, ncols, D;
  int q_ld, k_ld, out_ld;
  int64_t q_bh, k_bh, out_bh;  // element strides between (b, head) slices
};

__global__ void __launch_bounds__(kScoreThreads, 2)
    score_tile_kernel(const float* __restrict__ qT, const float* __restrict__ kT, float* __restrict__ scores,
                      const ScoreShape sh, float scale) {
  extern __shared__ __align__(16) float ssm[];
  const int j0 = blockIdx.x * kScoreTile, i0 = blockIdx.y * kScoreTile;
  const int64_t bh = blockIdx.z;
  const int D = sh.D;
  const float* qs = qT + bh * sh.q_bh;
  const float* ks = kT + bh * sh.k_bh;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;

  auto load_stage = [&](int st, int d0) {
    float* dst = ssm + st * kScoreStageFloats;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = tid + u * kScoreThreads;  // 16-byte chunk: [Q|K][dd][col4]
      const int which = c >> 10, rem = c & 1023;
      const int dd = rem >> 5, col = (rem & 31) * 4;
      const int g = (which ? j0 : i0) + col;
      const int ld = which ? sh.k_ld : sh.q_ld;
      const bool ok = g < ld;  // ld % 4 == 0: the chunk is wholly in or out
      const float* src = (which ? ks : qs) + static_cast<int64_t>(d0 + dd) * ld + (ok ? g : 0);
      cp_async16_zfill(dst + which * kScoreKc * kScoreTile + dd * kScoreTile + col, src, ok);
    }
    cp_async_commit();
  };

  unsigned long long acc[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0ull;

  const int nk = D / kScoreKc;
  load_stage(0, 0);
  if (nk > 1) load_stage(1, kScoreKc);
  for (int kc = 0; kc < nk; ++kc) {
    if (kc + 1 < nk)
      cp_async_wait<1>();
    else
      cp_async_wait<0>();
    __syncthreads();
    const float* sq = ssm + (kc & 1) * kScoreStageFloats;
    const float* sk = sq + kScoreKc * kScoreTile;
#pragma unroll 4
    for (int dd = 0; dd < kScoreKc; ++dd) {
      const float4 qa = *reinterpret_cast<const float4*>(sq + dd * kScoreTile + ty * 4);
      const float4 qb = *reinterpret_cast<const float4*>(sq + dd * kScoreTile + 64 + ty * 4);
      const ulonglong2 ka = *reinterpret_cast<const ulonglong2*>(sk + dd * kScoreTile + tx * 4);
      const ulonglong2 kb = *reinterpret_cast<const ulonglong2*>(sk + dd * kScoreTile + 64 + tx * 4);
      const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const unsigned long long qq = dup2(qv[r]);
        ffma2(acc[r][0], ka.x, qq);
        ffma2(acc[r][1], ka.y, qq);
        ffma2(acc[r][2], kb.x, qq);
        ffma2(acc[r][3], kb.y, qq);
      }
    }
    __syncthreads();
    if (kc + 2 < nk) load_stage(kc & 1, (kc + 2) * kScoreKc);
  }

  auto lo32 = [](unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v)); };
  auto hi32 = [](unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); };
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int row = i0 + (r < 4 ? ty * 4 + r : 64 + ty * 4 + (r - 4));
    if (row >= sh.nrows) continue;
    float* dst = scores + bh * sh.out_bh + static_cast<int64_t>(row) * sh.out_ld;
    const int ca = j0 + tx * 4, cb = j0 + 64 + tx * 4;
    if (ca < sh.out_ld)
      *reinterpret_cast<float4*>(dst + ca) =
          make_float4(__fmul_rn(lo32(acc[r][0]), scale), __fmul_rn(hi32(acc[r][0]), scale),
                      __fmul_rn(lo32(acc[r][1]), scale), __fmul_rn(hi32(acc[r][1]), scale));
    if (cb < sh.out_ld)
      *reinterpret_cast<float4*>(dst + cb) =
          make_float4(__fmul_rn(lo32(acc[r][2]), scale), __fmul_rn(hi32(acc[r][2]), scale),
                      __fmul_rn(lo32(acc[r][3]), scale), __fmul_rn(hi32(acc[r][3]), scale));
  }
}

// Launches score_tile_kernel for every (b, head) slice.
inline cudaError_t launch_score_tiles(const float* qT, const float* kT, float* out, const ScoreShape& sh, int bhs,
                                      float scale, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(score_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kScoreSmemBytes));
  if (e != cudaSuccess) return e;
  const dim3 grid((sh.ncols + kScoreTile - 1) / kScoreTile, (sh.nrows + kScoreTile - 1) / kScoreTile,
                  static_cast<unsigned>(bhs));
  score_tile_kernel<<<grid, kScoreThreads, kScoreSmemBytes, stream>>>(qT, kT, out, sh, scale);
  return cudaGetLastError();
}

// ------------------------------------------------ selection from the scratch
// One warp per row of the score scratch (rows taken in reverse order of the
// score kernel's writes, so the first ones read are still in L2).  Shared
// memory per warp: select_warp_bytes(Nb).
__global__ void __launch_bounds__(256, 1) select_rows_kernel(const MaskArgs a, const float* __restrict__ scores,
                                                          int64_t rows_total) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int Nb = a.Nb, Nbp = kbar_cols(Nb);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  unsigned char* mine = smem_raw + static_cast<size_t>(warp) * select_warp_bytes(Nb);
  int* cbuf = reinterpret_cast<int*>(mine);
  int* cand = cbuf + kSelCap;
  float* row = reinterpret_cast<float*>(cand + 32);
  const int64_t lin = static_cast<int64_t>(blockIdx.x) * nwarps + warp;
  if (lin >= rows_total) return;
  const int64_t rid = rows_total - 1 - lin;
  const int64_t bh = rid / Nb;
  const int i = static_cast<int>(rid - bh * Nb);
  const float* src = scores + rid * Nbp;
  const float4* src4 = reinterpret_cast<const float4*>(src);
  float4* row4 = reinterpret_cast<float4*>(row);
  for (int c = lane; c < (Nbp >> 2); c += 32) {
    float4 v = __ldcs(src4 + c);
    if (4 * c + 3 >= Nb) {
      if (4 * c + 0 >= Nb) v.x = -INFINITY;
      if (4 * c + 1 >= Nb) v.y = -INFINITY;
      if (4 * c + 2 >= Nb) v.z = -INFINITY;
      if (4 * c + 3 >= Nb) v.w = -INFINITY;
    }
    row4[c] = v;
  }
  __syncwarp();
  select_row(row, cbuf, cand, Nb, i, a, a.kv_idx + (bh * Nb + i) * static_cast<int64_t>(Nb), a.kv_count + bh * Nb + i,
             [src](int j) { return src[j]; });
}

// ------------------------------------- rows with their scores in shared memory
// The whole mask stage in one kernel, without a score scratch (used where no
// scratch can be had): R query-block rows per CTA, 256 threads.  Score
// phase: each thread owns four adjacent key blocks and all R rows; per
// (row, block) the same fused multiply-add chain as score_tile_kernel, two
// blocks per fma.rn.f32x2, qbar held in shared memory as duplicated pairs,
// kbar^T read from global memory two or four d ahead.  Then each warp
// selects rows warp, warp + 8, ... with select_row (exact numerators near
// the boundary from a scalar recomputation of the same chain).
// Shared memory: q pairs [D][R], score rows [R][Nbp], per-warp selection
// scratch (candidate slots; the rows are the score rows).
template <int R>
__global__ void __launch_bounds__(kMaskThreads, 1) mask_rows_smem_kernel(const MaskArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int D = a.D, Nb = a.Nb, Nbp = kbar_cols(Nb);
  unsigned long long* qd = reinterpret_cast<unsigned long long*>(smem_raw);  // [D][R]
  float* rows = reinterpret_cast<float*>(qd + static_cast<size_t>(R) * D);    // [R][Nbp]
  unsigned char* sel = reinterpret_cast<unsigned char*>(rows + static_cast<size_t>(R) * Nbp);

  const int i0 = blockIdx.x * R;
  const int hd = blockIdx.y, b = blockIdx.z;
  const int64_t bh = static_cast<int64_t>(b) * a.Hh + hd;
  const float* qt = a.qbar + bh * static_cast<int64_t>(D) * Nbp;  // qbar^T [D][Nbp]
  const float* kt = a.kbar + bh * static_cast<int64_t>(D) * Nbp;  // kbar^T [D][Nbp]
  const int tid = threadIdx.x, warp = tid >> 5;

  for (int e = tid; e < R * D; e += kMaskThreads) {
    const int d = e / R, r = e - d * R;
    qd[d * R + r] = dup2((i0 + r < Nb) ? qt[static_cast<int64_t>(d) * Nbp + i0 + r] : 0.f);
  }
  __syncthreads();

  for (int j = tid * kMaskCols; j < Nbp; j += kMaskThreads * kMaskCols) {
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
        const unsigned long long* qrow = qd + (d0 + u) * R;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          ffma2(acc[r][0], kv[u].x, qrow[r]);
          ffma2(acc[r][1], kv[u].y, qrow[r]);
        }
      }
#pragma unroll
      for (int u = 0; u < PF; ++u) kv[u] = kn[u];
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float* row = rows + static_cast<size_t>(r) * Nbp;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const unsigned long long v = acc[r][c >> 1];
        row[j + c] = j + c < Nb ? __fmul_rn(__uint_as_float(static_cast<uint32_t>(c & 1 ? v >> 32 : v)), a.scale)
                                : -INFINITY;
      }
    }
  }
  __syncthreads();

  int* cbuf = reinterpret_cast<int*>(sel + static_cast<size_t>(warp) * (kSelCap + 32) * 4);
  int* cand = cbuf + kSelCap;
  for (int r = warp; r < R; r += kMaskWarps) {
    const int i = i0 + r;
    if (i >= Nb) break;
    const int rr = r;
    auto score_of = [&](int j) {
      float acc = 0.f;
      for (int d = 0; d < D; ++d)
        acc = __fmaf_rn(__uint_as_float(static_cast<uint32_t>(qd[d * R + rr])), kt[static_cast<int64_t>(d) * Nbp + j], acc);
      return __fmul_rn(acc, a.scale);
    };
    select_row(rows + static_cast<size_t>(r) * Nbp, cbuf, cand, Nb, i, a,
               a.kv_idx + (bh * Nb + i) * static_cast<int64_t>(Nb), a.kv_count + bh * Nb + i, score_of);
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

// ------------------------------------------------------ radial window lists
// The radial decay window on its own (the Radial Attention article's static
// mask, "Zastosowanie zasad rozkladu energii"): row i lists, ascending, the
// blocks of every frame tj within r0 >> floor(log2(|ti - tj| + 1)) patch
// rows and columns of block i.  Walking the frames in order and each
// frame's clipped box row by row visits the flattened indices in ascending
// order, so entry positions are running offsets.  One warp per query block
// writes its row into every (b, head) copy blockIdx.y, blockIdx.y +
// gridDim.y, ...
__global__ void __launch_bounds__(256) radial_lists_kernel(int32_t* __restrict__ kv_count,
                                                           int32_t* __restrict__ kv_idx, int copies, int Nb, int nbh,
                                                           int nbw, int r0) {
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (i >= Nb) return;
  const int per_t = nbh * nbw;
  const int ti = i / per_t, hi = (i - ti * per_t) / nbw, wi = i - ti * per_t - hi * nbw;
  for (int c = blockIdx.y; c < copies; c += gridDim.y) {
    int32_t* out = kv_idx + (static_cast<int64_t>(c) * Nb + i) * Nb;
    const int n = radial_for_each(ti, hi, wi, Nb / per_t, nbh, nbw, r0, lane, [out](int j, int pos) { out[pos] = j; });
    if (lane == 0) kv_count[static_cast<int64_t>(c) * Nb + i] = n;
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
