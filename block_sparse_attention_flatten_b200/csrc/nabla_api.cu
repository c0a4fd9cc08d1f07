// C ABI of libnabla.so (declared in include/nabla.h): argument checks, TMA
// descriptor set-up and kernel launches.  Everything here is host code; the
// kernels live in the .cuh files included below (one translation unit, so
// the device status word is a single symbol).
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "ab.cuh"
#include "ab_attn.cuh"
#include "attn_bwd.cuh"
#include "attn_bwd_tc.cuh"
#include "attn_fwd.cuh"
#include "common.cuh"
#include "flatten.cuh"
#include "mask.cuh"
#include "nabla.h"

namespace nabla {
namespace {

constexpr int kMaxDevices = 64;

// NVTX range around one entry point (named after the function), so a
// profiler's timeline shows which library call launched which kernels; a
// no-op unless a tool is attached.
struct NvtxScope {
  explicit NvtxScope(const char* name) { nvtxRangePushA(name); }
  ~NvtxScope() { nvtxRangePop(); }
};
#define NABLA_NVTX_RANGE() ::nabla::NvtxScope nabla_nvtx_scope_(__func__)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
  bool ready = false;
  bool sm100 = false;
  int sms = 0;
  int max_smem_optin = 0;
  int smem_per_sm = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

// Per-device facts, looked up once.
int device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NABLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return NABLA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return NABLA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return NABLA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return NABLA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
      return NABLA_ERR_CUDA;
    d.sm100 = (major == 10 && minor == 0);
    d.ready = true;
  }
  *out = d;
  return NABLA_OK;
}

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? NABLA_OK : NABLA_ERR_CUDA;
}

// ----------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// View of a BSHD bf16 tensor as 4-D (D, Hh, S, B), box (64, 1, rows, 1),
// 128-byte swizzle: one box is `rows` tokens x 64 head-dim elements.
bool make_bshd_map(CUtensorMap* m, const void* base, int B, int S, int Hh, int D, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hh), static_cast<cuuint64_t>(S),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Hh) * D * 2,
                                 static_cast<cuuint64_t>(S) * Hh * D * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Grid-order BSHD tensor [B][T][H][W][Hh][D] seen as 5-D (d, head, w, h,
// frame = b*T + t); the box (64, 1, 8, 8, 1) is one 64-token block of one
// head (an 8 x 8 patch), its pixels row by row, 128-byte swizzled.
bool make_grid_map(CUtensorMap* m, const void* base, int B, int T, int H, int W, int Hh, int D) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(Hh) * D * 2;  // bytes per token
  const cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hh), static_cast<cuuint64_t>(W),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T) * B};
  const cuuint64_t strides[4] = {static_cast<cuuint64_t>(D) * 2, row, row * W, row * W * H};
  const cuuint32_t box[5] = {64, 1, 8, 8, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int check_grid(int B, int T, int H, int W, int P) {
  if (B <= 0 || T <= 0 || H <= 0 || W <= 0) return NABLA_ERR_INVALID;
  if (P != 8 || H % P != 0 || W % P != 0) return NABLA_ERR_INVALID;
  const int64_t S = static_cast<int64_t>(T) * H * W;
  if (S > (int64_t{1} << 30)) return NABLA_ERR_INVALID;
  return NABLA_OK;
}

template <bool kInverse>
int permute(const void* in, void* out, int B, int T, int H, int W, int P, int row_elems, cudaStream_t stream) {
  int rc = check_grid(B, T, H, W, P);
  if (rc != NABLA_OK) return rc;
  if (row_elems <= 0 || row_elems % 8 != 0) return NABLA_ERR_INVALID;
  if (in == nullptr || out == nullptr || in == out) return NABLA_ERR_INVALID;
  if (!aligned16(in) || !aligned16(out)) return NABLA_ERR_ALIGN;
  DeviceInfo di;
  if ((rc = device_info(&di)) != NABLA_OK) return rc;
  const int64_t S = static_cast<int64_t>(T) * H * W;
  const int64_t rows = S * B;
  const int chunks = row_elems / 8;
  const int64_t blocks_needed = (rows + 7) / 8;
  const int grid = static_cast<int>(blocks_needed < int64_t{di.sms} * 16 ? blocks_needed : int64_t{di.sms} * 16);
  permute_rows_kernel<kInverse><<<grid, 256, 0, stream>>>(static_cast<const uint4*>(in), static_cast<uint4*>(out),
                                                           rows, S, GridShape{T, H, W, P}, chunks);
  return launch_status();
}

// Shared memory of mask_rows_smem_kernel<R>: q pairs, R score rows, the
// eight warps' selection scratch.
size_t mask_smem_bytes(int R, int D, int Nb) {
  return static_cast<size_t>(R) * D * 8 + static_cast<size_t>(R) * kbar_cols(Nb) * 4 +
         static_cast<size_t>(kMaskWarps) * (kSelCap + 32) * 4;
}

template <int R>
int launch_mask_smem(const MaskArgs& a, int B, cudaStream_t stream) {
  const size_t smem = mask_smem_bytes(R, a.D, a.Nb);
  if (cudaFuncSetAttribute(mask_rows_smem_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return NABLA_ERR_CUDA;
  dim3 grid((a.Nb + R - 1) / R, a.Hh, B);
  mask_rows_smem_kernel<R><<<grid, kMaskThreads, smem, stream>>>(a);
  return launch_status();
}

// Validated mask configuration shared by the mask entry points.
struct MaskPlan {
  MaskArgs a;
  DeviceInfo di;
  int S, H, W;
  float* scores;  // score scratch [B*Hh][Nb][Nbp] (after the pooled vectors)
};

// Workspace layout: qbar^T, kbar^T (fp32 [B][Hh][D][Nbp] each), then the
// score scratch (fp32 [B][Hh][Nb][Nbp]).
size_t pooled_bytes(int B, int Hh, int D, int Nb) {
  return 2 * static_cast<size_t>(B) * Hh * D * kbar_cols(Nb) * sizeof(float);
}
size_t score_bytes(int B, int Hh, int Nb) {
  return static_cast<size_t>(B) * Hh * Nb * kbar_cols(Nb) * sizeof(float);
}

int mask_plan(int B, int Hh, int D, int T, int H, int W, const nabla_params* params, void* workspace,
              int32_t* kv_count, int32_t* kv_idx, MaskPlan* mp) {
  if (params == nullptr) return NABLA_ERR_INVALID;
  const nabla_params& p = *params;
  int rc = check_grid(B, T, H, W, p.P);
  if (rc != NABLA_OK) return rc;
  if (Hh <= 0 || (D != 64 && D != 128) || p.flags != 0u) return NABLA_ERR_INVALID;
  if (!(p.thr >= 0.f && p.thr <= 1.f)) return NABLA_ERR_INVALID;
  if (!(p.scale >= 0.f) || std::isinf(p.scale)) return NABLA_ERR_INVALID;
  const bool sta_on = p.sta_t != 0 || p.sta_h != 0 || p.sta_w != 0;
  if (sta_on && (p.sta_t <= 0 || p.sta_h <= 0 || p.sta_w <= 0 || p.sta_t % 2 == 0 || p.sta_h % 2 == 0 ||
                 p.sta_w % 2 == 0))
    return NABLA_ERR_INVALID;
  if (p.radial < 0 || p.radial > 65535) return NABLA_ERR_INVALID;
  if (workspace == nullptr) return NABLA_ERR_INVALID;
  if (!aligned16(workspace)) return NABLA_ERR_ALIGN;
  if (static_cast<int64_t>(Hh) * D > 3072 * 4) return NABLA_ERR_INVALID;
  const int S = T * H * W;
  const int Nb = S / 64;
  MaskArgs& a = mp->a;
  a.qbar = static_cast<float*>(workspace);
  a.kbar = const_cast<float*>(a.qbar) + static_cast<size_t>(B) * Hh * D * kbar_cols(Nb);
  mp->scores = const_cast<float*>(a.kbar) + static_cast<size_t>(B) * Hh * D * kbar_cols(Nb);
  a.kv_count = kv_count;
  a.kv_idx = kv_idx;
  a.Hh = Hh;
  a.Nb = Nb;
  a.D = D;
  a.nbh = H / p.P;
  a.nbw = W / p.P;
  a.sta_on = sta_on ? 1 : 0;
  a.sta_rt = p.sta_t / 2;
  a.sta_rh = p.sta_h / 2;
  a.sta_rw = p.sta_w / 2;
  a.radial_r0 = p.radial;
  a.keep_all = p.thr >= 1.f ? 1 : 0;
  a.scale = p.scale > 0.f ? p.scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  a.tau = 1.0 - static_cast<double>(p.thr);  // exact in double
  mp->S = S;
  mp->H = H;
  mp->W = W;
  return NABLA_OK;
}

template <bool kFlatten>
int launch_pool(const MaskPlan& mp, int B, const void* q, const void* k, void* qf, void* kf, cudaStream_t stream) {
  const int chunks = mp.a.Hh * mp.a.D / 8;
  const int slices = (chunks + kPoolThreads - 1) / kPoolThreads;
  if (2 * slices > 65535) return NABLA_ERR_INVALID;
  pool_kernel<kFlatten><<<dim3(mp.a.Nb, B, 2 * slices), kPoolThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(qf),
      static_cast<__nv_bfloat16*>(kf), const_cast<float*>(mp.a.qbar), const_cast<float*>(mp.a.kbar), mp.S, mp.a.Hh,
      mp.a.D, mp.H, mp.W);
  return launch_status();
}

// Mask stages 2-4 on pooled vectors.  With the score scratch: the tiled
// score GEMM, then one warp per row selecting from the scratch.  Without it
// (the no-allocation entry point): the single kernel holding R score rows in
// shared memory, R as large as keeps two CTAs per SM, else as fits.
int launch_mask_rows(const MaskPlan& mp, int B, cudaStream_t stream, bool use_scratch) {
  const int Nb = mp.a.Nb, D = mp.a.D;
  const size_t optin = static_cast<size_t>(mp.di.max_smem_optin);
  if (use_scratch) {
    const int64_t bhs = static_cast<int64_t>(B) * mp.a.Hh;
    if (bhs > 65535) return NABLA_ERR_INVALID;
    const int Nbp = kbar_cols(Nb);
    ScoreShape sh;
    sh.nrows = sh.ncols = Nb;
    sh.D = D;
    sh.q_ld = sh.k_ld = sh.out_ld = Nbp;
    sh.q_bh = sh.k_bh = static_cast<int64_t>(D) * Nbp;
    sh.out_bh = static_cast<int64_t>(Nb) * Nbp;
    if (launch_score_tiles(mp.a.qbar, mp.a.kbar, mp.scores, sh, static_cast<int>(bhs), mp.a.scale, stream) !=
        cudaSuccess)
      return NABLA_ERR_CUDA;
    // warps per CTA: the most warps per SM that the per-warp shared memory
    // allows (each CTA also costs 1 KB of reserved shared memory); on ties
    // the larger CTA
    const size_t per_warp = select_warp_bytes(Nb);
    if (per_warp > optin) return NABLA_ERR_INVALID;
    int wpc = 1, best = 0;
    for (int w = 8; w >= 1; w >>= 1) {
      if (per_warp * w > optin) continue;
      const int ctas = static_cast<int>(static_cast<size_t>(mp.di.smem_per_sm) / (per_warp * w + 1024));
      const int warps = ctas * w > 16 ? 16 : ctas * w;
      if (warps > best) {
        best = warps;
        wpc = w;
      }
    }
    const size_t smem = per_warp * wpc;
    if (cudaFuncSetAttribute(select_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return NABLA_ERR_CUDA;
    const int64_t rows = bhs * Nb;
    select_rows_kernel<<<static_cast<unsigned>((rows + wpc - 1) / wpc), 32 * wpc, smem, stream>>>(mp.a, mp.scores,
                                                                                                rows);
    return launch_status();
  }
  const size_t two_per_sm = optin / 2;
  if (mask_smem_bytes(16, D, Nb) <= two_per_sm) return launch_mask_smem<16>(mp.a, B, stream);
  if (mask_smem_bytes(8, D, Nb) <= two_per_sm) return launch_mask_smem<8>(mp.a, B, stream);
  if (mask_smem_bytes(4, D, Nb) <= optin) return launch_mask_smem<4>(mp.a, B, stream);
  if (mask_smem_bytes(2, D, Nb) <= optin) return launch_mask_smem<2>(mp.a, B, stream);
  if (mask_smem_bytes(1, D, Nb) <= optin) return launch_mask_smem<1>(mp.a, B, stream);
  return NABLA_ERR_INVALID;
}

// Failure-detection self-test: every thread of one CTA waits on an mbarrier
// nothing arrives on, with the kernels' bounded wait and a short limit.
__global__ void wait_timeout_selftest_kernel(long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait_limit(&bar, 0, &abort_flag, limit);
  __syncthreads();
}

// Scratch of nabla_build_mask_noalloc: the pooled queries then keys.  In host
// code this name is only a stand-in for the device symbol; its device address
// comes from cudaGetSymbolAddress with the caller's device current.
__device__ __align__(256) unsigned char g_noalloc_scratch[NABLA_NOALLOC_SCRATCH_BYTES];

// Workspace of the key-range split: the splits' outputs (bf16, the layout
// of O, o_stride elements apart) then their LSE (fp32, the layout of the
// LSE, lse_stride apart), each region 256-byte aligned.
struct AttnSplitLayout {
  int64_t o_stride, lse_stride;
  size_t o_off, lse_off, total;
};
AttnSplitLayout attn_split_layout(int B, int64_t S, int Hh, int D, int nsplit) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  AttnSplitLayout l;
  l.o_stride = static_cast<int64_t>(B) * S * Hh * D;
  l.lse_stride = static_cast<int64_t>(B) * Hh * S;
  l.o_off = 0;
  l.lse_off = up(static_cast<size_t>(l.o_stride) * 2 * nsplit);
  l.total = l.lse_off + up(static_cast<size_t>(l.lse_stride) * 4 * nsplit);
  return l;
}

// Shared body of the two attention entry points; grp_F > 0 selects the 2 x 2
// (w, t) grouping of query blocks (grp_F blocks per frame, grp_nbw per row).
// nsplit > 1: the key-range split, partial outputs in `part` (see
// attn_split_layout), then their merge into out and lse.
int sparse_attn_launch(const void* qf, const void* kf, const void* vf, const int32_t* kv_count,
                       const int32_t* kv_idx, int B, int S, int Hh, int D, float scale, void* out, float* lse,
                       int grp_F, int grp_nbw, int grid_T, int out_H, int out_W, cudaStream_t stream,
                       int nsplit = 1, void* part = nullptr) {
  if (B <= 0 || S <= 0 || Hh <= 0 || S % 64 != 0 || (D != 64 && D != 128)) return NABLA_ERR_INVALID;
  if (static_cast<int64_t>(S) * Hh * D >= (int64_t{1} << 40)) return NABLA_ERR_INVALID;
  if (!(scale >= 0.f) || std::isinf(scale)) return NABLA_ERR_INVALID;
  if (qf == nullptr || kf == nullptr || vf == nullptr || kv_count == nullptr || kv_idx == nullptr || out == nullptr)
    return NABLA_ERR_INVALID;
  if (!aligned16(qf) || !aligned16(kf) || !aligned16(vf) || !aligned16(out) || !aligned16(kv_idx) ||
      !aligned16(kv_count))
    return NABLA_ERR_ALIGN;
  if (lse != nullptr && !aligned16(lse)) return NABLA_ERR_ALIGN;
  if (nsplit < 1 || nsplit > 64 || static_cast<int64_t>(Hh) * nsplit > 65535) return NABLA_ERR_INVALID;
  if (nsplit > 1 && part == nullptr) return NABLA_ERR_INVALID;
  if (nsplit > 1 && !aligned16(part)) return NABLA_ERR_ALIGN;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc != NABLA_OK) return rc;
  if (!di.sm100) return NABLA_ERR_UNSUPPORTED;
  const int Nb = S / 64;
  if (Nb > kMaxListBlocks) return NABLA_ERR_INVALID;
  const float sc = scale > 0.f ? scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));

  // grid_T > 0: q, k, v are in grid order of a grid_T x out_H x out_W grid
  CUtensorMap tq, tk, tv;
  if (grid_T > 0) {
    if (!make_grid_map(&tq, qf, B, grid_T, out_H, out_W, Hh, D) || !make_grid_map(&tk, kf, B, grid_T, out_H, out_W, Hh, D) ||
        !make_grid_map(&tv, vf, B, grid_T, out_H, out_W, Hh, D))
      return NABLA_ERR_CUDA;
  } else if (!make_bshd_map(&tq, qf, B, S, Hh, D, 64) || !make_bshd_map(&tk, kf, B, S, Hh, D, 64) ||
             !make_bshd_map(&tv, vf, B, S, Hh, D, 64)) {
    return NABLA_ERR_CUDA;
  }
  AttnArgs a;
  a.kv_count = kv_count;
  a.kv_idx = kv_idx;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.S = S;
  a.Hh = Hh;
  a.Nb = Nb;
  a.grp_F = grp_F;
  a.grp_nbw = grp_nbw;
  a.out_H = out_H;
  a.out_W = out_W;
  a.in_T = grid_T;
  a.in_nbw = grid_T > 0 ? out_W / 8 : 0;
  a.in_per_t = grid_T > 0 ? (out_H / 8) * (out_W / 8) : 0;
  // exact quotients by multiply-high for block indices and divisors < 2^14
  auto inv = [](int d) -> uint32_t { return d > 1 ? static_cast<uint32_t>((uint64_t{1} << 32) / d + 1) : 0u; };
  a.in_inv_per_t = inv(a.in_per_t);
  a.in_inv_nbw = inv(a.in_nbw);
  a.scale_log2 = static_cast<float>(static_cast<double>(sc) * 1.4426950408889634);
  const AttnSplitLayout sl = attn_split_layout(B, S, Hh, D, nsplit);
  a.nsplit = nsplit;
  a.split_blocks = nsplit > 1 ? ((Nb + nsplit - 1) / nsplit + 31) & ~31 : Nb;
  a.split_out_stride = nsplit > 1 ? sl.o_stride : 0;
  a.split_lse_stride = nsplit > 1 ? sl.lse_stride : 0;
  if (nsplit > 1) {
    a.out = reinterpret_cast<__nv_bfloat16*>(static_cast<unsigned char*>(part) + sl.o_off);
    a.lse = reinterpret_cast<float*>(static_cast<unsigned char*>(part) + sl.lse_off);
  }
  const dim3 grid((Nb + 1) / 2, Hh * nsplit, B);
  auto go = [&](auto kernel, size_t smem) -> int {
    if (smem > static_cast<size_t>(di.max_smem_optin)) return NABLA_ERR_INVALID;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess)
      return NABLA_ERR_CUDA;
    kernel<<<grid, kAttnThreads, smem, stream>>>(tq, tk, tv, a);
    if (nsplit > 1) {
      const int64_t rows = static_cast<int64_t>(B) * S;
      const int64_t threads = rows * Hh * (D / 8);
      const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
      auto combine = nsplit == 2 ? attn_combine_kernel<2> : nsplit == 3 ? attn_combine_kernel<3>
                   : nsplit == 4 ? attn_combine_kernel<4> : attn_combine_kernel<0>;
      combine<<<blocks, 256, 0, stream>>>(a.out, a.lse, nsplit, sl.o_stride, sl.lse_stride,
                                          static_cast<__nv_bfloat16*>(out), lse, rows, S, Hh, D);
    }
    return launch_status();
  };
  return D == 128 ? go(attn_fwd_kernel<128>, AttnSmem<128>::bytes(Nb)) : go(attn_fwd_kernel<64>, AttnSmem<64>::bytes(Nb));
}

// Delta, then the dQ kernel over the row lists and the dK/dV kernel over the
// column lists, each a CTA per pair of blocks.
template <int D>
int launch_bwd_tc(const BwdArgs& ba, const void* qf, const void* kf, const void* vf, const void* out, int B,
                  const DeviceInfo& di, cudaStream_t stream) {
  // four walked stages where the lists leave room, else two
  const size_t optin = static_cast<size_t>(di.max_smem_optin);
  const bool deep = BwdTcSmem<D, 4>::bytes(ba.Nb) <= optin;
  const size_t smem = deep ? BwdTcSmem<D, 4>::bytes(ba.Nb) : BwdTcSmem<D, 2>::bytes(ba.Nb);
  if (smem > optin || ba.Nb > kMaxListBlocks) return NABLA_ERR_INVALID;
  CUtensorMap tq, tk, tv, tdo;
  const bool grid = ba.W > 0;
  const int T = grid ? ba.S / (ba.H * ba.W) : 0;
  if (grid) {
    if (!make_grid_map(&tq, qf, B, T, ba.H, ba.W, ba.Hh, D) || !make_grid_map(&tk, kf, B, T, ba.H, ba.W, ba.Hh, D) ||
        !make_grid_map(&tv, vf, B, T, ba.H, ba.W, ba.Hh, D) ||
        !make_grid_map(&tdo, ba.dout, B, T, ba.H, ba.W, ba.Hh, D))
      return NABLA_ERR_CUDA;
  } else if (!make_bshd_map(&tq, qf, B, ba.S, ba.Hh, D, 64) || !make_bshd_map(&tk, kf, B, ba.S, ba.Hh, D, 64) ||
             !make_bshd_map(&tv, vf, B, ba.S, ba.Hh, D, 64) || !make_bshd_map(&tdo, ba.dout, B, ba.S, ba.Hh, D, 64)) {
    return NABLA_ERR_CUDA;
  }
  BwdTcArgs a;
  a.lse = ba.lse;
  a.delta = ba.delta;
  a.S = ba.S;
  a.Hh = ba.Hh;
  a.Nb = ba.Nb;
  a.grid_H = grid ? ba.H : 0;
  a.grid_W = grid ? ba.W : 0;
  a.in_T = T;
  a.in_nbw = grid ? ba.W / 8 : 0;
  a.in_per_t = grid ? (ba.H / 8) * (ba.W / 8) : 0;
  a.scale = ba.scale;
  a.scale_log2 = ba.scale_log2;
  const int64_t rows = static_cast<int64_t>(B) * ba.S;
  bwd_delta_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(out), ba.dout, const_cast<float*>(ba.delta), rows, ba.S, ba.Hh, D);
  auto* kdq = deep ? bwd_tc_kernel<D, true, 4> : bwd_tc_kernel<D, true, 2>;
  auto* kdkdv = deep ? bwd_tc_kernel<D, false, 4> : bwd_tc_kernel<D, false, 2>;
  if (cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
          cudaSuccess ||
      cudaFuncSetAttribute(kdkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
          cudaSuccess)
    return NABLA_ERR_CUDA;
  const dim3 g((ba.Nb + 1) / 2, ba.Hh, B);
  a.row_count = ba.kv_count;
  a.row_idx = ba.kv_idx;
  a.out0 = ba.dq;
  a.out1 = nullptr;
  kdq<<<g, kBwdTcThreads, smem, stream>>>(tq, tdo, tk, tv, a);
  a.row_count = ba.q_count;
  a.row_idx = ba.q_idx;
  a.out0 = ba.dk;
  a.out1 = ba.dv;
  kdkdv<<<g, kBwdTcThreads, smem, stream>>>(tk, tv, tq, tdo, a);
  return launch_status();
}

int sparse_attn_bwd(const void* qf, const void* kf, const void* vf, const void* out, const void* dout,
                    const float* lse, const int32_t* kv_count, const int32_t* kv_idx, const int32_t* q_count,
                    const int32_t* q_idx, int B, int S, int Hh, int D, float scale, void* dq, void* dk, void* dv,
                    float* delta, int H, int W, cudaStream_t stream) {
  if (B <= 0 || S <= 0 || Hh <= 0 || S % 64 != 0 || (D != 64 && D != 128)) return NABLA_ERR_INVALID;
  if (B > 65535 || Hh > 65535 || static_cast<int64_t>(S) * Hh * D >= (int64_t{1} << 40)) return NABLA_ERR_INVALID;
  if (!(scale >= 0.f) || std::isinf(scale)) return NABLA_ERR_INVALID;
  const void* ptrs[] = {qf, kf, vf, out, dout, lse, kv_count, kv_idx, q_count, q_idx, dq, dk, dv, delta};
  for (const void* p : ptrs)
    if (p == nullptr) return NABLA_ERR_INVALID;
  for (const void* p : ptrs)
    if (!aligned16(p)) return NABLA_ERR_ALIGN;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc != NABLA_OK) return rc;
  if (!di.sm100) return NABLA_ERR_UNSUPPORTED;
  const float sc = scale > 0.f ? scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  BwdArgs a;
  a.q = static_cast<const __nv_bfloat16*>(qf);
  a.k = static_cast<const __nv_bfloat16*>(kf);
  a.v = static_cast<const __nv_bfloat16*>(vf);
  a.dout = static_cast<const __nv_bfloat16*>(dout);
  a.lse = lse;
  a.delta = delta;
  a.kv_count = kv_count;
  a.kv_idx = kv_idx;
  a.q_count = q_count;
  a.q_idx = q_idx;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.S = S;
  a.Hh = Hh;
  a.Nb = S / 64;
  a.scale = sc;
  a.scale_log2 = static_cast<float>(static_cast<double>(sc) * 1.4426950408889634);
  a.H = H;
  a.W = W;
  a.nbw = W / 8;
  a.per_t = (H / 8) * (W / 8);
  if (!di.sm100) return NABLA_ERR_UNSUPPORTED;
  return D == 128 ? launch_bwd_tc<128>(a, qf, kf, vf, out, B, di, stream)
                  : launch_bwd_tc<64>(a, qf, kf, vf, out, B, di, stream);
}

// AB-Attention plan workspace: kbar^T [B*Hh][D][NKB], cent^T [B*Hh][D][R],
// counts [B*Hh][NQB][8], logits [B*Hh][R][NKB] (R = NQB * 8), each region
// 256-byte aligned.
struct ABLayout {
  size_t kbar, cent, counts, logits, total;
};
ABLayout ab_layout(int B, int Hh, int D, int S) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t bh = static_cast<size_t>(B) * Hh, nkb = S / kABKBlock, nqb = S / kABQBlock;
  const size_t R = nqb * kABClusters;
  ABLayout l;
  l.kbar = 0;
  l.cent = up(bh * D * nkb * 4);
  l.counts = l.cent + up(bh * D * R * 4);
  l.logits = l.counts + up(bh * nqb * kABClusters * 4);
  l.total = l.logits + up(bh * R * nkb * 4);
  return l;
}

int ab_check(int B, int S, int Hh, int D) {
  if (B <= 0 || S <= 0 || Hh <= 0 || S % 128 != 0 || (D != 64 && D != 128)) return NABLA_ERR_INVALID;
  if (B > 65535 || Hh > 65535 || static_cast<int64_t>(S) * Hh * D >= (int64_t{1} << 40)) return NABLA_ERR_INVALID;
  // the selection holds one row of block scores in shared memory
  if (ab_select_smem(S / kABKBlock) > 200u * 1024u) return NABLA_ERR_INVALID;
  return NABLA_OK;
}

}  // namespace
}  // namespace nabla

using namespace nabla;

extern "C" {

int nabla_flatten(const void* in, void* out, int B, int T, int H, int W, int P, int row_elems,
                  nabla_stream_t stream) {
  NABLA_NVTX_RANGE();
  return permute<false>(in, out, B, T, H, W, P, row_elems, reinterpret_cast<cudaStream_t>(stream));
}

int nabla_unflatten(const void* in, void* out, int B, int T, int H, int W, int P, int row_elems,
                    nabla_stream_t stream) {
  NABLA_NVTX_RANGE();
  return permute<true>(in, out, B, T, H, W, P, row_elems, reinterpret_cast<cudaStream_t>(stream));
}

size_t nabla_mask_workspace_bytes(int B, int Hh, int D, int T, int H, int W, const nabla_params* params) {
  const int P = params ? params->P : 8;
  if (check_grid(B, T, H, W, P) != NABLA_OK || Hh <= 0 || (D != 64 && D != 128)) return 0;
  const int Nb = static_cast<int>(static_cast<int64_t>(T) * H * W / 64);
  return pooled_bytes(B, Hh, D, Nb) + score_bytes(B, Hh, Nb);
}

int nabla_build_mask(const void* qf, const void* kf, int B, int Hh, int D, int T, int H, int W,
                     const nabla_params* params, int32_t* kv_count, int32_t* kv_idx, void* workspace,
                     nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  MaskPlan mp;
  int rc = mask_plan(B, Hh, D, T, H, W, params, workspace, kv_count, kv_idx, &mp);
  if (rc != NABLA_OK) return rc;
  if (qf == nullptr || kf == nullptr || kv_count == nullptr || kv_idx == nullptr) return NABLA_ERR_INVALID;
  if (!aligned16(qf) || !aligned16(kf) || !aligned16(kv_count) || !aligned16(kv_idx)) return NABLA_ERR_ALIGN;
  if ((rc = device_info(&mp.di)) != NABLA_OK) return rc;
  if ((rc = launch_pool<false>(mp, B, qf, kf, nullptr, nullptr, stream)) != NABLA_OK) return rc;
  return launch_mask_rows(mp, B, stream, true);
}

int nabla_flatten_pool_qk(const void* q, const void* k, void* qf, void* kf, int B, int Hh, int D, int T, int H,
                          int W, const nabla_params* params, void* workspace, nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  MaskPlan mp;
  int rc = mask_plan(B, Hh, D, T, H, W, params, workspace, nullptr, nullptr, &mp);
  if (rc != NABLA_OK) return rc;
  if (q == nullptr || k == nullptr || (qf == nullptr) != (kf == nullptr)) return NABLA_ERR_INVALID;
  if (qf != nullptr && (q == qf || q == kf || k == qf || k == kf || qf == kf)) return NABLA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(qf) || !aligned16(kf)) return NABLA_ERR_ALIGN;
  if ((rc = device_info(&mp.di)) != NABLA_OK) return rc;
  return launch_pool<true>(mp, B, q, k, qf, kf, stream);
}

int nabla_build_mask_grid(const void* q, const void* k, int B, int Hh, int D, int T, int H, int W,
                          const nabla_params* params, int32_t* kv_count, int32_t* kv_idx, void* workspace,
                          nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  MaskPlan mp;
  int rc = mask_plan(B, Hh, D, T, H, W, params, workspace, kv_count, kv_idx, &mp);
  if (rc != NABLA_OK) return rc;
  if (q == nullptr || k == nullptr || kv_count == nullptr || kv_idx == nullptr) return NABLA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(kv_count) || !aligned16(kv_idx)) return NABLA_ERR_ALIGN;
  if ((rc = device_info(&mp.di)) != NABLA_OK) return rc;
  if ((rc = launch_pool<true>(mp, B, q, k, nullptr, nullptr, stream)) != NABLA_OK) return rc;
  return launch_mask_rows(mp, B, stream, true);
}

int nabla_build_mask_pooled(const void* workspace, int B, int Hh, int D, int T, int H, int W,
                            const nabla_params* params, int32_t* kv_count, int32_t* kv_idx, nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  MaskPlan mp;
  int rc = mask_plan(B, Hh, D, T, H, W, params, const_cast<void*>(workspace), kv_count, kv_idx, &mp);
  if (rc != NABLA_OK) return rc;
  if (kv_count == nullptr || kv_idx == nullptr) return NABLA_ERR_INVALID;
  if (!aligned16(kv_count) || !aligned16(kv_idx)) return NABLA_ERR_ALIGN;
  if ((rc = device_info(&mp.di)) != NABLA_OK) return rc;
  return launch_mask_rows(mp, B, stream, true);
}

int nabla_build_mask_sta(int B, int Hh, int T, int H, int W, int P, int sta_t, int sta_h, int sta_w,
                         int32_t* kv_count, int32_t* kv_idx, nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int rc = check_grid(B, T, H, W, P);
  if (rc != NABLA_OK) return rc;
  if (Hh <= 0 || static_cast<int64_t>(B) * Hh > (int64_t{1} << 30)) return NABLA_ERR_INVALID;
  for (const int s : {sta_t, sta_h, sta_w})
    if (s < 1 || s > 65535 || s % 2 == 0) return NABLA_ERR_INVALID;
  if (kv_count == nullptr || kv_idx == nullptr) return NABLA_ERR_INVALID;
  if (!aligned16(kv_count) || !aligned16(kv_idx)) return NABLA_ERR_ALIGN;
  DeviceInfo di;
  if ((rc = device_info(&di)) != NABLA_OK) return rc;
  const int Nb = T * H * W / 64;
  const int copies = B * Hh;
  const dim3 grid((Nb + 7) / 8, copies < 65535 ? copies : 65535);
  sta_lists_kernel<<<grid, 256, 0, stream>>>(kv_count, kv_idx, copies, Nb, H / 8, W / 8, sta_t / 2, sta_h / 2,
                                             sta_w / 2);
  return launch_status();
}

int nabla_build_mask_radial(int B, int Hh, int T, int H, int W, int P, int r0, int32_t* kv_count, int32_t* kv_idx,
                            nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int rc = check_grid(B, T, H, W, P);
  if (rc != NABLA_OK) return rc;
  if (Hh <= 0 || static_cast<int64_t>(B) * Hh > (int64_t{1} << 30)) return NABLA_ERR_INVALID;
  if (r0 < 1 || r0 > 65535) return NABLA_ERR_INVALID;
  if (kv_count == nullptr || kv_idx == nullptr) return NABLA_ERR_INVALID;
  if (!aligned16(kv_count) || !aligned16(kv_idx)) return NABLA_ERR_ALIGN;
  DeviceInfo di;
  if ((rc = device_info(&di)) != NABLA_OK) return rc;
  const int Nb = T * H * W / 64;
  const int copies = B * Hh;
  const dim3 grid((Nb + 7) / 8, copies < 65535 ? copies : 65535);
  radial_lists_kernel<<<grid, 256, 0, stream>>>(kv_count, kv_idx, copies, Nb, H / 8, W / 8, r0);
  return launch_status();
}

int nabla_sparse_attn_fwd(const void* qf, const void* kf, const void* vf, const int32_t* kv_count,
                          const int32_t* kv_idx, int B, int S, int Hh, int D, float scale, void* out, float* lse,
                          nabla_stream_t stream) {
  NABLA_NVTX_RANGE();
  return sparse_attn_launch(qf, kf, vf, kv_count, kv_idx, B, S, Hh, D, scale, out, lse, 0, 0, 0, 0, 0,
                            reinterpret_cast<cudaStream_t>(stream));
}

int nabla_sparse_attn_fwd_grid(const void* q, const void* k, const void* v, const int32_t* kv_count,
                               const int32_t* kv_idx, int B, int Hh, int D, int T, int H, int W, float scale,
                               void* out, float* lse, nabla_stream_t stream) {
  NABLA_NVTX_RANGE();
  if (T <= 0 || H <= 0 || W <= 0 || H % 8 != 0 || W % 8 != 0) return NABLA_ERR_INVALID;
  const int64_t S = static_cast<int64_t>(T) * H * W;
  if (S > (int64_t{1} << 30)) return NABLA_ERR_INVALID;
  const int nbw = W / 8, F = (H / 8) * nbw;
  const bool groups = T % 2 == 0 && nbw % 2 == 0;
  return sparse_attn_launch(q, k, v, kv_count, kv_idx, B, static_cast<int>(S), Hh, D, scale, out, lse,
                            groups ? F : 0, groups ? nbw : 0, T, H, W, reinterpret_cast<cudaStream_t>(stream));
}

size_t nabla_attn_split_workspace_bytes(int B, int Hh, int D, int T, int H, int W, int nsplit) {
  if (B <= 0 || Hh <= 0 || (D != 64 && D != 128) || T <= 0 || H <= 0 || W <= 0 || nsplit < 2 || nsplit > 64)
    return 0;
  return attn_split_layout(B, static_cast<int64_t>(T) * H * W, Hh, D, nsplit).total;
}

int nabla_sparse_attn_fwd_grid_split(const void* q, const void* k, const void* v, const int32_t* kv_count,
                                     const int32_t* kv_idx, int B, int Hh, int D, int T, int H, int W, float scale,
                                     int nsplit, void* workspace, void* out, float* lse, nabla_stream_t stream) {
  NABLA_NVTX_RANGE();
  if (T <= 0 || H <= 0 || W <= 0 || H % 8 != 0 || W % 8 != 0) return NABLA_ERR_INVALID;
  const int64_t S = static_cast<int64_t>(T) * H * W;
  if (S > (int64_t{1} << 30)) return NABLA_ERR_INVALID;
  if (nsplit < 2 || nsplit > 64 || workspace == nullptr) return NABLA_ERR_INVALID;
  const int nbw = W / 8, F = (H / 8) * nbw;
  const bool groups = T % 2 == 0 && nbw % 2 == 0;
  return sparse_attn_launch(q, k, v, kv_count, kv_idx, B, static_cast<int>(S), Hh, D, scale, out, lse,
                            groups ? F : 0, groups ? nbw : 0, T, H, W, reinterpret_cast<cudaStream_t>(stream), nsplit,
                            workspace);
}

int nabla_transpose_lists(const int32_t* kv_count, const int32_t* kv_idx, int B, int Hh, int Nb, int32_t* q_count,
                          int32_t* q_idx, nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B <= 0 || Hh <= 0 || Nb <= 0 || Nb > (1 << 24) || static_cast<int64_t>(B) * Hh > 65535) return NABLA_ERR_INVALID;
  if (kv_count == nullptr || kv_idx == nullptr || q_count == nullptr || q_idx == nullptr) return NABLA_ERR_INVALID;
  if (!aligned16(kv_count) || !aligned16(kv_idx) || !aligned16(q_count) || !aligned16(q_idx)) return NABLA_ERR_ALIGN;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc != NABLA_OK) return rc;
  const size_t smem = static_cast<size_t>(Nb) * 4;
  if (Nb <= kTransposeMaxNb && smem <= static_cast<size_t>(di.max_smem_optin)) {
    if (cudaFuncSetAttribute(transpose_lists_tiled_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return NABLA_ERR_CUDA;
    transpose_lists_tiled_kernel<<<dim3((Nb + 31) / 32, B * Hh), 256, smem, stream>>>(kv_count, kv_idx, q_count,
                                                                                     q_idx, Nb);
  } else {
    transpose_lists_kernel<<<dim3((Nb + 7) / 8, B * Hh), 256, 0, stream>>>(kv_count, kv_idx, q_count, q_idx, Nb);
  }
  return launch_status();
}

int nabla_sparse_attn_bwd(const void* qf, const void* kf, const void* vf, const void* out, const void* dout,
                          const float* lse, const int32_t* kv_count, const int32_t* kv_idx, const int32_t* q_count,
                          const int32_t* q_idx, int B, int S, int Hh, int D, float scale, void* dq, void* dk,
                          void* dv, float* delta, nabla_stream_t stream) {
  NABLA_NVTX_RANGE();
  return sparse_attn_bwd(qf, kf, vf, out, dout, lse, kv_count, kv_idx, q_count, q_idx, B, S, Hh, D, scale, dq, dk,
                         dv, delta, 0, 0, reinterpret_cast<cudaStream_t>(stream));
}

int nabla_sparse_attn_bwd_grid(const void* q, const void* k, const void* v, const void* out, const void* dout,
                               const float* lse, const int32_t* kv_count, const int32_t* kv_idx,
                               const int32_t* q_count, const int32_t* q_idx, int B, int Hh, int D, int T, int H,
                               int W, float scale, void* dq, void* dk, void* dv, float* delta,
                               nabla_stream_t stream) {
  NABLA_NVTX_RANGE();
  if (check_grid(B, T, H, W, 8) != NABLA_OK) return NABLA_ERR_INVALID;
  return sparse_attn_bwd(q, k, v, out, dout, lse, kv_count, kv_idx, q_count, q_idx, B, T * H * W, Hh, D, scale, dq,
                         dk, dv, delta, H, W, reinterpret_cast<cudaStream_t>(stream));
}

int nabla_build_mask_noalloc(const void* qf, const void* kf, int B, int Hh, int D, int T, int H, int W,
                             const nabla_params* params, int32_t* kv_count, int32_t* kv_idx,
                             nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (params == nullptr || nabla_mask_workspace_bytes(B, Hh, D, T, H, W, params) == 0) return NABLA_ERR_INVALID;
  const int Nb = static_cast<int>(static_cast<int64_t>(T) * H * W / 64);
  if (pooled_bytes(B, Hh, D, Nb) > NABLA_NOALLOC_SCRATCH_BYTES) return NABLA_ERR_TOO_LARGE;
  // The buffer's device address, looked up on every call with the caller's
  // device current (cheap, host-only): nothing is cached, so a context torn
  // down and recreated in between cannot leave a stale address behind.
  void* scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || scratch == nullptr) return NABLA_ERR_CUDA;
  MaskPlan mp;
  int rc = mask_plan(B, Hh, D, T, H, W, params, scratch, kv_count, kv_idx, &mp);
  if (rc != NABLA_OK) return rc;
  if (qf == nullptr || kf == nullptr || kv_count == nullptr || kv_idx == nullptr) return NABLA_ERR_INVALID;
  if (!aligned16(qf) || !aligned16(kf) || !aligned16(kv_count) || !aligned16(kv_idx)) return NABLA_ERR_ALIGN;
  if ((rc = device_info(&mp.di)) != NABLA_OK) return rc;
  if ((rc = launch_pool<false>(mp, B, qf, kf, nullptr, nullptr, stream)) != NABLA_OK) return rc;
  return launch_mask_rows(mp, B, stream, false);
}

size_t nabla_ab_workspace_bytes(int B, int S, int Hh, int D) {
  if (ab_check(B, S, Hh, D) != NABLA_OK) return 0;
  return ab_layout(B, Hh, D, S).total;
}

int nabla_ab_plan(const void* q, const void* k, const float* u, int B, int S, int Hh, int D, int kmeans_iters,
                  double budget, float scale, int32_t* kcount, int32_t* kidx, float* kshift, void* workspace,
                  nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int rc = ab_check(B, S, Hh, D);
  if (rc != NABLA_OK) return rc;
  if (kmeans_iters < 0 || kmeans_iters > 64 || !(budget >= 0.0) || std::isinf(budget)) return NABLA_ERR_INVALID;
  if (!(scale >= 0.f) || std::isinf(scale)) return NABLA_ERR_INVALID;
  const void* ptrs[] = {q, k, u, kcount, kidx, kshift, workspace};
  for (const void* p : ptrs)
    if (p == nullptr) return NABLA_ERR_INVALID;
  for (const void* p : ptrs)
    if (!aligned16(p)) return NABLA_ERR_ALIGN;
  DeviceInfo di;
  if ((rc = device_info(&di)) != NABLA_OK) return rc;
  const float sc = scale > 0.f ? scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  const ABLayout lay = ab_layout(B, Hh, D, S);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  float* kbarT = reinterpret_cast<float*>(ws + lay.kbar);
  float* centT = reinterpret_cast<float*>(ws + lay.cent);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + lay.counts);
  float* logits = reinterpret_cast<float*>(ws + lay.logits);
  const int nkb = S / kABKBlock, nqb = S / kABQBlock, R = nqb * kABClusters;
  ab_key_means_kernel<<<dim3(nkb / 8, B), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(k), kbarT, S, Hh, D);
  if ((rc = launch_status()) != NABLA_OK) return rc;
  const size_t ksm = ab_kmeans_smem(D);
  if (cudaFuncSetAttribute(ab_kmeans_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(ksm)) !=
      cudaSuccess)
    return NABLA_ERR_CUDA;
  ab_kmeans_kernel<<<dim3(nqb, Hh, B), 256, ksm, stream>>>(static_cast<const __nv_bfloat16*>(q), centT, counts, S, Hh,
                                                           D, kmeans_iters);
  if ((rc = launch_status()) != NABLA_OK) return rc;
  ScoreShape sh;
  sh.nrows = R;
  sh.ncols = nkb;
  sh.D = D;
  sh.q_ld = R;
  sh.k_ld = sh.out_ld = nkb;
  sh.q_bh = static_cast<int64_t>(D) * R;
  sh.k_bh = static_cast<int64_t>(D) * nkb;
  sh.out_bh = static_cast<int64_t>(R) * nkb;
  if (launch_score_tiles(centT, kbarT, logits, sh, B * Hh, sc, stream) != cudaSuccess) return NABLA_ERR_CUDA;
  ABSelectArgs sa;
  sa.logits = logits;
  sa.counts = counts;
  sa.u = u;
  sa.kcount = kcount;
  sa.kidx = kidx;
  sa.kshift = kshift;
  sa.nqb = nqb;
  sa.nkb = nkb;
  sa.budget = budget;
  const size_t ssm = ab_select_smem(nkb);
  if (cudaFuncSetAttribute(ab_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(ssm)) !=
      cudaSuccess)
    return NABLA_ERR_CUDA;
  ab_select_kernel<<<dim3(nqb, B * Hh), kABSelectWarps * 32, ssm, stream>>>(sa);
  return launch_status();
}

int nabla_ab_attn_fwd(const void* q, const void* k, const void* v, const int32_t* kcount, const int32_t* kidx,
                      const float* kshift, int B, int S, int Hh, int D, float scale, void* out, float* lse,
                      nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int rc = ab_check(B, S, Hh, D);
  if (rc != NABLA_OK) return rc;
  if (!(scale >= 0.f) || std::isinf(scale)) return NABLA_ERR_INVALID;
  const void* ptrs[] = {q, k, v, kcount, kidx, kshift, out};
  for (const void* p : ptrs)
    if (p == nullptr) return NABLA_ERR_INVALID;
  for (const void* p : ptrs)
    if (!aligned16(p)) return NABLA_ERR_ALIGN;
  if (lse != nullptr && !aligned16(lse)) return NABLA_ERR_ALIGN;
  DeviceInfo di;
  if ((rc = device_info(&di)) != NABLA_OK) return rc;
  if (!di.sm100) return NABLA_ERR_UNSUPPORTED;
  const float sc = scale > 0.f ? scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  CUtensorMap tq;
  if (!make_bshd_map(&tq, q, B, S, Hh, D, 128)) return NABLA_ERR_CUDA;
  ABAttnArgs a;
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.kcount = kcount;
  a.kidx = kidx;
  a.kshift = kshift;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.S = S;
  a.Hh = Hh;
  a.nkb = S / kABKBlock;
  a.scale_log2 = static_cast<float>(static_cast<double>(sc) * 1.4426950408889634);
  const dim3 grid(S / 128, Hh, B);
  if (D == 128) {
    const size_t smem = ABAttnSmem<128>::kBytes;
    if (cudaFuncSetAttribute(ab_attn_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return NABLA_ERR_CUDA;
    ab_attn_fwd_kernel<128><<<grid, kABAttnThreads, smem, stream>>>(tq, a);
  } else {
    const size_t smem = ABAttnSmem<64>::kBytes;
    if (cudaFuncSetAttribute(ab_attn_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return NABLA_ERR_CUDA;
    ab_attn_fwd_kernel<64><<<grid, kABAttnThreads, smem, stream>>>(tq, a);
  }
  return launch_status();
}

int nabla_selftest_wait_timeout(long long limit_cycles, nabla_stream_t stream_) {
  if (limit_cycles < 1000 || limit_cycles > kWaitLimitCycles) return NABLA_ERR_INVALID;
  wait_timeout_selftest_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream_)>>>(limit_cycles);
  return launch_status();
}

int nabla_get_status(nabla_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return NABLA_ERR_CUDA;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return NABLA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return NABLA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return NABLA_ERR_CUDA;
  return v;
}

int nabla_validate_mask(const int32_t* kv_count, const int32_t* kv_idx, int B, int Hh, int Nb, int32_t* bad_rows,
                        nabla_stream_t stream_) {
  NABLA_NVTX_RANGE();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B <= 0 || Hh <= 0 || Nb <= 0 || kv_count == nullptr || kv_idx == nullptr || bad_rows == nullptr)
    return NABLA_ERR_INVALID;
  if (cudaMemsetAsync(bad_rows, 0, sizeof(int32_t), stream) != cudaSuccess) return NABLA_ERR_CUDA;
  const int64_t rows = static_cast<int64_t>(B) * Hh * Nb;
  validate_mask_kernel<<<static_cast<unsigned>((rows + 255) / 256), 256, 0, stream>>>(kv_count, kv_idx, rows, Nb,
                                                                                       bad_rows);
  return launch_status();
}

const char* nabla_strerror(int code) {
  switch (code) {
    case NABLA_OK: return "ok";
    case NABLA_ERR_INVALID: return "invalid argument (shape or parameter)";
    case NABLA_ERR_ALIGN: return "pointer or row stride not 16-byte aligned";
    case NABLA_ERR_CUDA: return "CUDA runtime error or kernel launch failure";
    case NABLA_ERR_DEVICE_TIMEOUT: return "device wait exceeded its time limit";
    case NABLA_ERR_DEVICE_BOUNDS: return "block index or count out of range";
    case NABLA_ERR_UNSUPPORTED: return "device is not an sm_100 GPU";
    case NABLA_ERR_TOO_LARGE: return "mask workspace exceeds the static scratch of nabla_build_mask_noalloc (16 MiB)";
    default: return "unknown error";
  }
}

}  // extern "C"
