// Block-sparse flash-attention forward on the kept 64 x 64 tiles (NABLA
// technical summary, "Metodologia: NABLA", item 2 "Expansao": only the
// listed N x N blocks are computed; a dropped block is in neither the
// numerator nor the softmax normaliser).
//
// One CTA owns a query tile of 128 rows = two 64-token query blocks of one
// (batch, head), so every tcgen05.mma runs at the full M = 128.  It walks the
// ascending union of the two blocks' key-block lists; a key block listed by
// only one of them is masked for the other half's rows (their probabilities
// are set to zero and their running max and sum are left alone).  Which two
// blocks share a CTA decides how many masked half-tiles it runs:
//   - without the token grid, blocks 2p and 2p+1 of the flattened order
//     (horizontally adjacent patches of one frame);
//   - with the grid, each 2 x 2 group {(t, w), (t, w+1), (t+1, w), (t+1, w+1)}
//     of patch positions (same patch row, two frames) is split into two CTAs
//     either along w or along t, whichever pairing has the smaller total
//     union of lists.  Both CTAs of a group take the same decision from the
//     same four lists; one block of each CTA is the same under both pairings,
//     so its half of Q is loaded before the lists are read.
//
// Warp roles (224 threads, two CTAs per SM):
//   warps 0-3  softmax: thread t owns query row t = TMEM lane t.  Reads the
//              64 scores of its row from TMEM, keeps an online max/sum,
//              rescales its O row in TMEM when the max grew by more than
//              2^8, writes the bf16 probabilities back into the first 32
//              columns of the same TMEM score buffer, and finally normalises
//              O and stores it with the LSE.
//   warp 4     TMA producer: Q once, then K_j and V_j of each listed block j
//              (contiguous 64-token boxes of the flattened layout) into a
//              ring of kStages stages.
//   warp 5     QK^T issuer (one thread): S = Q K_j^T into one of two TMEM
//              score buffers (M=128, N=64, K=D).
//   warp 6     PV issuer (one thread): O += P V_j with P read from tensor
//              memory and V MN-major straight from its TMA tile (M=128, N=D,
//              K=64).
// Tensor memory per CTA: S0 | S1 (64 columns each, P aliases their first 32)
// | O (D columns) = 256 columns, so two CTAs share an SM's 512 columns.
// Every wait is bounded (see mbar_wait); a timeout raises the CTA's abort
// flag, records NABLA_ERR_DEVICE_TIMEOUT and all roles drain and exit, with
// the tensor memory freed.
#pragma once

#include "common.cuh"

namespace nabla {

constexpr int kAttnThreads = 224;
constexpr int kMaxListBlocks = 16383;  // list entries hold a 14-bit block index

template <int D>
struct AttnSmem {
  static constexpr int kChunks = D / 64;          // 64-element (128-byte) column chunks
  static constexpr int kStages = D == 128 ? 2 : 4;
  static constexpr int kQBytes = 128 * 128 * kChunks;
  static constexpr int kKVBytes = 64 * 128 * kChunks;
  // offsets from a 1024-byte-aligned base
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + kStages * kKVBytes;
  static constexpr int kBars = kV + kStages * kKVBytes;
  // q, k full + empty, v full + empty, s full, p full, pv done, mma drain
  static constexpr int kNumBars = 1 + 4 * kStages + 2 * 3 + 1;
  // tmem base, abort flag, list length, the two query blocks
  static constexpr int kMisc = kBars + 8 * kNumBars;
  static constexpr int kList = kMisc + 32;
  __host__ __device__ static size_t list_bytes(int Nb) { return (static_cast<size_t>(Nb) * 2 + 15) & ~size_t(15); }
  // followed by four key-block bitmaps of (Nb + 31) / 32 words
  static size_t bytes(int Nb) {
    const int words = (Nb + 31) / 32;
    return 1024 + kList + list_bytes(Nb) + 4 * static_cast<size_t>(words) * 4;
  }
};

struct AttnArgs {
  const int32_t* kv_count;  // [B][Hh][Nb]
  const int32_t* kv_idx;    // [B][Hh][Nb][Nb]
  __nv_bfloat16* out;       // [B][S][Hh][D]
  float* lse;               // [B][Hh][S] or null
  int S, Hh, Nb;
  int grp_F;                // query blocks per frame for 2 x 2 (w, t) grouping, 0 = pairs 2p, 2p+1
  int grp_nbw;              // blocks per patch row (W / 8) when grp_F > 0
  int out_H, out_W;         // > 0: O and LSE rows are stored in grid order of a T x H x W grid
  int in_T, in_nbw, in_per_t;  // in_nbw > 0: Q, K, V are in grid order, read through 5-D maps
  uint32_t in_inv_per_t, in_inv_nbw;  // floor(2^32 / d) + 1 (0 for d = 1): j / d = umulhi(j, inv) for j, d < 2^14
  float scale_log2;         // scale * log2(e)
  // Key-range split: blockIdx.y = head * nsplit + split; the CTA walks only
  // the listed key blocks in [split * split_blocks, (split + 1) *
  // split_blocks) and stores its O (normalised over that range) and LSE at
  // out + split * split_out_stride, lse + split * split_lse_stride, for a
  // merge by attn_combine_kernel.  nsplit = 1: the whole list, one output.
  int nsplit, split_blocks;
  int64_t split_out_stride, split_lse_stride;
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using L = AttnSmem<D>;
  constexpr int kStages = L::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kStages;
  uint64_t* k_empty = v_full + kStages;
  uint64_t* v_empty = k_empty + kStages;
  uint64_t* s_full = v_empty + kStages;   // [2]
  uint64_t* p_full = s_full + 2;          // [2]
  uint64_t* pv_done = p_full + 2;         // [2]
  uint64_t* mma_drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kMisc + 4);
  int* list_len = reinterpret_cast<int*>(sm + L::kMisc + 8);
  int* half_blk = reinterpret_cast<int*>(sm + L::kMisc + 12);  // [2]; -1 = no block
  uint16_t* list = reinterpret_cast<uint16_t*>(sm + L::kList);
  const int Nb = a.Nb;
  const int words = (Nb + 31) >> 5;
  uint32_t* bm = reinterpret_cast<uint32_t*>(sm + L::kList + L::list_bytes(Nb));  // [4][words]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p = blockIdx.x, hd = blockIdx.y / a.nsplit, split = blockIdx.y - hd * a.nsplit, b = blockIdx.z;
  const int64_t bh = static_cast<int64_t>(b) * a.Hh + hd;
  const int k0 = split * a.split_blocks, k1 = k0 + a.split_blocks;  // key blocks this CTA walks
  // One 64-token block j of Q, K or V, 64 columns (chunk c) of one head, as
  // 64 rows of 128 bytes.  Flattened input: rows 64j..64j+63 (4-D map).
  // Grid-order input: block j is the 8 x 8 patch (bh, bw) of frame t, read
  // through a 5-D map (d, head, w, h, frame) whose box lists its pixels row
  // by row, i.e. in the flattened order inside the block: the fractal
  // flattening happens in the copy.
  // All kChunks column chunks of block j; the block's patch coordinates are
  // derived once, with multiply-high reciprocals (the producer is a single
  // thread on the critical path, where integer divisions would cost).
  auto load_block = [&](unsigned char* dst, const CUtensorMap* map, uint64_t* bar, int j, int chunk_stride) {
    if (a.in_nbw > 0) {
      // (an inverse of 0 stands for the divisor 1, whose reciprocal 2^32 does not fit)
      const int t = a.in_inv_per_t ? static_cast<int>(__umulhi(static_cast<uint32_t>(j), a.in_inv_per_t)) : j;
      const int rem = j - t * a.in_per_t;
      const int bhh = a.in_inv_nbw ? static_cast<int>(__umulhi(static_cast<uint32_t>(rem), a.in_inv_nbw)) : rem;
      const int bww = rem - bhh * a.in_nbw;
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_5d(dst + c * chunk_stride, map, bar, c * 64, hd, bww * 8, bhh * 8, b * a.in_T + t);
    } else {
      for (int c = 0; c < L::kChunks; ++c) tma_load_4d(dst + c * chunk_stride, map, bar, c * 64, hd, j * 64, b);
    }
  };

  // Candidate query blocks.  Group mode: cand = {(t,w), (t,w+1), (t+1,w),
  // (t+1,w+1)}; CTA slot 0 owns cand[0] in half 0 and slot 1 owns cand[3] in
  // half 1; the other half is cand[1] or cand[2] (see the decision below).
  // Pair mode: cand = {2p, 2p+1} in halves 0 and 1.
  const bool grouped = a.grp_F > 0;
  const int slot = p & 1;
  int cand[4];
  if (grouped) {
    const int g = p >> 1, ngw = a.grp_nbw >> 1, nbh = a.grp_F / a.grp_nbw;
    const int bw2 = g % ngw, rest = g / ngw;
    const int a0 = 2 * (rest / nbh) * a.grp_F + (rest % nbh) * a.grp_nbw + 2 * bw2;
    cand[0] = a0;
    cand[1] = a0 + 1;
    cand[2] = a0 + a.grp_F;
    cand[3] = a0 + a.grp_F + 1;
  } else {
    cand[0] = 2 * p;
    cand[1] = 2 * p + 1 < Nb ? 2 * p + 1 : -1;
    cand[2] = cand[3] = -1;
  }
  const int nlists = grouped ? 4 : 2;

  // ---- set-up: barriers, tensor memory, merged block list
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 4);  // one arrival per softmax warp
      mbar_init(pv_done + s, 1);
    }
    mbar_init(mma_drain, 2);  // one commit from each MMA-issuing thread
    *abort_flag = 0;
    fence_mbar_init();
    // The half of Q whose block is already known loads right away; in pair
    // mode both halves do (a missing second block loads the first one again:
    // its rows are never listed and never stored).
    tma_prefetch_desc(&tmQ);
    mbar_arrive_expect_tx(q_full, L::kQBytes);
    if (grouped) {
      load_block(sm + L::kQ + slot * 64 * 128, &tmQ, q_full, cand[slot ? 3 : 0], 128 * 128);
    } else {
      const int q1 = cand[1] >= 0 ? cand[1] : cand[0];
      load_block(sm + L::kQ, &tmQ, q_full, cand[0], 128 * 128);
      load_block(sm + L::kQ + 64 * 128, &tmQ, q_full, q1, 128 * 128);
    }
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
  }
  // The counts of the lists and their first 32 entries (warp h reads list
  // h, one cache line) are loaded together, so the common case of lists of
  // at most 32 blocks waits for one memory latency.  Entries past a row's
  // count are read and ignored (a row has Nb entries); reading further ahead
  // would touch lines the mask never wrote, which come from DRAM.
  int cnt[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const bool have = h < nlists && cand[h] >= 0;
    cnt[h] = have ? __ldg(a.kv_count + bh * Nb + (have ? cand[h] : 0)) : 0;
  }
  int first = 0;
  const int my_cand = warp == 0 ? cand[0] : warp == 1 ? cand[1] : warp == 2 ? cand[2] : warp == 3 ? cand[3] : -1;
  const bool first_list = warp < nlists && my_cand >= 0 && lane < Nb;
  if (first_list) first = __ldg(a.kv_idx + (bh * Nb + my_cand) * static_cast<int64_t>(Nb) + lane);
  for (int w = tid; w < 4 * words; w += kAttnThreads) bm[w] = 0u;
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    int c = cnt[h];
    if (c < 0 || c > Nb) {
      if (tid == 0) report(NABLA_ERR_DEVICE_BOUNDS);
      c = c < 0 ? 0 : Nb;
    }
    uint32_t* bmh = bm + h * words;
    const int32_t* src = a.kv_idx + (bh * Nb + (cand[h] >= 0 ? cand[h] : 0)) * static_cast<int64_t>(Nb);
    if (warp == h && lane < c && first_list) {
      if (first < 0 || first >= Nb) report(NABLA_ERR_DEVICE_BOUNDS);
      else if (first >= k0 && first < k1) atomicOr(bmh + (first >> 5), 1u << (first & 31));
    }
    for (int e = 32 + tid; e < c; e += kAttnThreads) {
      const int j = src[e];
      if (j < 0 || j >= Nb) {
        report(NABLA_ERR_DEVICE_BOUNDS);
        continue;
      }
      if (j >= k0 && j < k1) atomicOr(bmh + (j >> 5), 1u << (j & 31));
    }
  }
  __syncthreads();
  // Which candidate list each half of the tile holds.  Group mode: split
  // along t when the two unions along t hold fewer blocks in total than the
  // two along w.  Evaluated by a whole warp; every warp that calls it gets
  // the same answer.
  auto halves = [&](int& x_half0, int& x_half1, bool& along_t) {
    x_half0 = 0;
    x_half1 = 1;
    along_t = false;
    if (!grouped) return;
    int cw = 0, ct = 0;
    for (int w = lane; w < words; w += 32) {
      const uint32_t b0 = bm[w], b1 = bm[words + w], b2 = bm[2 * words + w], b3 = bm[3 * words + w];
      cw += __popc(b0 | b1) + __popc(b2 | b3);
      ct += __popc(b0 | b2) + __popc(b1 | b3);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      cw += __shfl_xor_sync(0xffffffffu, cw, o);
      ct += __shfl_xor_sync(0xffffffffu, ct, o);
    }
    along_t = ct < cw;
    x_half0 = slot == 0 ? 0 : (along_t ? 1 : 2);
    x_half1 = slot == 0 ? (along_t ? 2 : 1) : 3;
  };
  bool k0_early = false;  // producer: K of the first listed block already requested
  if (warp == 4) {
    // The producer finds the first block of the merged list from the
    // bitmaps and requests its K now, while warp 0 builds the list.
    int x0, x1;
    bool along_t;
    halves(x0, x1, along_t);
    int j0 = -1;
    for (int w0 = 0; w0 < words && j0 < 0; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t u = w < words ? (bm[x0 * words + w] | bm[x1 * words + w]) : 0u;
      const unsigned bal = __ballot_sync(0xffffffffu, u != 0u);
      if (bal != 0u) {
        const int src_lane = __ffs(bal) - 1;
        const uint32_t uw = __shfl_sync(0xffffffffu, u, src_lane);
        j0 = (w0 + src_lane) * 32 + __ffs(uw) - 1;
      }
    }
    if (j0 >= 0) {
      k0_early = true;
      if (lane == 0) {
        mbar_arrive_expect_tx(k_full, L::kKVBytes);
        load_block(sm + L::kK, &tmK, k_full, j0, 64 * 128);
      }
    }
  }
  if (warp == 0) {
    int x_half0, x_half1;
    bool along_t;
    halves(x_half0, x_half1, along_t);
    if (grouped && lane == 0) {
      // the other half of Q; q_full already expects its bytes
      const int other = slot ? x_half0 : x_half1;
      load_block(sm + L::kQ + (slot ? 0 : 64 * 128), &tmQ, q_full, cand[other], 128 * 128);
    }
    if (lane == 0) {
      half_blk[0] = cand[x_half0];
      half_blk[1] = cand[x_half1];
    }
    const uint32_t* bm0 = bm + x_half0 * words;
    const uint32_t* bm1 = bm + x_half1 * words;
    int base = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t x0 = w < words ? bm0[w] : 0u, x1 = w < words ? bm1[w] : 0u;
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
  const uint32_t tS0 = tmem, tS1 = tmem + 64, tO = tmem + 128;

  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
  const uint32_t sQ = smem_u32(sm + L::kQ), sK = smem_u32(sm + L::kK), sV = smem_u32(sm + L::kV);

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // One thread streams K and V through two rings.  A K stage frees as soon
    // as its QK^T MMA is done, a V stage after its PV MMA; the MMA order is
    // QK(n), PV(n-1), so K runs one block ahead of V: step n loads K(n) (its
    // stage freed by QK(n-2)) and then V(n-1) (freed by PV(n-3)).  Blocking
    // waits of a second producer lane in this warp would stall this one.
    if (lane == 0 && L_n > 0) {
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int n = 0; ok && n <= L_n; ++n) {
        if (n < L_n && !(n == 0 && k0_early)) {
          const int s = n % kStages;
          if (n >= kStages && !mbar_wait(k_empty + s, ((n / kStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int j = static_cast<int>(list[n] & 0x3FFFu);
          mbar_arrive_expect_tx(k_full + s, L::kKVBytes);
          load_block(sm + L::kK + s * L::kKVBytes, &tmK, k_full + s, j, 64 * 128);
        }
        if (n < L_n) k_issued = n + 1;
        if (n >= 1) {
          const int m = n - 1, s = m % kStages;
          if (m >= kStages && !mbar_wait(v_empty + s, ((m / kStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int j = static_cast<int>(list[m] & 0x3FFFu);
          mbar_arrive_expect_tx(v_full + s, L::kKVBytes);
          load_block(sm + L::kV + s * L::kKVBytes, &tmV, v_full + s, j, 64 * 128);
          v_issued = m + 1;
        }
      }
      // Drain: wait for the last issued loads of every stage so no copy is in
      // flight when the CTA exits, also on the abort path (time-bounded).
      for (int n = (k_issued > kStages ? k_issued - kStages : 0); n < k_issued; ++n)
        mbar_wait_drain(k_full + n % kStages, (n / kStages) & 1);
      for (int n = (v_issued > kStages ? v_issued - kStages : 0); n < v_issued; ++n)
        mbar_wait_drain(v_full + n % kStages, (n / kStages) & 1);
    }
    if (lane == 0) mbar_wait_drain(q_full, 0);
  } else if (warp == 5) {
    // ---------------------------------------------------------- QK^T issue
    if (lane == 0 && L_n > 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag);
      tc_fence_after();
      for (int n = 0; ok && n < L_n; ++n) {
        const int s = n % kStages;
        if (!mbar_wait(k_full + s, (n / kStages) & 1, abort_flag)) { ok = false; break; }
        // S buffer (n & 1) still holds P(n-2) until PV(n-2) has read it.
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
      // Every MMA this thread issued must finish before the tensor memory is
      // freed, also on the abort path (time-bounded).
      umma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------- PV issue
    // A thread of its own, so a PV is issued as soon as its P is written
    // instead of queueing behind the issue of the next QK^T.
    if (lane == 0 && L_n > 0) {
      bool ok = true;
      for (int m = 0; ok && m < L_n; ++m) {
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
    const int r = tid;  // query row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t flag = 0x4000u << (r >> 6);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int n = 0; n < L_n; ++n) {
      if (!__all_sync(0xffffffffu, mbar_wait(s_full + (n & 1), (n >> 1) & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[4][16];
      const uint32_t tS = ((n & 1) ? tS1 : tS0) + lane_off;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16(tS + c * 16, sv[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence16(sv[c]);

      const bool inc = (static_cast<uint32_t>(list[n]) & flag) != 0u;
      float factor = 1.f;
      bool need = false;
      if (inc) {
        float mc[4];  // four independent max chains, three inputs per step
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          mc[c] = fmaxf(__uint_as_float(sv[c][0]), __uint_as_float(sv[c][15]));
#pragma unroll
          for (int e = 1; e < 15; e += 2) mc[c] = fmax3(mc[c], __uint_as_float(sv[c][e]), __uint_as_float(sv[c][e + 1]));
        }
        float mx = fmax3(fmaxf(mc[0], mc[1]), mc[2], mc[3]);
        mx *= a.scale_log2;
        if (mx > m_run + 8.f) {  // also true while m_run is -inf
          factor = ex2_approx(m_run - mx);  // 0 when m_run = -inf
          need = (n > 0) && (l_run > 0.f);  // an all-zero O row needs no rescale
          m_run = mx;
        }
      }
      // pairs of columns: x = s * scale_log2 - m in one two-lane FMA, two
      // exponentials, two-lane sums (four independent accumulators)
      unsigned long long rs2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[2][16];
      const unsigned long long sc2 = f2_pack(a.scale_log2, a.scale_log2), nm2 = f2_pack(-m_run, -m_run);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float p0 = 0.f, p1 = 0.f;
          if (inc) {
            const unsigned long long x2 = f2_fma((static_cast<unsigned long long>(sv[c][e + 1]) << 32) | sv[c][e], sc2, nm2);
            p0 = ex2_approx(f2_lo(x2));
            p1 = ex2_approx(f2_hi(x2));
          }
          rs2[c] = f2_add(rs2[c], f2_pack(p0, p1));
          const int k = c * 8 + e / 2;
          pk[k >> 4][k & 15] = pack_bf16x2(p0, p1);
        }
        // the first 32 keys' P go to tensor memory while the last 32 are
        // computed (S is already in registers)
        if (c == 1) tmem_st16(((n & 1) ? tS1 : tS0) + lane_off, pk[0]);
      }
      const unsigned long long r01 = f2_add(rs2[0], rs2[1]), r23 = f2_add(rs2[2], rs2[3]);
      const unsigned long long rall = f2_add(r01, r23);
      l_run = l_run * factor + (f2_lo(rall) + f2_hi(rall));

      __syncwarp();
      if (__any_sync(0xffffffffu, need)) {
        // O must not be rescaled while PV(n-1) still accumulates into it.
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
      // P(n): bf16 pairs into the first 32 columns of the score buffer (the
      // first half was stored above).
      tmem_st16(tS + 16, pk[1]);
      tmem_st_wait();
      tc_fence_before();
      // one arrival per warp, after every lane's stores have completed: 128
      // arrivals on one mbarrier serialised in shared memory on the softmax's
      // critical path
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + (n & 1));
    }

    // ---------------------------------------------------------------- epilogue
    const int qblk = half_blk[r >> 6];
    const bool row_valid = qblk >= 0;
    int64_t row_g = static_cast<int64_t>(row_valid ? qblk : 0) * 64 + (r & 63);
    if (a.out_W > 0) {
      // store in grid order (the inverse fractal flattening, fused): row r of
      // block qblk is pixel (r / 8, r % 8) of the block's 8 x 8 patch
      const int nbw = a.out_W >> 3, per_t = (a.out_H >> 3) * nbw;
      const int blk = row_valid ? qblk : 0;
      const int t = blk / per_t, rem = blk - t * per_t, bhh = rem / nbw, bww = rem - bhh * nbw;
      row_g = (static_cast<int64_t>(t) * a.out_H + bhh * 8 + ((r & 63) >> 3)) * a.out_W + bww * 8 + (r & 7);
    }
    if (ok && L_n > 0) ok = __all_sync(0xffffffffu, mbar_wait(pv_done + ((L_n - 1) & 1), ((L_n - 1) >> 1) & 1, abort_flag));
    tc_fence_after();
    __syncwarp();
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    __nv_bfloat16* orow =
        a.out + split * a.split_out_stride + ((static_cast<int64_t>(b) * a.S + row_g) * a.Hh + hd) * D;
#pragma unroll 1
    for (int c0 = 0; c0 < D / 16; c0 += 4) {
      uint32_t ob[4][16];
      if (ok && L_n > 0) {
#pragma unroll
        for (int u = 0; u < 4; ++u) tmem_ld16(tO + lane_off + (c0 + u) * 16, ob[u]);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 4; ++u) reg_fence16(ob[u]);
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int e = 0; e < 16; ++e) ob[u][e] = 0u;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
      const int c = c0 + u;
      const uint32_t (&ov)[16] = ob[u];
      uint4 w0, w1;
      w0.x = pack_bf16x2(__uint_as_float(ov[0]) * inv_l, __uint_as_float(ov[1]) * inv_l);
      w0.y = pack_bf16x2(__uint_as_float(ov[2]) * inv_l, __uint_as_float(ov[3]) * inv_l);
      w0.z = pack_bf16x2(__uint_as_float(ov[4]) * inv_l, __uint_as_float(ov[5]) * inv_l);
      w0.w = pack_bf16x2(__uint_as_float(ov[6]) * inv_l, __uint_as_float(ov[7]) * inv_l);
      w1.x = pack_bf16x2(__uint_as_float(ov[8]) * inv_l, __uint_as_float(ov[9]) * inv_l);
      w1.y = pack_bf16x2(__uint_as_float(ov[10]) * inv_l, __uint_as_float(ov[11]) * inv_l);
      w1.z = pack_bf16x2(__uint_as_float(ov[12]) * inv_l, __uint_as_float(ov[13]) * inv_l);
      w1.w = pack_bf16x2(__uint_as_float(ov[14]) * inv_l, __uint_as_float(ov[15]) * inv_l);
      if (row_valid) {
        reinterpret_cast<uint4*>(orow + c * 16)[0] = w0;
        reinterpret_cast<uint4*>(orow + c * 16)[1] = w1;
      }
      }
    }
    if (row_valid && a.lse != nullptr)
      a.lse[split * a.split_lse_stride + bh * a.S + row_g] =
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

// Merge of the key-range split: per (token row, head), O = sum over the
// splits of exp(lse_s - L) O_s and LSE L = log sum exp(lse_s), where O_s is
// the split's output normalised over its own key range (a split with no
// kept block there has lse_s = -inf and weight 0).  Thread t handles 8
// consecutive elements of a row's head (D / 8 threads per row and head).
// NS > 0: exactly NS splits, every load issued before the first use (one
// memory latency per thread); NS = 0: any nsplit, split by split.
template <int NS>
__global__ void __launch_bounds__(256) attn_combine_kernel(const __nv_bfloat16* __restrict__ part_o,
                                                           const float* __restrict__ part_lse, int nsplit,
                                                           int64_t o_stride, int64_t lse_stride,
                                                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                                                           int64_t rows, int S, int Hh, int D) {
  const int per = D / 8;
  const int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / per;
  const int part = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) - item * per);
  if (item >= rows * Hh) return;
  const int64_t row = item / Hh;  // b * S + s
  const int hd = static_cast<int>(item - row * Hh);
  const int64_t b = row / S, sidx = row - b * S;
  const int64_t li = (b * Hh + hd) * S + sidx;
  const int64_t oi = item * D + part * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float m = -INFINITY, wsum = 0.f;
  auto accumulate = [&](float w, const uint4& v) {
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
      acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
    }
  };
  if constexpr (NS > 0) {
    float l[NS];
    uint4 v[NS];
#pragma unroll
    for (int t = 0; t < NS; ++t) {
      l[t] = __ldg(part_lse + t * lse_stride + li);
      v[t] = __ldg(reinterpret_cast<const uint4*>(part_o + t * o_stride + oi));
    }
#pragma unroll
    for (int t = 0; t < NS; ++t) m = fmaxf(m, l[t]);
    if (m != -INFINITY) {
#pragma unroll
      for (int t = 0; t < NS; ++t) {
        const float w = __expf(l[t] - m);
        wsum += w;
        accumulate(w, v[t]);
      }
    }
  } else {
    for (int t = 0; t < nsplit; ++t) m = fmaxf(m, __ldg(part_lse + t * lse_stride + li));
    if (m != -INFINITY) {
      for (int t = 0; t < nsplit; ++t) {
        const float w = __expf(__ldg(part_lse + t * lse_stride + li) - m);
        wsum += w;
        accumulate(w, __ldg(reinterpret_cast<const uint4*>(part_o + t * o_stride + oi)));
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint4 o;
  o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  o.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  o.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(out + oi) = o;
  if (part == 0 && lse != nullptr) lse[li] = m == -INFINITY ? -INFINITY : m + __logf(wsum);
}

}  // namespace nabla
