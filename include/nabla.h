/*
 * nabla.h -- C ABI of libnabla.so: NABLA adaptive block-sparse attention on
 * one NVIDIA B200 (sm_100a).
 *
 * The method (page "Resumo Tecnico: NABLA - Atencao de Bloco Adaptativa de
 * Vizinhanca para Geracao de Video Eficiente", gist.science paper 2507.13546,
 * section "Metodologia: NABLA") has three stages:
 *   1. fractal flattening of the T x H x W token grid
 *   2. adaptive block mask (pool, reduced attention, CDF threshold, optional
 *      STA union)
 *   3. attention on the kept 64 x 64 tiles
 * Two ways to run them:
 *   - on tensors in grid order, without any flattened copy (the flattening
 *     happens in the kernels' loads and stores):
 *       nabla_build_mask_grid (or nabla_flatten_pool_qk in pool-only mode +
 *       nabla_build_mask_pooled), then nabla_sparse_attn_fwd_grid;
 *   - on materialised flattened tensors:
 *       nabla_flatten, nabla_build_mask (or nabla_build_mask_noalloc),
 *       nabla_sparse_attn_fwd, nabla_unflatten.
 * The block lists are plain device buffers: one mask may serve several
 * attention calls (rebuilt every few steps), and nabla_build_mask_sta
 * writes the static window alone, without reading Q or K.
 *
 * Conventions shared by every call
 *   - Tensors are bf16 in BSHD layout [B][S][Hh][D] (D contiguous), S = T*H*W
 *     tokens, Hh heads, head dimension D in {64, 128}.  A block is P*P = 64
 *     consecutive tokens of the flattened order (P = 8), i.e. one 8 x 8 patch
 *     of one frame; Nb = S / 64.  Block lists always index blocks in the
 *     flattened order.
 *   - Every pointer argument is a DEVICE pointer owned by the caller, who
 *     allocates it (the library allocates no device memory) and keeps it alive
 *     until the stream has executed the call.  Inputs and outputs never alias.
 *   - Calls are asynchronous on the given stream (0 = legacy default stream)
 *     and never synchronise, except nabla_get_status.
 *   - CUDA graphs: nabla_flatten, nabla_unflatten, nabla_build_mask,
 *     nabla_build_mask_grid, nabla_flatten_pool_qk, nabla_build_mask_pooled,
 *     nabla_build_mask_sta, nabla_build_mask_radial, the nabla_sparse_attn_fwd
 *     calls (flattened, grid order, key-range split), nabla_transpose_lists,
 *     both nabla_sparse_attn_bwd calls, nabla_ab_plan and nabla_ab_attn_fwd
 *     launch only on the given stream and allocate nothing, so a sequence
 *     of them can be captured into one CUDA graph; replaying it on new data
 *     in the same buffers gives the same bits as making the calls directly.
 *     Make the library's first call on a device outside a capture (it looks
 *     up the device's attributes and the driver's tensor-map encoder).
 *   - Return value: NABLA_OK, or an error code; on error nothing is launched.
 *     Device-side faults of the data (an out-of-range block index, a wait that
 *     ran out of time) are recorded in a per-device status word that
 *     nabla_get_status reads and clears.
 */
#ifndef NABLA_H_
#define NABLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nabla_stream_t; /* same object as cudaStream_t */

enum {
  NABLA_OK = 0,
  NABLA_ERR_INVALID = 1,        /* bad shape or parameter */
  NABLA_ERR_ALIGN = 2,          /* pointer not 16-byte aligned */
  NABLA_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed */
  NABLA_ERR_DEVICE_TIMEOUT = 4, /* (device status) a bounded wait expired */
  NABLA_ERR_DEVICE_BOUNDS = 5,  /* (device status) a block index or count was out of range */
  NABLA_ERR_UNSUPPORTED = 6,    /* no sm_100 device */
  NABLA_ERR_TOO_LARGE = 7       /* problem exceeds NABLA_NOALLOC_SCRATCH_BYTES */
};

/* Mask parameters.
 *   P      patch side; must be 8 (64-token blocks).
 *   thr    CDF threshold in [0, 1]: per row, blocks sorted by probability
 *          ascending are kept where the cumulative mass exceeds 1 - thr
 *          ("Limiarizacao CDF").  thr = 1 keeps every block; the row's
 *          arg-max block is always kept.
 *   sta_t, sta_h, sta_w
 *          Sliding-Tile window in blocks (frames, patch rows, patch columns),
 *          odd sizes; all three 0 disables the STA union ("Integracao Hibrida
 *          com STA", M = M_nabla OR M_STA).  The window is centred on the query
 *          block and truncated at the grid border.
 *   scale  score scale; 0 selects 1/sqrt(D).
 *   flags  reserved, must be 0.
 *   radial radial decay window OR-ed into the mask, the static mask of the
 *          Radial Attention article ("Zastosowanie zasad rozkladu energii":
 *          a neighbourhood window that shrinks as the temporal distance
 *          grows).  0 disables it; r0 = radial >= 1 keeps block j for block
 *          i when their patch rows and columns each differ by at most
 *          r0 >> floor(log2(|ti - tj| + 1)), ti, tj their frames: the
 *          window halves each time the temporal distance (plus one)
 *          doubles, and the co-located block of every frame stays. */
typedef struct {
  int P;
  float thr;
  int sta_t, sta_h, sta_w;
  float scale;
  unsigned flags;
  int radial;
} nabla_params;

/* Fractal flattening ("Metodologia: NABLA", item 1, "Reordenacao de Tokens"):
 * out[b, f(t,h,w), :] = in[b, (t*H + h)*W + w, :] with
 *   f = t*H*W + ((h/P)*(W/P) + w/P)*P*P + (h%P)*P + (w%P),
 * so each P x P spatial patch of a frame becomes P*P contiguous rows and the
 * frames stay in order.
 *   in, out     device bf16 [B][T*H*W][row_elems]; row_elems*2 bytes per row
 *               (e.g. Hh*D), a multiple of 16 bytes; both 16-byte aligned.
 * Errors: NABLA_ERR_INVALID unless P == 8, H % P == 0, W % P == 0, all sizes
 * positive and row_elems % 8 == 0; NABLA_ERR_ALIGN; NABLA_ERR_CUDA. */
int nabla_flatten(const void* in, void* out, int B, int T, int H, int W, int P, int row_elems,
                  nabla_stream_t stream);

/* Inverse of nabla_flatten (same arguments and rules): takes flattened rows
 * back to grid order. */
int nabla_unflatten(const void* in, void* out, int B, int T, int H, int W, int P, int row_elems,
                    nabla_stream_t stream);

/* Bytes of device workspace nabla_build_mask needs: the pooled queries and
 * the pooled keys, both transposed, fp32 [B][Hh][D][Nbp] each with Nbp = Nb
 * rounded up to a multiple of 4 (columns >= Nb are padding), then the
 * block-score scratch, fp32 [B][Hh][Nb][Nbp] (4*B*Hh*Nb*Nbp bytes: 1.4 GB
 * for 24 heads of 3,840 blocks).  Returns 0 for invalid sizes. */
size_t nabla_mask_workspace_bytes(int B, int Hh, int D, int T, int H, int W,
                                  const nabla_params* params);

/* Adaptive block mask ("Metodologia: NABLA", item 2, and item 3):
 *   1. pooling: qbar[b,hd,i,:] = mean of the 64 flattened query rows of block
 *      i (fp32 accumulation, rows in ascending order), same for keys
 *      ("Downsampling");
 *   2. reduced attention: s_ij = (qbar_i . kbar_j) * scale in fp32,
 *      p_i = softmax_j(s_i) ("Atencao Reduzida");
 *   3. CDF threshold as described for nabla_params.thr ("Limiarizacao CDF");
 *   4. optional STA union, then compaction into block lists ("Expansao").
 *   qf, kf      device bf16 [B][S][Hh][D], flattened order.
 *   kv_count    device int32 [B][Hh][Nb]: kept key blocks per query block.
 *   kv_idx      device int32 [B][Hh][Nb][Nb]: row (b,hd,i) holds its kept key
 *               blocks ascending in entries [0, kv_count); later entries are
 *               not written.
 *   workspace   device buffer of nabla_mask_workspace_bytes() bytes, 16-byte
 *               aligned; on return it holds qbar^T, kbar^T and the block
 *               scores s_ij (layouts as for nabla_mask_workspace_bytes).
 * The scores are computed as a tiled fp32 GEMM with the same rounding as
 * the definition above (one fused multiply-add chain over d ascending per
 * entry, then the scale), and each row is thresholded from them. 
 * Errors: NABLA_ERR_INVALID (shape, D not 64/128, thr outside [0,1], even or
 * negative STA sizes, radial outside [0, 65535], flags != 0);
 * NABLA_ERR_ALIGN; NABLA_ERR_CUDA. */
int nabla_build_mask(const void* qf, const void* kf, int B, int Hh, int D, int T, int H, int W,
                     const nabla_params* params, int32_t* kv_count, int32_t* kv_idx,
                     void* workspace, nabla_stream_t stream);

/* Fractal flattening of Q and K fused with the pooling stage of
 * nabla_build_mask: one pass reads q and k (grid order), writes qf and kf
 * (flattened, exactly as nabla_flatten with row_elems = Hh*D) and the pooled
 * queries and transposed keys into `workspace` (layout of
 * nabla_mask_workspace_bytes, identical bits to the pooling inside
 * nabla_build_mask).  Saves the second read of the flattened Q and K.
 *   q, k        device bf16 [B][T*H*W][Hh][D], grid order.
 *   qf, kf      device bf16 [B][T*H*W][Hh][D] outputs, flattened order.
 *   workspace   as for nabla_build_mask.
 * qf and kf may both be NULL: then only the pooled vectors are written (the
 * pooling stage of nabla_build_mask_grid on its own).  The tensors must not
 * alias.  Errors: as nabla_build_mask (params are validated the same way
 * although only P is used here). */
int nabla_flatten_pool_qk(const void* q, const void* k, void* qf, void* kf, int B, int Hh, int D, int T, int H,
                          int W, const nabla_params* params, void* workspace, nabla_stream_t stream);

/* nabla_build_mask on Q and K in GRID order ([B][T*H*W][Hh][D], row of
 * token (t, h, w) = (t*H + h)*W + w): the pooling gathers each block's 64
 * tokens in the flattened order (identical bits to pooling the flattened
 * tensors), then stages 2-4 run as in nabla_build_mask.  Same arguments,
 * results and errors as nabla_build_mask with q, k in place of qf, kf. */
int nabla_build_mask_grid(const void* q, const void* k, int B, int Hh, int D, int T, int H, int W,
                          const nabla_params* params, int32_t* kv_count, int32_t* kv_idx, void* workspace,
                          nabla_stream_t stream);

/* Stages 2-4 of nabla_build_mask (reduced attention, CDF threshold, STA
 * union, compaction) on a workspace that already holds the pooled queries
 * and keys (written by nabla_flatten_pool_qk, nabla_build_mask or
 * nabla_build_mask_grid).  Same
 * arguments, results and errors as nabla_build_mask without qf and kf. */
int nabla_build_mask_pooled(const void* workspace, int B, int Hh, int D, int T, int H, int W,
                            const nabla_params* params, int32_t* kv_count, int32_t* kv_idx, nabla_stream_t stream);

/* The static Sliding-Tile window on its own, M_STA of "Integracao Hibrida
 * com STA" without the content-adaptive term (the pure-STA configuration the
 * summary compares NABLA with, "Comparacao com Metodos Estaticos").  No Q or
 * K is read: row i of every (b, head) lists the blocks j whose frame, patch
 * row and patch column each differ from block i's by at most sta_t/2,
 * sta_h/2, sta_w/2 (window centred on block i, truncated at the grid
 * border), ascending; the lists are the STA part of nabla_build_mask's union
 * with the same window.
 *   P           must be 8; H and W multiples of 8.
 *   sta_t, sta_h, sta_w   odd window sizes in [1, 65535] (in frames, patch
 *               rows, patch columns).
 *   kv_count, kv_idx      as for nabla_build_mask (16-byte aligned).
 * Errors: NABLA_ERR_INVALID (grid, Hh, window sizes, NULL lists);
 * NABLA_ERR_ALIGN; NABLA_ERR_CUDA. */
int nabla_build_mask_sta(int B, int Hh, int T, int H, int W, int P, int sta_t, int sta_h, int sta_w,
                         int32_t* kv_count, int32_t* kv_idx, nabla_stream_t stream);

/* The radial decay window on its own (nabla_params.radial without the
 * content-adaptive term; the static mask the Radial Attention article
 * describes).  No Q or K is read: row i of every (b, head) lists, ascending,
 * the blocks j with |patch row difference| <= rho and |patch column
 * difference| <= rho, rho = r0 >> floor(log2(|ti - tj| + 1)) for frames
 * ti, tj.  The lists are the radial part of nabla_build_mask's union with
 * the same r0.
 *   P           must be 8; H and W multiples of 8.
 *   r0          spatial half-width (in patches) at temporal distance 0, in
 *               [1, 65535].
 *   kv_count, kv_idx   as for nabla_build_mask (16-byte aligned).
 * Errors: NABLA_ERR_INVALID (grid, Hh, r0, NULL lists); NABLA_ERR_ALIGN;
 * NABLA_ERR_CUDA. */
int nabla_build_mask_radial(int B, int Hh, int T, int H, int W, int P, int r0, int32_t* kv_count, int32_t* kv_idx,
                            nabla_stream_t stream);

/* Block-sparse attention forward on the kept tiles ("Expansao": only the
 * listed N x N blocks are computed; a dropped block is in neither the
 * numerator nor the softmax normaliser).  For query block i of (b, hd):
 *   O_i = softmax over the tokens of kv_idx[b,hd,i,0..kv_count) of
 *         (Q_i K^T * scale), applied to V;   LSE = log of the normaliser.
 *   qf, kf, vf  device bf16 [B][S][Hh][D], flattened order, 16-byte aligned;
 *               S a multiple of 64.
 *   kv_count, kv_idx   block lists as written by nabla_build_mask (entries
 *               must be ascending and < Nb; a bad entry is skipped and
 *               recorded as NABLA_ERR_DEVICE_BOUNDS).
 *   scale       0 selects 1/sqrt(D).
 *   out         device bf16 [B][S][Hh][D], flattened order.
 *   lse         device fp32 [B][Hh][S] (natural log) or NULL.
 * A query block with kv_count == 0 gets O = 0 and LSE = -inf.
 * Errors: NABLA_ERR_INVALID (D not 64/128, S % 64 != 0, sizes); NABLA_ERR_ALIGN;
 * NABLA_ERR_CUDA; NABLA_ERR_UNSUPPORTED when the device is not sm_100. */
int nabla_sparse_attn_fwd(const void* qf, const void* kf, const void* vf, const int32_t* kv_count,
                          const int32_t* kv_idx, int B, int S, int Hh, int D, float scale, void* out,
                          float* lse, nabla_stream_t stream);

/* Block-sparse attention on tensors in GRID order: the fractal flattening
 * and its inverse happen inside the kernel, so no flattened copy of Q, K, V
 * or O is ever materialised.  For a T x H x W grid (S = T*H*W, P = 8):
 *   q, k, v   device bf16 [B][S][Hh][D] in grid order: the row of token
 *             (t, h, w) is (t*H + h)*W + w.  Block j of the flattened order
 *             (the 8 x 8 patch (bh, bw) of frame t, j = t*(H/8)*(W/8) +
 *             bh*(W/8) + bw) is fetched by one 5-D TMA box (d, head, w, h,
 *             frame) whose rows come out in the flattened order inside the
 *             block.
 *   kv_count, kv_idx   block lists over flattened block indices, as
 *             written by any of the mask entry points.
 *   out       device bf16 [B][S][Hh][D] in grid order;
 *   lse       fp32 [B][Hh][S] in grid order (or NULL).
 * Results equal nabla_unflatten of nabla_sparse_attn_fwd run on the
 * flattened tensors (up to the summation order of the online softmax, see
 * the pairing below).  Knowing the grid also lets the kernel choose which
 * two query blocks share one 128-row tile: when T and W/8 are even, each
 * 2 x 2 group of patch positions {(t, w), (t, w+1), (t+1, w), (t+1, w+1)}
 * (same patch row) is split along w or along t, whichever leaves fewer key
 * blocks listed by only one of the two (those run as half-masked tiles);
 * with T or W/8 odd the pairs are 2p, 2p+1.  Errors: as
 * nabla_sparse_attn_fwd, plus NABLA_ERR_INVALID unless H and W are
 * multiples of 8. */
int nabla_sparse_attn_fwd_grid(const void* q, const void* k, const void* v, const int32_t* kv_count,
                               const int32_t* kv_idx, int B, int Hh, int D, int T, int H, int W, float scale,
                               void* out, float* lse, nabla_stream_t stream);

/* The same attention as nabla_sparse_attn_fwd_grid with each head's walk
 * split by key range ("Metodologia: NABLA", item 2 "Expansao": the kept
 * tiles are computed, grouped differently): the key blocks are cut into
 * nsplit ranges of ceil(Nb / nsplit) rounded up to 32 blocks; every query
 * tile is attended over each range by its own CTA, all ranges of one head
 * in turn, so the CTAs resident at a time read only one range's K and V
 * (for a mask whose kept blocks are spread over the whole sequence, the
 * L2 then holds that range instead of missing on a whole head).  Each
 * range's output (normalised over the range) and LSE go to the workspace;
 * a second kernel merges them: O = sum_s exp(lse_s - L) O_s, L = log sum_s
 * exp(lse_s).  Results equal nabla_sparse_attn_fwd_grid's up to rounding
 * (the range outputs are stored in bf16 before the merge).
 *   nsplit     2 .. 64 (Hh * nsplit <= 65535)
 *   workspace  device, at least nabla_attn_split_workspace_bytes(...)
 *              bytes, 16-byte aligned, owned by the caller, overwritten.
 * Other arguments and errors as nabla_sparse_attn_fwd_grid; a null or
 * misaligned workspace gives NABLA_ERR_INVALID / NABLA_ERR_ALIGN. */
int nabla_sparse_attn_fwd_grid_split(const void* q, const void* k, const void* v, const int32_t* kv_count,
                                     const int32_t* kv_idx, int B, int Hh, int D, int T, int H, int W, float scale,
                                     int nsplit, void* workspace, void* out, float* lse, nabla_stream_t stream);

/* Bytes of workspace nabla_sparse_attn_fwd_grid_split needs: nsplit range
 * outputs (bf16, B*S*Hh*D each) and their LSE (fp32, B*Hh*S each), S =
 * T*H*W.  0 for invalid arguments (including nsplit < 2). */
size_t nabla_attn_split_workspace_bytes(int B, int Hh, int D, int T, int H, int W, int nsplit);

/* Column (transposed) block lists for the backward pass: for key block j of
 * (b, hd), the query blocks i whose row kv_idx[b,hd,i,0..kv_count) lists j,
 * ascending.
 *   kv_count, kv_idx   row lists as written by the mask entry points
 *               ([B][Hh][Nb], [B][Hh][Nb][Nb], rows ascending).
 *   q_count     device int32 [B][Hh][Nb] output: query blocks per key block.
 *   q_idx       device int32 [B][Hh][Nb][Nb] output: entries [0, q_count)
 *               of row (b,hd,j); later entries are not written.
 * A row whose count is outside [0, Nb] is taken as empty and recorded as
 * NABLA_ERR_DEVICE_BOUNDS.  Errors: NABLA_ERR_INVALID (sizes, B*Hh > 65535,
 * NULL); NABLA_ERR_ALIGN (pointers not 16-byte aligned); NABLA_ERR_CUDA. */
int nabla_transpose_lists(const int32_t* kv_count, const int32_t* kv_idx, int B, int Hh, int Nb, int32_t* q_count,
                          int32_t* q_idx, nabla_stream_t stream);

/* Backward pass of nabla_sparse_attn_fwd over the same kept tiles: the
 * gradients of sum(dO * O) with respect to Q, K and V, for training (the
 * summary's "Aceleracao de Dupla Fase": the method also speeds up
 * pre-training and fine-tuning).  With P the forward's probabilities
 * (recomputed from lse), for query token a and the tokens c of its kept
 * blocks:
 *   Delta_a = dO_a . O_a,  dS_ac = P_ac (dO_a . v_c - Delta_a),
 *   dQ_a = scale sum_c dS_ac k_c,  dK_c = scale sum_a dS_ac q_a,
 *   dV_c = sum_a P_ac dO_a;
 * a key block kept by no row gets dK = dV = 0, an empty row dQ = 0.
 *   qf, kf, vf, out, dout   device bf16 [B][S][Hh][D], flattened order: the
 *               forward's inputs, its output O and the output gradient.
 *   lse         device fp32 [B][Hh][S]: the forward's LSE.
 *   kv_count, kv_idx   the forward's row lists; q_count, q_idx their
 *               transpose (nabla_transpose_lists).
 *   scale       0 selects 1/sqrt(D) (must match the forward).
 *   dq, dk, dv  device bf16 [B][S][Hh][D] outputs (every element written).
 *   delta       device fp32 [B][Hh][S] workspace, written with Delta.
 * Each output element is computed by one CTA in a fixed order: results are
 * deterministic.  Errors: as nabla_sparse_attn_fwd (every pointer required,
 * B and Hh at most 65535); list faults are recorded as for the forward. */
int nabla_sparse_attn_bwd(const void* qf, const void* kf, const void* vf, const void* out, const void* dout,
                          const float* lse, const int32_t* kv_count, const int32_t* kv_idx, const int32_t* q_count,
                          const int32_t* q_idx, int B, int S, int Hh, int D, float scale, void* dq, void* dk,
                          void* dv, float* delta, nabla_stream_t stream);

/* nabla_sparse_attn_bwd on tensors in GRID order (as nabla_sparse_attn_fwd_grid
 * reads and writes them): q, k, v, out, dout, dq, dk, dv [B][T*H*W][Hh][D]
 * and lse, delta [B][Hh][T*H*W] indexed by the grid row (t*H + h)*W + w;
 * the block lists index blocks in the flattened order.  Results equal
 * nabla_sparse_attn_bwd on the flattened tensors, permuted back.  Errors:
 * as nabla_sparse_attn_bwd, plus NABLA_ERR_INVALID unless H and W are
 * multiples of 8. */
int nabla_sparse_attn_bwd_grid(const void* q, const void* k, const void* v, const void* out, const void* dout,
                               const float* lse, const int32_t* kv_count, const int32_t* kv_idx,
                               const int32_t* q_count, const int32_t* q_idx, int B, int Hh, int D, int T, int H,
                               int W, float scale, void* dq, void* dk, void* dv, float* delta,
                               nabla_stream_t stream);

/* Same mask as nabla_build_mask, for callers that cannot allocate device
 * memory.  This entry point has no counterpart in the paper; it exists for
 * code that hands the library only its input and output buffers: a plug-in
 * host or serving runtime that owns all device memory and exposes no
 * allocator, or a latency-critical path where cudaMalloc's implicit
 * device-wide synchronisation is not acceptable.
 *   The pooled queries and keys (the first part of nabla_build_mask's
 *   workspace, 8*B*Hh*D*Nbp bytes) live in a static device buffer of
 *   NABLA_NOALLOC_SCRATCH_BYTES inside the library; the block scores are
 *   kept in shared memory instead of a scratch.  Every GPU that loads the
 *   library holds that buffer until the process exits.  The call allocates
 *   nothing and frees nothing.
 *   Arguments, layouts and results are those of nabla_build_mask without the
 *   workspace argument.  A problem whose pooled vectors exceed
 *   NABLA_NOALLOC_SCRATCH_BYTES is rejected with NABLA_ERR_TOO_LARGE before
 *   anything is launched.
 *   Every call looks up the buffer's device address (cudaGetSymbolAddress,
 *   with the caller's device current), so nothing is cached across a
 *   context teardown; make a first call before any stream capture.
 *   All calls share the one buffer and each call overwrites it completely:
 *   calls that overlap on the GPU (other streams, other host threads) race
 *   on it, so the caller must order them. */
#define NABLA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int nabla_build_mask_noalloc(const void* qf, const void* kf, int B, int Hh, int D, int T, int H, int W,
                             const nabla_params* params, int32_t* kv_count, int32_t* kv_idx,
                             nabla_stream_t stream);

/* ---------------------------------------------------------------------
 * AB-Attention, a second sparse-attention scheme over the same tensors
 * (news page "AB-Attention acelera a geracao de video em ate 2,23x e pula
 * 92% da atencao", section "Os tres recursos do AB-Attention"), on tensors
 * in their original (grid) order -- the scheme does not permute tokens.
 * Query blocks are 128 consecutive tokens (NQB = S / 128), key blocks 4
 * consecutive tokens (NKB = S / 4).  nabla_ab_plan builds the sampling plan
 * (the page re-plans every few denoising steps); nabla_ab_attn_fwd runs the
 * attention on it.
 * --------------------------------------------------------------------- */

/* Bytes of device workspace nabla_ab_plan needs: the mean keys (transposed,
 * fp32 [B][Hh][D][NKB]), the centroids (transposed, fp32 [B][Hh][D][NQB*8]),
 * the cluster counts (int32 [B][Hh][NQB][8]) and the centroid logits (fp32
 * [B][Hh][NQB*8][NKB]), each region 256-byte aligned, in that order
 * (2.9 GB for 12 heads of 61,440 tokens).  Returns 0 for invalid sizes. */
size_t nabla_ab_workspace_bytes(int B, int S, int Hh, int D);

/* The sampling plan ("IBCS" and "SIP"):
 *   1. mean key of every 4-token block (fp32, tokens in order, * 0.25);
 *   2. per 128-query block, 8 clusters by kmeans_iters Lloyd iterations
 *      from the queries at positions 0, 16, ..., 112: squared distances as
 *      an fp32 fused multiply-add chain over d of the rounded differences,
 *      ties to the lower cluster; each centroid the fp32 mean of its
 *      queries (empty clusters keep theirs); weight = count / 128;
 *   3. block scores s_J = sum_c weight_c softmax_J(cent_c . kbar_J * scale);
 *   4. inclusion probabilities pi_J = min(1, lambda s_J) with
 *      sum_J pi_J = budget (water-filling); key block J is sampled iff
 *      u_J < pi_J, and gets the logit shift -log(pi_J) (its
 *      Horvitz-Thompson weight 1 / pi_J).
 *   q, k        device bf16 [B][S][Hh][D], S a multiple of 128.
 *   u           device fp32 [B][Hh][NQB][NKB]: the uniform random numbers
 *               in [0, 1) of the sampling (the caller draws them).
 *   kmeans_iters  0 .. 64;  budget  expected sample size per query block;
 *   scale       0 selects 1/sqrt(D).
 *   kcount      device int32 [B][Hh][NQB] output: sampled key blocks.
 *   kidx        device int32 [B][Hh][NQB][NKB] output: sampled blocks
 *               ascending in entries [0, kcount); later entries unwritten.
 *   kshift      device fp32 [B][Hh][NQB][NKB] output: entry e's shift.
 *   workspace   nabla_ab_workspace_bytes() bytes, 16-byte aligned.
 * Steps 1-2 and the logits of step 3 follow the fp32 definition above
 * operation for operation; pi is computed with expf and sums in the GPU's
 * order (within about 1e-7 of the exact value).  The NKB block scores of a
 * row are held in shared memory (NKB <= about 50,000).
 * Errors: NABLA_ERR_INVALID (shapes, iterations, budget, scale, NULL);
 * NABLA_ERR_ALIGN; NABLA_ERR_CUDA. */
int nabla_ab_plan(const void* q, const void* k, const float* u, int B, int S, int Hh, int D, int kmeans_iters,
                  double budget, float scale, int32_t* kcount, int32_t* kidx, float* kshift, void* workspace,
                  nabla_stream_t stream);

/* Attention of every 128-query block over its sampled 4-token key blocks,
 * each key's logit shifted by its block's kshift:
 *   O_a = softmax_c((q_a . k_c) * scale + kshift(c)) V, LSE = log of the
 *   normaliser; the sampled blocks are gathered by index into 64-key
 *   tensor-core tiles (16 blocks each).
 *   q, k, v     device bf16 [B][S][Hh][D], grid order, 16-byte aligned.
 *   kcount, kidx, kshift   as written by nabla_ab_plan (entries in [0, NKB);
 *               a bad entry is skipped and recorded as
 *               NABLA_ERR_DEVICE_BOUNDS).
 *   out         device bf16 [B][S][Hh][D]; lse fp32 [B][Hh][S] or NULL.
 * A query block with no sampled block gets O = 0, LSE = -inf.
 * Errors: as nabla_sparse_attn_fwd. */
int nabla_ab_attn_fwd(const void* q, const void* k, const void* v, const int32_t* kcount, const int32_t* kidx,
                      const float* kshift, int B, int S, int Hh, int D, float scale, void* out, float* lse,
                      nabla_stream_t stream);

/* Synchronises the stream, then returns and clears the current device's
 * status word (NABLA_OK, NABLA_ERR_DEVICE_TIMEOUT or NABLA_ERR_DEVICE_BOUNDS),
 * or NABLA_ERR_CUDA if the synchronisation itself failed. */
int nabla_get_status(nabla_stream_t stream);

/* Debug check of block lists on the device: every row must have
 * 1 <= count <= Nb and strictly ascending entries in [0, Nb).  Writes the
 * number of bad rows to *bad_rows (device int32, zeroed by the call).
 * Asynchronous like the others. */
int nabla_validate_mask(const int32_t* kv_count, const int32_t* kv_idx, int B, int Hh, int Nb,
                        int32_t* bad_rows, nabla_stream_t stream);

/* Failure-detection self-test (no counterpart in the paper): launches one CTA
 * whose threads wait on an mbarrier that nothing arrives on, using the same
 * bounded wait as the kernels with a limit of limit_cycles SM cycles
 * (1000 .. 4e9).  The wait gives up, records NABLA_ERR_DEVICE_TIMEOUT in the
 * status word and the kernel returns normally, so the context stays usable;
 * read the code with nabla_get_status.  NABLA_ERR_INVALID for a limit out of
 * range. */
int nabla_selftest_wait_timeout(long long limit_cycles, nabla_stream_t stream);

/* Static description of an error code. */
const char* nabla_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* NABLA_H_ */
