/*
 * CPU oracle for NABLA block-sparse attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, scalar C that restates what the method computes so the CUDA
 * path can be checked against it.  Only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load this library; the product path
 * never calls it and shares no code with it.
 *
 * Source of every step: the page "Resumo Tecnico: NABLA - Atencao de Bloco
 * Adaptativa de Vizinhanca para Geracao de Video Eficiente" (gist.science,
 * paper 2507.13546), section "Metodologia: NABLA":
 *   item 1  "Reordenacao de Tokens (Fractal Flattening)"       -> oracle_flatten
 *   item 2  "Downsampling"                                     -> oracle_pool
 *           "Atencao Reduzida"                -> block_numerators, block_probs
 *           "Limiarizacao CDF"                                 -> cdf_keep_row
 *           "Expansao"                                         -> kv lists
 *   item 3  "Integracao Hibrida com STA", M = M_nabla OR M_STA -> sta_keep
 * The Radial Attention article's static decay mask as another OR-term
 * (aisight.pl, "Zastosowanie zasad rozkladu energii")       -> radial_keep
 * and the attention on the kept N x N blocks (same section, "Expansao"),
 * with dropped blocks absent from both numerator and normaliser (the
 * AB-Attention news page, section "Onde os esquemas esparsos anteriores
 * falham", second bullet) -> oracle_attention.
 * Also: the window mask on its own (item 3 without the adaptive term; the
 * summary's "Comparacao com Metodos Estaticos") -> oracle_sta_lists; and the
 * gradient of the attention on the kept blocks, for the training the
 * summary says NABLA also speeds up ("Aceleracao de Dupla Fase")
 * -> oracle_attention_bwd, oracle_attention_bwd_sampled.
 *
 * Precision: the mask is fp32 (pooled vectors, scores, exponentials,
 * probabilities) with fp64 accumulation of the softmax normaliser and of the
 * CDF; attention accumulates in fp64.  Build with -ffp-contract=off so every
 * a*b+c below is two roundings, as written.
 *
 * Parity pins (each in tests/): see the functions' comments.  Functions with
 * no external pin say "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BLOCK 64 /* N = P*P tokens per block, P = 8 */

static inline float bf16_bits_to_f32(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads of the OpenMP loops from now on (n >= 1).  Every loop is over
 * independent rows, so results do not depend on it; the benchmark uses it
 * to time the oracle on one core as well as on all of them. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* Fractal flattening (NABLA summary, Metodologia item 1).                   */
/* Grid order s = (t*H + h)*W + w.  Flattened order: frame-major, then the   */
/* P x P patch (bh, bw) row-major, then the token inside the patch           */
/* row-major:  f = t*H*W + (bh*nbw + bw)*P*P + (h%P)*P + (w%P).              */
/* Pinned by: an independent reshape/transpose formulation, bijectivity,     */
/* unflatten(flatten(x)) == x, and the T=1,H=W=P identity case.              */
/* ------------------------------------------------------------------------ */
static int64_t flat_index(int t, int h, int w, int H, int W, int P) {
  int nbw = W / P;
  int bh = h / P, bw = w / P;
  return (int64_t)t * H * W + (int64_t)(bh * nbw + bw) * P * P + (h % P) * P + (w % P);
}

void oracle_flatten(const uint16_t* in, uint16_t* out, int B, int T, int H, int W, int P,
                    int64_t row_elems) {
  int64_t S = (int64_t)T * H * W;
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t)
      for (int h = 0; h < H; ++h)
        for (int w = 0; w < W; ++w) {
          int64_t src = ((int64_t)t * H + h) * W + w;
          int64_t dst = flat_index(t, h, w, H, W, P);
          memcpy(out + (b * S + dst) * row_elems, in + (b * S + src) * row_elems,
                 (size_t)row_elems * 2);
        }
}

void oracle_unflatten(const uint16_t* in, uint16_t* out, int B, int T, int H, int W, int P,
                      int64_t row_elems) {
  int64_t S = (int64_t)T * H * W;
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t)
      for (int h = 0; h < H; ++h)
        for (int w = 0; w < W; ++w) {
          int64_t grid = ((int64_t)t * H + h) * W + w;
          int64_t flat = flat_index(t, h, w, H, W, P);
          memcpy(out + (b * S + grid) * row_elems, in + (b * S + flat) * row_elems,
                 (size_t)row_elems * 2);
        }
}

/* ------------------------------------------------------------------------ */
/* Block average pooling (NABLA summary, Metodologia item 2, "Downsampling"):*/
/* xbar[b,hd,i,:] = (sum_{r=0..63} x[b, 64 i + r, hd, :]) / 64, summed in    */
/* fp32 with r ascending; dividing by 64 is exact.                           */
/* x is flattened BSHD bf16 [B][S][Hh][D]; xbar is fp32 [B][Hh][Nb][D].      */
/* Pinned by bilinearity: qbar_i . kbar_j equals the mean of the 64 x 64     */
/* token-logit tile (checked in fp64).                                       */
/* ------------------------------------------------------------------------ */
void oracle_pool(const uint16_t* x, float* xbar, int B, int S, int Hh, int D) {
  int Nb = S / ORACLE_BLOCK;
  for (int b = 0; b < B; ++b)
    for (int hd = 0; hd < Hh; ++hd)
      for (int i = 0; i < Nb; ++i)
        for (int d = 0; d < D; ++d) {
          float acc = 0.0f;
          for (int r = 0; r < ORACLE_BLOCK; ++r) {
            int64_t tok = (int64_t)i * ORACLE_BLOCK + r;
            acc = acc + bf16_bits_to_f32(x[(((int64_t)b * S + tok) * Hh + hd) * D + d]);
          }
          xbar[(((int64_t)b * Hh + hd) * Nb + i) * D + d] = acc * (1.0f / 64.0f);
        }
}

/* ------------------------------------------------------------------------ */
/* Reduced attention (NABLA summary, "Atencao Reduzida"): one row i of the   */
/* block-level softmax, in fp32 as the method's mask stage is:               */
/*   s_ij = fl32(sum_d qbar_id * kbar_jd) * scale, the sum a chain of fused  */
/*          multiply-adds in ascending d (fmaf), then one fp32 multiply;     */
/*   m    = max_j s_ij;                                                      */
/*   e_j  = exp(s_ij - m) correctly rounded to fp32 (s - m in fp32, exp in   */
/*          fp64, then rounded): the softmax numerators, 0 < e_j <= 1;       */
/*   Z    = sum_j e_j in fp64 (j ascending);  p_j = fl32(e_j / Z).           */
/* block_numerators stops at e; block_probs goes on to p.                    */
/* Pinned by: scores against the fp64 mean of token logits; sum p = 1 within */
/* Nb * 2^-24; the all-equal-scores case giving exactly 1/Nb.                */
/* ------------------------------------------------------------------------ */
static void block_numerators(const float* qbar_i, const float* kbar, int Nb, int D, float scale,
                             float* e) {
  float m = -INFINITY;
  for (int j = 0; j < Nb; ++j) {
    float dot = 0.0f;
    for (int d = 0; d < D; ++d) dot = fmaf(qbar_i[d], kbar[(int64_t)j * D + d], dot);
    float s = dot * scale;
    e[j] = s;
    if (s > m) m = s;
  }
  for (int j = 0; j < Nb; ++j) e[j] = (float)exp((double)(e[j] - m));
}

static void block_probs(const float* qbar_i, const float* kbar, int Nb, int D, float scale,
                        float* p) {
  block_numerators(qbar_i, kbar, Nb, D, scale, p);
  double Z = 0.0;
  for (int j = 0; j < Nb; ++j) Z += (double)p[j];
  for (int j = 0; j < Nb; ++j) p[j] = (float)((double)p[j] / Z);
}

typedef struct {
  float w;
  int j;
} wj_t;

/* Ascending by weight, ties by ascending block index. */
static int cmp_wj(const void* a, const void* b) {
  const wj_t* x = (const wj_t*)a;
  const wj_t* y = (const wj_t*)b;
  if (x->w < y->w) return -1;
  if (x->w > y->w) return 1;
  return (x->j > y->j) - (x->j < y->j);
}

/* ------------------------------------------------------------------------ */
/* CDF thresholding (NABLA summary, "Limiarizacao CDF"): sort the row's       */
/* probabilities ascending, take the running sum c_k and keep the block at   */
/* position k iff c_k > 1 - thr.  thr >= 1 keeps every block; the arg-max    */
/* (last position) is always kept.                                           */
/* The row is given as weights w_j >= 0 whose normalised values w_j / sum(w) */
/* are the probabilities (the softmax numerators e_j, or the probabilities   */
/* themselves).  All probabilities of a row share one normaliser, so their   */
/* ascending order is the ascending order of the weights, ties by ascending  */
/* block index; rounding each quotient to fp32 first would merge distinct    */
/* neighbours into ties the method does not have.                            */
/*   Z = sum_j w_j (fp64, j ascending);  c_k = (w_(0) + ... + w_(k)) / Z,    */
/* the running sum in fp64 in the sorted order.  cum[j] receives c at block  */
/* j's position.  band[j] (if not NULL) marks blocks whose cumulative mass   */
/* lies within band_width of 1 - thr.                                        */
/* Pinned by: an exact-rational top-p (nucleus) restatement on real rows,    */
/* kept mass >= thr and minimality, and the uniform Nb=16 case.              */
/* ------------------------------------------------------------------------ */
static int cdf_keep_row(const float* w, int Nb, float thr, uint8_t* keep, double* cum,
                        uint8_t* band, double band_width, wj_t* scratch) {
  double Z = 0.0;
  for (int j = 0; j < Nb; ++j) {
    scratch[j].w = w[j];
    scratch[j].j = j;
    Z += (double)w[j];
  }
  qsort(scratch, (size_t)Nb, sizeof(wj_t), cmp_wj);
  double tau = 1.0 - (double)thr;
  double run = 0.0;
  for (int k = 0; k < Nb; ++k) {
    run += (double)scratch[k].w;
    double c = run / Z;
    int j = scratch[k].j;
    cum[j] = c;
    keep[j] = (uint8_t)((thr >= 1.0f) || (c > tau) || (k == Nb - 1));
  }
  if (band)
    for (int j = 0; j < Nb; ++j) band[j] = (uint8_t)(fabs(cum[j] - tau) < band_width);
  return scratch[Nb - 1].j; /* the arg-max block */
}

/* ------------------------------------------------------------------------ */
/* Sliding Tile Attention window in block space (NABLA summary, Metodologia  */
/* item 3): blocks i=(ti,hi,wi) and j=(tj,hj,wj) interact iff each           */
/* coordinate differs by at most floor(window/2); the window is centred and  */
/* truncated at the grid border.  A window size of 0 disables STA.           */
/* Pinned by the closed-form per-row count prod_axis(min(x+r,n-1) -          */
/* max(x-r,0) + 1) and its totals per configuration.                         */
/* ------------------------------------------------------------------------ */
static int sta_keep(int i, int j, int nbh, int nbw, int st, int sh, int sw) {
  if (st <= 0 || sh <= 0 || sw <= 0) return 0;
  int per_t = nbh * nbw;
  int ti = i / per_t, hi = (i % per_t) / nbw, wi = i % nbw;
  int tj = j / per_t, hj = (j % per_t) / nbw, wj = j % nbw;
  return abs(ti - tj) <= st / 2 && abs(hi - hj) <= sh / 2 && abs(wi - wj) <= sw / 2;
}

/* ------------------------------------------------------------------------ */
/* Radial window in block space (Radial Attention article, aisight.pl,       */
/* "Radial Attention: Efektywnosc bez kompromisow" and "Zastosowanie zasad   */
/* rozkladu energii": a static mask that keeps interactions mostly within    */
/* the spatiotemporal neighbourhood, its window shrinking as the temporal    */
/* distance grows, the kept attention decaying exponentially in space and   */
/* time).  The page gives no formula; the reading here: blocks              */
/* i=(ti,hi,wi) and j=(tj,hj,wj) at temporal distance dt = |ti - tj| fall in */
/* band r = floor(log2(dt + 1)) (dt 0; 1-2; 3-6; 7-14; ...), whose spatial   */
/* half-width is rho = floor(r0 / 2^r): the window halves each time the     */
/* temporal distance doubles.  keep iff |hi - hj| <= rho and                 */
/* |wi - wj| <= rho (the co-located block of every frame is always kept).    */
/* r0 <= 0 disables the window.                                              */
/* Pinned by: the closed-form per-row count (sum over frames of the clipped */
/* box areas), an enumeration of the window written independently with     */
/* floating-point log2, symmetry, and monotone shrinking in dt.             */
/* ------------------------------------------------------------------------ */
static int radial_band(int dt) {
  int r = 0;
  while ((dt + 1) >> (r + 1)) ++r;
  return r;
}

static int radial_keep(int i, int j, int nbh, int nbw, int r0) {
  if (r0 <= 0) return 0;
  int per_t = nbh * nbw;
  int ti = i / per_t, hi = (i % per_t) / nbw, wi = i % nbw;
  int tj = j / per_t, hj = (j % per_t) / nbw, wj = j % nbw;
  int rho = r0 >> radial_band(abs(ti - tj));
  return abs(hi - hj) <= rho && abs(wi - wj) <= rho;
}

/* The radial window on its own as block lists for one (b, head), as        */
/* oracle_sta_lists does for the sliding-tile window.                        */
void oracle_radial_lists(int Nb, int nbh, int nbw, int r0, int32_t* kv_count, int32_t* kv_idx) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int i = 0; i < Nb; ++i) {
    int n = 0;
    for (int j = 0; j < Nb; ++j)
      if (radial_keep(i, j, nbh, nbw, r0)) kv_idx[(int64_t)i * Nb + n++] = j;
    kv_count[i] = n;
  }
}

/* Radial predicate for one block pair (see radial_keep). */
int oracle_radial(int i, int j, int nbh, int nbw, int r0) { return radial_keep(i, j, nbh, nbw, r0); }

/* ------------------------------------------------------------------------ */
/* Full mask construction for every (b, head, query block) row, producing    */
/* the block-CSR lists consumed by the attention ("Expansao"), with the     */
/* static windows (sliding tile, radial) OR-ed into the adaptive mask:      */
/*   kv_count[b,hd,i]   number of kept key blocks                            */
/*   kv_idx[b,hd,i,:]   kept key-block indices ascending (row stride Nb)      */
/* status (optional, [B,Hh,Nb,Nb] uint8): bit0 = kept, bit1 = band block     */
/* (decided by the CDF alone, cumulative mass within `band` of 1 - thr).     */
/* probs (optional, [B,Hh,Nb,Nb] fp32): the row probabilities p.             */
/* qbar/kbar: fp32 [B][Hh][Nb][D].  Rows are independent; OpenMP splits them */
/* without changing any element's arithmetic.                                */
/* ------------------------------------------------------------------------ */
void oracle_mask(const float* qbar, const float* kbar, int B, int Hh, int Nb, int D, float scale,
                 float thr, int nbh, int nbw, int sta_t, int sta_h, int sta_w, int radial_r0, double band,
                 int32_t* kv_count, int32_t* kv_idx, uint8_t* status, float* probs) {
  int64_t rows = (int64_t)B * Hh * Nb;
#pragma omp parallel
  {
    float* e = (float*)malloc(sizeof(float) * (size_t)Nb);
    uint8_t* keep = (uint8_t*)malloc((size_t)Nb);
    uint8_t* bandf = (uint8_t*)malloc((size_t)Nb);
    double* cum = (double*)malloc(sizeof(double) * (size_t)Nb);
    wj_t* scratch = (wj_t*)malloc(sizeof(wj_t) * (size_t)Nb);
#pragma omp for schedule(dynamic, 4)
    for (int64_t row = 0; row < rows; ++row) {
      int64_t bh = row / Nb;
      int i = (int)(row % Nb);
      const float* qi = qbar + (bh * Nb + i) * D;
      const float* kb = kbar + bh * Nb * D;
      block_numerators(qi, kb, Nb, D, scale, e);
      double Z = 0.0;
      for (int j = 0; j < Nb; ++j) Z += (double)e[j];
      int argmax = cdf_keep_row(e, Nb, thr, keep, cum, status ? bandf : NULL, band, scratch);
      int32_t n = 0;
      for (int j = 0; j < Nb; ++j) {
        int cdf_kept = keep[j];
        int sta = sta_keep(i, j, nbh, nbw, sta_t, sta_h, sta_w) || radial_keep(i, j, nbh, nbw, radial_r0);
        int kept = cdf_kept || sta;
        if (kept) kv_idx[row * Nb + n++] = j;
        if (status) {
          /* A block is "band" only when the CDF comparison alone decides it. */
          int forced = sta || thr >= 1.0f || j == argmax;
          int in_band = !forced && bandf[j];
          status[row * Nb + j] = (uint8_t)(kept | (in_band << 1));
        }
        if (probs) probs[row * Nb + j] = (float)((double)e[j] / Z);
      }
      kv_count[row] = n;
    }
    free(e);
    free(keep);
    free(bandf);
    free(cum);
    free(scratch);
  }
}

/* ------------------------------------------------------------------------ */
/* Attention restricted to the kept 64 x 64 tiles ("Expansao"), for the      */
/* query blocks listed in qblocks (all heads).  For query token a of block i */
/* and every token c of the kept blocks of row (b,hd,i):                     */
/*   l = (sum_d q_a,d k_c,d) * scale (fp64),  w = exp(l - max_c l),          */
/*   O_a = sum_c w v_c / sum_c w,   LSE_a = max + log(sum_c w).              */
/* Dropped tiles enter neither numerator nor normaliser.  A row with no kept */
/* block gives O = 0 and LSE = -inf.                                         */
/* kv_count: int32 [B][Hh][nq] and kv_idx: int32 [B][Hh][nq][Nb] hold the    */
/* lists of the listed query blocks only, in qblocks order.                  */
/* out: fp64 [B][nq*64][Hh][D]; lse: fp64 [B][Hh][nq*64] (may be NULL).      */
/* Pinned by: thr=1 equals dense softmax attention computed independently in */
/* grid order; V constant -> O constant; Q = 0 -> O = mean of kept V;        */
/* a row keeping only its own block equals tile-local attention.             */
/* ------------------------------------------------------------------------ */
void oracle_attention(const uint16_t* qf, const uint16_t* kf, const uint16_t* vf,
                      const int32_t* kv_count, const int32_t* kv_idx, int B, int S, int Hh, int D,
                      double scale, const int32_t* qblocks, int nq, double* out, double* lse) {
  int Nb = S / ORACLE_BLOCK;
  int64_t units = (int64_t)B * Hh * nq * ORACLE_BLOCK;
#pragma omp parallel
  {
    double* logit = (double*)malloc(sizeof(double) * (size_t)S);
    double* acc = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 16)
    for (int64_t u = 0; u < units; ++u) {
      int r = (int)(u % ORACLE_BLOCK);
      int64_t t1 = u / ORACLE_BLOCK;
      int qn = (int)(t1 % nq);
      int64_t t2 = t1 / nq;
      int hd = (int)(t2 % Hh);
      int b = (int)(t2 / Hh);
      int i = qblocks[qn];
      int64_t a = (int64_t)i * ORACLE_BLOCK + r;
      int64_t row = ((int64_t)b * Hh + hd) * nq + qn;
      int cnt = kv_count[row];
      const int32_t* lst = kv_idx + row * Nb;
      const uint16_t* q = qf + (((int64_t)b * S + a) * Hh + hd) * D;
      int64_t out_row = (int64_t)qn * ORACLE_BLOCK + r;
      double* o = out + (((int64_t)b * nq * ORACLE_BLOCK + out_row) * Hh + hd) * D;
      double mx = -INFINITY;
      int64_t n = 0;
      for (int e = 0; e < cnt; ++e) {
        int j = lst[e];
        for (int c = 0; c < ORACLE_BLOCK; ++c) {
          int64_t tok = (int64_t)j * ORACLE_BLOCK + c;
          const uint16_t* k = kf + (((int64_t)b * S + tok) * Hh + hd) * D;
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += (double)bf16_bits_to_f32(q[d]) * (double)bf16_bits_to_f32(k[d]);
          double l = dot * scale;
          logit[n++] = l;
          if (l > mx) mx = l;
        }
      }
      for (int d = 0; d < D; ++d) acc[d] = 0.0;
      double den = 0.0;
      n = 0;
      for (int e = 0; e < cnt; ++e) {
        int j = lst[e];
        for (int c = 0; c < ORACLE_BLOCK; ++c) {
          int64_t tok = (int64_t)j * ORACLE_BLOCK + c;
          const uint16_t* v = vf + (((int64_t)b * S + tok) * Hh + hd) * D;
          double w = exp(logit[n++] - mx);
          den += w;
          for (int d = 0; d < D; ++d) acc[d] += w * (double)bf16_bits_to_f32(v[d]);
        }
      }
      for (int d = 0; d < D; ++d) o[d] = cnt > 0 ? acc[d] / den : 0.0;
      if (lse) lse[((int64_t)b * Hh + hd) * nq * ORACLE_BLOCK + out_row] = cnt > 0 ? mx + log(den) : -INFINITY;
    }
    free(logit);
    free(acc);
  }
}

/* Probability row for one (b, head, i): exposed so tests can pin the softmax
 * and CDF steps on their own. */
void oracle_block_probs_row(const float* qbar, const float* kbar, int Nb, int D, float scale,
                            int i, float* p_out) {
  block_probs(qbar + (int64_t)i * D, kbar, Nb, D, scale, p_out);
}

/* Softmax numerators e of one (b, head, i) row (see block_numerators). */
void oracle_block_numerators_row(const float* qbar, const float* kbar, int Nb, int D, float scale,
                                 int i, float* e_out) {
  block_numerators(qbar + (int64_t)i * D, kbar, Nb, D, scale, e_out);
}

/* CDF keep decision for one row of weights (see cdf_keep_row). */
int oracle_cdf_keep(const float* w, int Nb, float thr, uint8_t* keep, double* cum, uint8_t* band,
                    double band_width) {
  wj_t* scratch = (wj_t*)malloc(sizeof(wj_t) * (size_t)Nb);
  int argmax = cdf_keep_row(w, Nb, thr, keep, cum, band, band_width, scratch);
  free(scratch);
  return argmax;
}

/* STA predicate for one block pair (see sta_keep). */
int oracle_sta(int i, int j, int nbh, int nbw, int sta_t, int sta_h, int sta_w) {
  return sta_keep(i, j, nbh, nbw, sta_t, sta_h, sta_w);
}

/* ------------------------------------------------------------------------ */
/* The static window on its own, M_STA (Metodologia item 3 without the      */
/* content-adaptive term; the "pure STA" configurations the summary compares */
/* NABLA with under "Comparacao com Metodos Estaticos"): for every query     */
/* block i, the blocks j with sta_keep(i, j) in ascending order.  The lists  */
/* depend only on the grid, so this fills one (b, head):                     */
/*   kv_count[i], kv_idx[i*Nb + 0..kv_count[i])                              */
/* Entries past the count are left as they are.  Pinned by the closed-form   */
/* per-row counts (any window), the identity lists of a 1x1x1 window, the    */
/* full lists of a window covering the grid, and an enumeration of the       */
/* window by coordinates written independently in the tests.                 */
/* ------------------------------------------------------------------------ */
void oracle_sta_lists(int Nb, int nbh, int nbw, int sta_t, int sta_h, int sta_w, int32_t* kv_count,
                      int32_t* kv_idx) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int i = 0; i < Nb; ++i) {
    int n = 0;
    for (int j = 0; j < Nb; ++j)
      if (sta_keep(i, j, nbh, nbw, sta_t, sta_h, sta_w)) kv_idx[(int64_t)i * Nb + n++] = j;
    kv_count[i] = n;
  }
}

/* ------------------------------------------------------------------------ */
/* Gradient of the attention on the kept tiles (the backward pass a training  */
/* step needs: the summary states that NABLA speeds up both pre-training /   */
/* fine-tuning and inference, "Principais Contribuicoes", "Aceleracao de     */
/* Dupla Fase", and reports pre-training iteration times, "Resultados        */
/* Experimentais" item 2).  It is the exact derivative of oracle_attention   */
/* on the same lists, written out with the chain rule, in fp64: for query    */
/* token a of block i and every token c of the kept blocks of its row,       */
/*   P_ac  = softmax_c(l_ac),  l_ac = (q_a . k_c) * scale                    */
/*   dP_ac = dO_a . v_c                                                      */
/*   dS_ac = P_ac * (dP_ac - sum_c' P_ac' dP_ac')     (softmax Jacobian)     */
/*   dV_c += P_ac dO_a,  dQ_a += scale dS_ac k_c,  dK_c += scale dS_ac q_a.  */
/* A dropped tile contributes nothing; a token kept by no row gets dK = dV = */
/* 0; a row with no kept block gets dQ = 0.                                  */
/* qf, kf, vf, dof: bf16 bits [B][S][Hh][D] (flattened order); lists as for  */
/* nabla's forward ([B][Hh][Nb], [B][Hh][Nb][Nb]).  dq, dk, dv: fp64         */
/* [B][S][Hh][D], overwritten.  OpenMP over (b, head): each head's dK, dV    */
/* are accumulated by one thread in query order.                             */
/* Pinned by: autograd (fp64) of a token-level masked softmax attention      */
/* built from the lists; sum_c dK_c = 0 and sum_c dV_c = sum_a dO_a over     */
/* rows with kept blocks; zero gradients for unkept key blocks and empty     */
/* rows.                                                                     */
/* ------------------------------------------------------------------------ */
void oracle_attention_bwd(const uint16_t* qf, const uint16_t* kf, const uint16_t* vf, const uint16_t* dof,
                          const int32_t* kv_count, const int32_t* kv_idx, int B, int S, int Hh, int D,
                          double scale, double* dq, double* dk, double* dv) {
  int Nb = S / ORACLE_BLOCK;
  int64_t n_all = (int64_t)B * S * Hh * D;
  for (int64_t x = 0; x < n_all; ++x) dq[x] = dk[x] = dv[x] = 0.0;
#pragma omp parallel
  {
    double* pr = (double*)malloc(sizeof(double) * (size_t)S);
    double* dp = (double*)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < (int64_t)B * Hh; ++bh) {
      int b = (int)(bh / Hh), hd = (int)(bh % Hh);
#define ORACLE_AT(base, tok) ((base) + (((int64_t)b * S + (tok)) * Hh + hd) * D)
      for (int i = 0; i < Nb; ++i) {
        int64_t row = bh * Nb + i;
        int cnt = kv_count[row];
        const int32_t* lst = kv_idx + row * Nb;
        for (int r = 0; r < ORACLE_BLOCK; ++r) {
          int64_t a = (int64_t)i * ORACLE_BLOCK + r;
          const uint16_t* q = ORACLE_AT(qf, a);
          const uint16_t* g = ORACLE_AT(dof, a);
          /* probabilities of the row */
          double mx = -INFINITY, den = 0.0;
          int64_t n = 0;
          for (int e = 0; e < cnt; ++e)
            for (int c = 0; c < ORACLE_BLOCK; ++c) {
              const uint16_t* k = ORACLE_AT(kf, (int64_t)lst[e] * ORACLE_BLOCK + c);
              double dot = 0.0;
              for (int d = 0; d < D; ++d) dot += (double)bf16_bits_to_f32(q[d]) * (double)bf16_bits_to_f32(k[d]);
              pr[n] = dot * scale;
              if (pr[n] > mx) mx = pr[n];
              ++n;
            }
          for (int64_t c = 0; c < n; ++c) {
            pr[c] = exp(pr[c] - mx);
            den += pr[c];
          }
          for (int64_t c = 0; c < n; ++c) pr[c] /= den;
          /* dP and the softmax Jacobian's row term sum_c P dP */
          double pdp = 0.0;
          n = 0;
          for (int e = 0; e < cnt; ++e)
            for (int c = 0; c < ORACLE_BLOCK; ++c) {
              const uint16_t* v = ORACLE_AT(vf, (int64_t)lst[e] * ORACLE_BLOCK + c);
              double dot = 0.0;
              for (int d = 0; d < D; ++d) dot += (double)bf16_bits_to_f32(g[d]) * (double)bf16_bits_to_f32(v[d]);
              dp[n] = dot;
              pdp += pr[n] * dot;
              ++n;
            }
          double* dqa = ORACLE_AT(dq, a);
          n = 0;
          for (int e = 0; e < cnt; ++e)
            for (int c = 0; c < ORACLE_BLOCK; ++c) {
              int64_t tok = (int64_t)lst[e] * ORACLE_BLOCK + c;
              const uint16_t* k = ORACLE_AT(kf, tok);
              double* dkc = ORACLE_AT(dk, tok);
              double* dvc = ORACLE_AT(dv, tok);
              double ds = pr[n] * (dp[n] - pdp);
              for (int d = 0; d < D; ++d) {
                dvc[d] += pr[n] * (double)bf16_bits_to_f32(g[d]);
                dqa[d] += scale * ds * (double)bf16_bits_to_f32(k[d]);
                dkc[d] += scale * ds * (double)bf16_bits_to_f32(q[d]);
              }
              ++n;
            }
        }
      }
#undef ORACLE_AT
    }
    free(pr);
    free(dp);
  }
}

/* ------------------------------------------------------------------------ */
/* The same gradient as oracle_attention_bwd, restricted to listed blocks so */
/* that full-size layers can be checked on a sample: dQ for the query blocks */
/* in qblocks (nq of them) and dK, dV for the key blocks in kblocks (nk).    */
/* dQ of a query token needs only its own row; dK, dV of a key token need    */
/* every row that keeps its block, so those rows are evaluated in full (the  */
/* row's softmax and its sum_c P dP run over all of the row's kept tokens).  */
/* Arithmetic per row as in oracle_attention_bwd.                            */
/* dq: fp64 [B][nq*64][Hh][D] (qblocks order); dk, dv: fp64 [B][nk*64][Hh][D] */
/* (kblocks order); all overwritten.  Either list may be empty (n = 0).      */
/* Pinned by: autograd of the token-level masked attention on the listed     */
/* blocks.                                                                   */
/* ------------------------------------------------------------------------ */
void oracle_attention_bwd_sampled(const uint16_t* qf, const uint16_t* kf, const uint16_t* vf,
                                  const uint16_t* dof, const int32_t* kv_count, const int32_t* kv_idx, int B,
                                  int S, int Hh, int D, double scale, const int32_t* qblocks, int nq,
                                  const int32_t* kblocks, int nk, double* dq, double* dk, double* dv) {
  int Nb = S / ORACLE_BLOCK;
  int* qpos = (int*)malloc(sizeof(int) * (size_t)Nb);
  int* kpos = (int*)malloc(sizeof(int) * (size_t)Nb);
  for (int j = 0; j < Nb; ++j) qpos[j] = kpos[j] = -1;
  for (int x = 0; x < nq; ++x) qpos[qblocks[x]] = x;
  for (int x = 0; x < nk; ++x) kpos[kblocks[x]] = x;
  for (int64_t x = 0; x < (int64_t)B * nq * ORACLE_BLOCK * Hh * D; ++x) dq[x] = 0.0;
  for (int64_t x = 0; x < (int64_t)B * nk * ORACLE_BLOCK * Hh * D; ++x) dk[x] = dv[x] = 0.0;
#pragma omp parallel
  {
    double* pr = (double*)malloc(sizeof(double) * (size_t)S);
    double* dp = (double*)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < (int64_t)B * Hh; ++bh) {
      int b = (int)(bh / Hh), hd = (int)(bh % Hh);
#define ORACLE_AT(base, tok) ((base) + (((int64_t)b * S + (tok)) * Hh + hd) * D)
#define ORACLE_OUT(base, n, pos, r) ((base) + (((int64_t)b * (n) * ORACLE_BLOCK + (int64_t)(pos) * ORACLE_BLOCK + (r)) * Hh + hd) * D)
      for (int i = 0; i < Nb; ++i) {
        int64_t row = bh * Nb + i;
        int cnt = kv_count[row];
        const int32_t* lst = kv_idx + row * Nb;
        int needed = qpos[i] >= 0;
        for (int e = 0; e < cnt && !needed; ++e) needed = kpos[lst[e]] >= 0;
        if (!needed) continue;
        for (int r = 0; r < ORACLE_BLOCK; ++r) {
          int64_t a = (int64_t)i * ORACLE_BLOCK + r;
          const uint16_t* q = ORACLE_AT(qf, a);
          const uint16_t* g = ORACLE_AT(dof, a);
          double mx = -INFINITY, den = 0.0, pdp = 0.0;
          int64_t n = 0;
          for (int e = 0; e < cnt; ++e)
            for (int c = 0; c < ORACLE_BLOCK; ++c) {
              const uint16_t* k = ORACLE_AT(kf, (int64_t)lst[e] * ORACLE_BLOCK + c);
              double dot = 0.0;
              for (int d = 0; d < D; ++d) dot += (double)bf16_bits_to_f32(q[d]) * (double)bf16_bits_to_f32(k[d]);
              pr[n] = dot * scale;
              if (pr[n] > mx) mx = pr[n];
              ++n;
            }
          for (int64_t c = 0; c < n; ++c) {
            pr[c] = exp(pr[c] - mx);
            den += pr[c];
          }
          for (int64_t c = 0; c < n; ++c) pr[c] /= den;
          n = 0;
          for (int e = 0; e < cnt; ++e)
            for (int c = 0; c < ORACLE_BLOCK; ++c) {
              const uint16_t* v = ORACLE_AT(vf, (int64_t)lst[e] * ORACLE_BLOCK + c);
              double dot = 0.0;
              for (int d = 0; d < D; ++d) dot += (double)bf16_bits_to_f32(g[d]) * (double)bf16_bits_to_f32(v[d]);
              dp[n] = dot;
              pdp += pr[n] * dot;
              ++n;
            }
          double* dqa = qpos[i] >= 0 ? ORACLE_OUT(dq, nq, qpos[i], r) : NULL;
          n = 0;
          for (int e = 0; e < cnt; ++e) {
            int kp = kpos[lst[e]];
            for (int c = 0; c < ORACLE_BLOCK; ++c) {
              const uint16_t* k = ORACLE_AT(kf, (int64_t)lst[e] * ORACLE_BLOCK + c);
              double ds = pr[n] * (dp[n] - pdp);
              if (dqa)
                for (int d = 0; d < D; ++d) dqa[d] += scale * ds * (double)bf16_bits_to_f32(k[d]);
              if (kp >= 0) {
                double* dkc = ORACLE_OUT(dk, nk, kp, c);
                double* dvc = ORACLE_OUT(dv, nk, kp, c);
                for (int d = 0; d < D; ++d) {
                  dvc[d] += pr[n] * (double)bf16_bits_to_f32(g[d]);
                  dkc[d] += scale * ds * (double)bf16_bits_to_f32(q[d]);
                }
              }
              ++n;
            }
          }
        }
      }
#undef ORACLE_OUT
#undef ORACLE_AT
    }
    free(pr);
    free(dp);
  }
  free(qpos);
  free(kpos);
}

/* ======================================================================== */
/* AB-Attention (news page "AB-Attention acelera a geracao de video em ate  */
/* 2,23x e pula 92% da atencao", section "Os tres recursos do AB-Attention")*/
/* as a second workload over the same token tensors, kept in their original */
/* (grid) order: the page says the tokens are not permuted.                 */
/*   IBCS: query blocks of 128 tokens, 8 clusters per block, each with a     */
/*         centroid and a weight = its fraction of the block's queries; a   */
/*         key block is scored by the weighted attention of the centroids   */
/*         to its mean key.                                                 */
/*   SIP:  a key block enters the sample with probability proportional to   */
/*         its score, the most important ones always; a sampled block counts */
/*         1 / (inclusion probability) times (Horvitz-Thompson), applied as  */
/*         a logit shift of -log(pi).                                       */
/*   Key blocks of 4 tokens, gathered by index.                             */
/* Readings where the page is silent: k-means starts from the queries at    */
/* positions 0, 16, ..., 112 of the block and runs `iters` Lloyd iterations  */
/* (assignment to the nearest centroid by squared distance, ties to the      */
/* lower cluster; each centroid becomes the mean of its queries, an empty   */
/* cluster keeps its centroid); the weights come from the last assignment.  */
/* The score softmax runs over all key blocks of the (b, head), scale       */
/* 1/sqrt(D).  Inclusion probabilities pi = min(1, lambda * score) with      */
/* lambda such that sum(pi) equals the sampling budget (the expected number  */
/* of sampled blocks); a block is sampled iff u < pi for its uniform random */
/* number u, drawn outside and passed in.                                   */
/* ======================================================================== */
#define AB_QBLOCK 128
#define AB_CLUSTERS 8
#define AB_KBLOCK 4

/* Mean key of every 4-token block: kbar[b][hd][J][d] = (sum_{r<4} k[b][4J+r]
 * [hd][d], fp32, r ascending) * 0.25.  k is bf16 [B][S][Hh][D], grid order.
 * Pinned by: the fp64 block mean. */
void oracle_ab_key_means(const uint16_t* k, int B, int S, int Hh, int D, float* kbar) {
  int nkb = S / AB_KBLOCK;
  for (int b = 0; b < B; ++b)
    for (int hd = 0; hd < Hh; ++hd)
      for (int J = 0; J < nkb; ++J)
        for (int d = 0; d < D; ++d) {
          float acc = 0.0f;
          for (int r = 0; r < AB_KBLOCK; ++r)
            acc = acc + bf16_bits_to_f32(k[(((int64_t)b * S + (int64_t)J * AB_KBLOCK + r) * Hh + hd) * D + d]);
          kbar[(((int64_t)b * Hh + hd) * nkb + J) * D + d] = acc * 0.25f;
        }
}

/* Squared distance, fp32: diff = x - mu rounded, then a fused multiply-add  */
/* chain over d ascending. */
static float ab_dist(const float* x, const float* mu, int D) {
  float acc = 0.0f;
  for (int d = 0; d < D; ++d) {
    float diff = x[d] - mu[d];
    acc = fmaf(diff, diff, acc);
  }
  return acc;
}

/* IBCS clustering of every 128-query block (see the section comment):      */
/* cent [B][Hh][NQB][8][D] fp32, counts [B][Hh][NQB][8] int32, assign         */
/* [B][Hh][S] int32 (may be NULL).  Centroid update: fp32 sum of the         */
/* cluster's queries in ascending token order, divided by the count (one     */
/* fp32 division).  Pinned by: recovery of well-separated clusters, each    */
/* centroid the mean of its queries, each query at its nearest centroid of   */
/* the last assignment, and non-increasing within-cluster sum of squares.   */
void oracle_ab_kmeans(const uint16_t* q, int B, int S, int Hh, int D, int iters, float* cent, int32_t* counts,
                      int32_t* assign_out) {
  int nqb = S / AB_QBLOCK;
#pragma omp parallel
  {
    float* x = (float*)malloc(sizeof(float) * AB_QBLOCK * (size_t)D);
    float* mu = (float*)malloc(sizeof(float) * AB_CLUSTERS * (size_t)D);
    float* acc = (float*)malloc(sizeof(float) * (size_t)D);
    int asg[AB_QBLOCK];
    int cnt[AB_CLUSTERS];
#pragma omp for schedule(dynamic, 4)
    for (int64_t u = 0; u < (int64_t)B * Hh * nqb; ++u) {
      int I = (int)(u % nqb);
      int64_t bh = u / nqb;
      int b = (int)(bh / Hh), hd = (int)(bh % Hh);
      for (int t = 0; t < AB_QBLOCK; ++t)
        for (int d = 0; d < D; ++d)
          x[t * D + d] = bf16_bits_to_f32(q[(((int64_t)b * S + (int64_t)I * AB_QBLOCK + t) * Hh + hd) * D + d]);
      for (int c = 0; c < AB_CLUSTERS; ++c)
        for (int d = 0; d < D; ++d) mu[c * D + d] = x[(c * (AB_QBLOCK / AB_CLUSTERS)) * D + d];
      for (int c = 0; c < AB_CLUSTERS; ++c) cnt[c] = 0;
      for (int it = 0; it < iters; ++it) {
        for (int t = 0; t < AB_QBLOCK; ++t) {
          int best = 0;
          float bd = ab_dist(x + t * D, mu, D);
          for (int c = 1; c < AB_CLUSTERS; ++c) {
            float dd = ab_dist(x + t * D, mu + c * D, D);
            if (dd < bd) {
              bd = dd;
              best = c;
            }
          }
          asg[t] = best;
        }
        for (int c = 0; c < AB_CLUSTERS; ++c) {
          int n = 0;
          for (int d = 0; d < D; ++d) acc[d] = 0.0f;
          for (int t = 0; t < AB_QBLOCK; ++t)
            if (asg[t] == c) {
              for (int d = 0; d < D; ++d) acc[d] = acc[d] + x[t * D + d];
              ++n;
            }
          cnt[c] = n;
          if (n > 0)
            for (int d = 0; d < D; ++d) mu[c * D + d] = acc[d] / (float)n;
        }
      }
      for (int c = 0; c < AB_CLUSTERS; ++c) {
        counts[u * AB_CLUSTERS + c] = cnt[c];
        for (int d = 0; d < D; ++d) cent[(u * AB_CLUSTERS + c) * D + d] = mu[c * D + d];
      }
      if (assign_out)
        for (int t = 0; t < AB_QBLOCK; ++t) assign_out[bh * S + (int64_t)I * AB_QBLOCK + t] = asg[t];
    }
    free(x);
    free(mu);
    free(acc);
  }
}

/* IBCS block scores: for query block I and every key block J,              */
/*   l_cJ = fl32(fmaf chain over d of cent_c . kbar_J) * scale,            */
/*   a_cJ = exp(l_cJ - max_J l_cJ) / sum_J exp(...)   (fp64),               */
/*   score_IJ = sum_c (counts_c / 128) * a_cJ        (fp64, c ascending;    */
/*              empty clusters have weight 0).                              */
/* score [B][Hh][NQB][NKB] fp64.  Pinned by: an fp64 restatement with numpy, */
/* sum_J score = 1, and the single-cluster case equal to one softmax.       */
void oracle_ab_scores(const float* cent, const int32_t* counts, const float* kbar, int B, int Hh, int nqb, int nkb,
                      int D, float scale, double* score) {
#pragma omp parallel
  {
    float* l = (float*)malloc(sizeof(float) * (size_t)nkb);
#pragma omp for schedule(dynamic, 4)
    for (int64_t u = 0; u < (int64_t)B * Hh * nqb; ++u) {
      int64_t bh = u / nqb;
      const float* kb = kbar + bh * nkb * D;
      double* s = score + u * nkb;
      for (int J = 0; J < nkb; ++J) s[J] = 0.0;
      for (int c = 0; c < AB_CLUSTERS; ++c) {
        int n = counts[u * AB_CLUSTERS + c];
        if (n == 0) continue;
        const float* mu = cent + (u * AB_CLUSTERS + c) * D;
        float m = -INFINITY;
        for (int J = 0; J < nkb; ++J) {
          float dot = 0.0f;
          for (int d = 0; d < D; ++d) dot = fmaf(mu[d], kb[(int64_t)J * D + d], dot);
          l[J] = dot * scale;
          if (l[J] > m) m = l[J];
        }
        double Z = 0.0;
        for (int J = 0; J < nkb; ++J) Z += exp((double)l[J] - (double)m);
        double w = (double)n / (double)AB_QBLOCK;
        for (int J = 0; J < nkb; ++J) s[J] += w * (exp((double)l[J] - (double)m) / Z);
      }
    }
    free(l);
  }
}

typedef struct {
  double s;
  int j;
} sj_t;

static int cmp_sj_desc(const void* a, const void* b) {
  const sj_t* x = (const sj_t*)a;
  const sj_t* y = (const sj_t*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->j > y->j) - (x->j < y->j);
}

/* SIP inclusion probabilities of one row of n scores for an expected sample */
/* size `budget`: pi_J = min(1, lambda * s_J) with sum_J pi_J = budget.      */
/* With the scores sorted descending, the first m blocks are capped at 1,   */
/* m the smallest count for which lambda = (budget - m) / (sum of the rest)  */
/* leaves the largest remaining score below 1 / lambda.  A budget at or     */
/* above the number of positive scores samples every positive-score block.  */
/* Returns lambda.  Pinned by: sum pi = budget, pi proportional to s below  */
/* the cap, the capped blocks' lambda * s >= 1, and an exact-rational       */
/* restatement.                                                             */
double oracle_ab_inclusion(const double* s, int n, double budget, double* pi) {
  sj_t* v = (sj_t*)malloc(sizeof(sj_t) * (size_t)n);
  double* tail = (double*)malloc(sizeof(double) * ((size_t)n + 1));
  int npos = 0;
  for (int j = 0; j < n; ++j) {
    v[j].s = s[j];
    v[j].j = j;
    npos += s[j] > 0.0;
  }
  qsort(v, (size_t)n, sizeof(sj_t), cmp_sj_desc);
  tail[n] = 0.0;
  for (int k = n - 1; k >= 0; --k) tail[k] = tail[k + 1] + v[k].s; /* smallest first */
  double lambda = 0.0;
  int m = 0;
  if (budget >= (double)npos) {
    m = npos;
    lambda = INFINITY;
  } else {
    while (m < npos) {
      lambda = (budget - (double)m) / tail[m];
      if (lambda * v[m].s < 1.0) break;
      ++m;
    }
  }
  for (int k = 0; k < n; ++k) {
    int j = v[k].j;
    pi[j] = v[k].s <= 0.0 ? 0.0 : (k < m ? 1.0 : lambda * v[k].s);
  }
  free(v);
  free(tail);
  return lambda;
}

/* Inclusion probabilities for every (b, head, query block) row of scores. */
void oracle_ab_inclusion_all(const double* score, int64_t rows, int nkb, double budget, double* pi) {
#pragma omp parallel for schedule(dynamic, 8)
  for (int64_t r = 0; r < rows; ++r) oracle_ab_inclusion(score + r * nkb, nkb, budget, pi + r * nkb);
}

/* Attention of the query blocks listed in qblocks (all heads) over their   */
/* sampled 4-token key blocks, each logit shifted by that block's shift     */
/* (-log pi for the Horvitz-Thompson weight 1 / pi):                        */
/*   l = (q_a . k_c) * scale + shift_J(c),  O_a = softmax(l) V,  LSE.       */
/* kcount [B][Hh][nq], kidx [B][Hh][nq][NKB] (sampled blocks ascending),     */
/* shift [B][Hh][nq][NKB] fp64 (entry e belongs to kidx entry e); q, k, v    */
/* bf16 [B][S][Hh][D] in grid order.  out fp64 [B][nq*128][Hh][D], lse fp64  */
/* [B][Hh][nq*128].  A row with no sampled block gives O = 0, LSE = -inf.   */
/* Pinned by: unbiasedness of the numerator and the normaliser over every   */
/* sample of a small case, weighted by its probability (exact enumeration), */
/* and equality with dense attention when every block is sampled with pi=1. */
void oracle_ab_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* kcount,
                         const int32_t* kidx, const double* shift, int B, int S, int Hh, int D, double scale,
                         const int32_t* qblocks, int nq, double* out, double* lse) {
  int nkb = S / AB_KBLOCK;
  int64_t units = (int64_t)B * Hh * nq * AB_QBLOCK;
#pragma omp parallel
  {
    double* logit = (double*)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(dynamic, 16)
    for (int64_t u = 0; u < units; ++u) {
      int r = (int)(u % AB_QBLOCK);
      int64_t t1 = u / AB_QBLOCK;
      int qn = (int)(t1 % nq);
      int64_t t2 = t1 / nq;
      int hd = (int)(t2 % Hh), b = (int)(t2 / Hh);
      int64_t row = ((int64_t)b * Hh + hd) * nq + qn;
      int cnt = kcount[row];
      const int32_t* lst = kidx + row * nkb;
      const double* sh = shift + row * nkb;
      int64_t a = (int64_t)qblocks[qn] * AB_QBLOCK + r;
      const uint16_t* qa = q + (((int64_t)b * S + a) * Hh + hd) * D;
      double mx = -INFINITY;
      int64_t n = 0;
      for (int e = 0; e < cnt; ++e)
        for (int c = 0; c < AB_KBLOCK; ++c) {
          const uint16_t* kc = k + (((int64_t)b * S + (int64_t)lst[e] * AB_KBLOCK + c) * Hh + hd) * D;
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += (double)bf16_bits_to_f32(qa[d]) * (double)bf16_bits_to_f32(kc[d]);
          logit[n] = dot * scale + sh[e];
          if (logit[n] > mx) mx = logit[n];
          ++n;
        }
      double* o = out + (((int64_t)b * nq * AB_QBLOCK + (int64_t)qn * AB_QBLOCK + r) * Hh + hd) * D;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      double den = 0.0;
      n = 0;
      for (int e = 0; e < cnt; ++e)
        for (int c = 0; c < AB_KBLOCK; ++c) {
          const uint16_t* vc = v + (((int64_t)b * S + (int64_t)lst[e] * AB_KBLOCK + c) * Hh + hd) * D;
          double w = exp(logit[n++] - mx);
          den += w;
          for (int d = 0; d < D; ++d) o[d] += w * (double)bf16_bits_to_f32(vc[d]);
        }
      for (int d = 0; d < D; ++d) o[d] = cnt > 0 ? o[d] / den : 0.0;
      if (lse) lse[((int64_t)b * Hh + hd) * nq * AB_QBLOCK + (int64_t)qn * AB_QBLOCK + r] = cnt > 0 ? mx + log(den) : -INFINITY;
    }
    free(logit);
  }
}
