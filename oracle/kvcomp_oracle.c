/*
 * CPU oracle for the attention-score-driven KV selection and compaction path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it. It shares no code, header, table or constant with the
 * CUDA path. It is plain, slow, double-precision C that restates each step of
 * the method in the order and notation of the pages:
 *
 *   [AudioKV]  AudioKV blog post ("1. 音频语言模型中的KV缓存挑战 ..."),
 *              §1.2 (raw importance scores), §2.2 (Spectral Score Smoothing),
 *              §3.1 (head-aware allocation), §5.1 (deployment parameters).
 *   [AudioKV-abs] "AudioKV: KV Cache Eviction in Efficient Large Audio
 *              Language Models" (arxivlens abstract): SSS is an FFT low-pass.
 *   [VoxZip]   "VoxZip: Semantic-Anchored Temporal KV Cache Compression for
 *              Long-Context Audio Inference", 方法概述和架构, second stage
 *              (Temporally Decayed KV Cache Eviction): the A^(t) update and the
 *              Concat(K[:T], K[I_hist], K[-M:]) rule; 细节详述 (gamma, T, M).
 *   [C3]       "C3: Speech-Guided KV Retrieval for Long-Context SpeechLLM
 *              Inference": the budget bypass (audio length <= B keeps all).
 *
 * Readings of points the pages leave open are marked READING in the comments.
 *
 * Parity status: every function here is pinned by closed forms, invariants,
 * brute force or an independent library routine in tests/test_oracle_*.py.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC -pthread
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif

/* ------------------------------------------------------------------------- */
/* A tiny thread pool: run fn(i, ctx) for i in [0, n) on up to n_threads.     */
/* ------------------------------------------------------------------------- */
typedef void (*orc_task_fn)(int64_t i, void* ctx);
typedef struct {
  orc_task_fn fn;
  void* ctx;
  int64_t n;
  int64_t next;
  pthread_mutex_t mu;
} orc_pool;

static void* orc_worker(void* arg) {
  orc_pool* p = (orc_pool*)arg;
  for (;;) {
    pthread_mutex_lock(&p->mu);
    int64_t i = p->next++;
    pthread_mutex_unlock(&p->mu);
    if (i >= p->n) break;
    p->fn(i, p->ctx);
  }
  return NULL;
}

static void orc_parallel(int64_t n, int n_threads, orc_task_fn fn, void* ctx) {
  if (n_threads <= 1 || n <= 1) {
    for (int64_t i = 0; i < n; ++i) fn(i, ctx);
    return;
  }
  if (n_threads > n) n_threads = (int)n;
  orc_pool p = {fn, ctx, n, 0, PTHREAD_MUTEX_INITIALIZER};
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
  int started = 0;
  for (int t = 0; t < n_threads; ++t)
    if (pthread_create(&th[t], NULL, orc_worker, &p) == 0) ++started;
  if (started == 0) orc_worker(&p);
  for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
  free(th);
}

/* ------------------------------------------------------------------------- */
/* Step 1. Observation-window importance scores ([AudioKV] §1.2 names the raw */
/* importance scores of SnapKV/AdaKV that SSS smooths).                       */
/* s_j = sum over the R = g*w window queries r of softmax_j(q_r . K_j / sqrt d)*/
/* READING: every one of the L audio keys is visible to every window query    */
/* (no causal mask), no pooling, a sum (not a mean) over the group's heads.   */
/* ------------------------------------------------------------------------- */
void orc_score_row(const float* q, int R, const float* K, int64_t L, int d, double* s) {
  double* x = (double*)malloc(sizeof(double) * (size_t)L);
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int64_t j = 0; j < L; ++j) s[j] = 0.0;
  for (int r = 0; r < R; ++r) {
    const float* qr = q + (size_t)r * d;
    double m = -INFINITY;
    for (int64_t j = 0; j < L; ++j) {
      const float* kj = K + (size_t)j * d;
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += (double)qr[c] * (double)kj[c];
      x[j] = dot * inv_sqrt_d;
      if (x[j] > m) m = x[j];
    }
    double Z = 0.0;
    for (int64_t j = 0; j < L; ++j) {
      x[j] = exp(x[j] - m);
      Z += x[j];
    }
    for (int64_t j = 0; j < L; ++j) s[j] += x[j] / Z;
  }
  free(x);
}

typedef struct {
  const int64_t* L;
  const int64_t* key_off;
  const float* qwin;
  int R, d;
  const float* K;
  double* s;
} score_ctx;

static void score_task(int64_t i, void* vctx) {
  score_ctx* c = (score_ctx*)vctx;
  orc_score_row(c->qwin + (size_t)i * c->R * c->d, c->R, c->K + (size_t)c->key_off[i] * c->d,
                c->L[i], c->d, c->s + c->key_off[i]);
}

/* rows: qwin [n_rows][R][d]; K concatenated [sum L][d] (row i starts at key_off[i]);
 * s concatenated like K's rows. */
void orc_score_rows(int64_t n_rows, const int64_t* L, const int64_t* key_off, const float* qwin, int R,
                    int d, const float* K, double* s, int n_threads) {
  score_ctx c = {L, key_off, qwin, R, d, K, s};
  orc_parallel(n_rows, n_threads, score_task, &c);
}

/* ------------------------------------------------------------------------- */
/* Step 2. Spectral Score Smoothing ([AudioKV] §2.2; [AudioKV-abs]).          */
/*   F = RFFT(s); E(k) = sum_{i<=k} |F_i|^2; k* = min{k : E(k) >= rho E(L/2)};  */
/*   s_hat = (1 - alpha) s + alpha * IRFFT(F . lowpass(k*)).                   */
/* READINGS: the garbled blend reads s_hat = (1-a)s + a*IRFFT(F.w); the filter */
/* w is the brick wall 1[i <= k*]; E starts at the DC bin and uses one-sided   */
/* bins without doubling; IRFFT has numpy irfft semantics (1/L scaling, real   */
/* parts of bins 0 and L/2 only); L is even.                                    */
/* ------------------------------------------------------------------------- */

/* cos/sin(2 pi m / L) for m in [0, L): angles reduced exactly by index. */
static void twiddles(int64_t L, double* c, double* sn) {
  for (int64_t m = 0; m < L; ++m) {
    double a = 2.0 * M_PI * (double)m / (double)L;
    c[m] = cos(a);
    sn[m] = sin(a);
  }
}

/* Direct DFT, bins i = 0..L/2: F_i = sum_n s_n exp(-2 pi i i n / L). */
void orc_rdft(const double* s, int64_t L, double* re, double* im) {
  double* c = (double*)malloc(sizeof(double) * (size_t)L);
  double* sn = (double*)malloc(sizeof(double) * (size_t)L);
  twiddles(L, c, sn);
  for (int64_t i = 0; i <= L / 2; ++i) {
    double a = 0.0, b = 0.0;
    int64_t m = 0; /* (i * n) mod L */
    for (int64_t n = 0; n < L; ++n) {
      a += s[n] * c[m];
      b -= s[n] * sn[m];
      m += i;
      if (m >= L) m -= L;
    }
    re[i] = a;
    im[i] = b;
  }
  free(c);
  free(sn);
}

/* Energy prefix E(k), k = 0..L/2, summed in index order; returns k*. */
int64_t orc_kstar(const double* re, const double* im, int64_t L, double rho, double* E) {
  double acc = 0.0;
  for (int64_t i = 0; i <= L / 2; ++i) {
    acc += re[i] * re[i] + im[i] * im[i];
    E[i] = acc;
  }
  double thr = rho * E[L / 2];
  for (int64_t k = 0; k <= L / 2; ++k)
    if (E[k] >= thr) return k;
  return L / 2;
}

/* y = IRFFT(F . 1[i <= kstar], n = L), direct sum:
 * y_n = (1/L) [ Re F_0 + 2 sum_{0<i<=k*, i<L/2} Re(F_i e^{+2 pi i i n/L})
 *               + (k* = L/2 ? Re F_{L/2} (-1)^n : 0) ]. */
void orc_irdft_lowpass(const double* re, const double* im, int64_t L, int64_t kstar, double* y) {
  double* c = (double*)malloc(sizeof(double) * (size_t)L);
  double* sn = (double*)malloc(sizeof(double) * (size_t)L);
  twiddles(L, c, sn);
  int64_t top = kstar < L / 2 ? kstar : L / 2 - 1;
  for (int64_t n = 0; n < L; ++n) {
    double acc = re[0];
    int64_t m = 0; /* (i * n) mod L */
    for (int64_t i = 1; i <= top; ++i) {
      m += n;
      if (m >= L) m -= L;
      acc += 2.0 * (re[i] * c[m] - im[i] * sn[m]);
    }
    if (kstar >= L / 2) acc += (n % 2 == 0 ? re[L / 2] : -re[L / 2]);
    y[n] = acc / (double)L;
  }
  free(c);
  free(sn);
}

/* One row. kstar_force < 0: compute k*; else smooth at the given k*. */
void orc_sss_row(const double* s, int64_t L, double alpha, double rho, int64_t kstar_force,
                 double* s_hat, int64_t* kstar_out, double* E_out) {
  int64_t nb = L / 2 + 1;
  double* re = (double*)malloc(sizeof(double) * (size_t)nb);
  double* im = (double*)malloc(sizeof(double) * (size_t)nb);
  double* E = E_out ? E_out : (double*)malloc(sizeof(double) * (size_t)nb);
  double* y = (double*)malloc(sizeof(double) * (size_t)L);
  orc_rdft(s, L, re, im);
  int64_t ks = orc_kstar(re, im, L, rho, E);
  if (kstar_force >= 0) ks = kstar_force;
  orc_irdft_lowpass(re, im, L, ks, y);
  for (int64_t n = 0; n < L; ++n) s_hat[n] = (1.0 - alpha) * s[n] + alpha * y[n];
  *kstar_out = ks;
  free(re);
  free(im);
  if (!E_out) free(E);
  free(y);
}

typedef struct {
  const int64_t* L;
  const int64_t* off;
  const double* s;
  double alpha, rho;
  const int64_t* kstar_force;
  double* s_hat;
  int64_t* kstar;
} sss_ctx;

static void sss_task(int64_t i, void* vctx) {
  sss_ctx* c = (sss_ctx*)vctx;
  int64_t kf = c->kstar_force ? c->kstar_force[i] : -1;
  orc_sss_row(c->s + c->off[i], c->L[i], c->alpha, c->rho, kf, c->s_hat + c->off[i], &c->kstar[i], NULL);
}

void orc_sss_rows(int64_t n_rows, const int64_t* L, const int64_t* off, const double* s, double alpha,
                  double rho, const int64_t* kstar_force, double* s_hat, int64_t* kstar, int n_threads) {
  sss_ctx c = {L, off, s, alpha, rho, kstar_force, s_hat, kstar};
  orc_parallel(n_rows, n_threads, sss_task, &c);
}

/* ------------------------------------------------------------------------- */
/* Step 3. Head-aware budget allocation ([AudioKV] §3.1, §5.1).               */
/*   b_{l,h} = w + r B_rem / H + (1 - r) B_rem S_{l,h} / sum_h S_{l,h}          */
/* READINGS: per layer over that layer's H KV heads; budget_pct is the kept   */
/* fraction, B = floor(pct L H / 100) in integers, B_rem = B - H w; b_h =      */
/* floor(x_h), the remainder B - sum b_h goes +1 to the largest fractional     */
/* parts (ties to the lower head); a head with b_h > L is capped at L and the  */
/* others are re-allocated with what is left; sum S = 0 splits evenly.         */
/* Evaluation order (fixed): t1 = r*B_rem; t1 = t1/H; t2 = (1-r)*B_rem;        */
/* t2 = t2*S_h; t2 = t2/sumS; x = (w + t1) + t2, all in double, no FMA.        */
/* Returns 0, or 3 when B_rem < 0 (budget below H*w).                          */
/* ------------------------------------------------------------------------- */
static int alloc_layer(int H, int64_t L, int w, int64_t B, double r, const float* S, int32_t* b) {
  int active[1024];
  double xs[1024];
  int n_act = 0;
  for (int h = 0; h < H; ++h) active[n_act++] = h;
  int64_t B_left = B;
  for (;;) {
    if (n_act == 0) return 0;
    int64_t B_rem = B_left - (int64_t)n_act * w;
    if (B_rem < 0) return 3;
    double sumS = 0.0;
    for (int a = 0; a < n_act; ++a) sumS += (double)S[active[a]];
    int64_t sum_b = 0;
    for (int a = 0; a < n_act; ++a) {
      int h = active[a];
      double x;
      if (sumS > 0.0) {
        double t1 = r * (double)B_rem;
        t1 = t1 / (double)n_act;
        double t2 = (1.0 - r) * (double)B_rem;
        t2 = t2 * (double)S[h];
        t2 = t2 / sumS;
        x = ((double)w + t1) + t2;
      } else {
        x = (double)w + (double)B_rem / (double)n_act;
      }
      xs[a] = x;
      b[h] = (int32_t)floor(x);
      sum_b += b[h];
    }
    int64_t rem = B_left - sum_b;
    /* +1 to the rem largest fractional parts, ties to the lower head index */
    char taken[1024];
    memset(taken, 0, sizeof(taken));
    for (int64_t k = 0; k < rem; ++k) {
      int best = -1;
      double bf = -1.0;
      for (int a = 0; a < n_act; ++a) {
        if (taken[a]) continue;
        double f = xs[a] - floor(xs[a]);
        if (f > bf) { bf = f; best = a; }
      }
      if (best < 0) break;
      taken[best] = 1;
      b[active[best]] += 1;
    }
    int capped = 0;
    int keep[1024];
    int n_keep = 0;
    for (int a = 0; a < n_act; ++a) {
      int h = active[a];
      if (b[h] > L) {
        b[h] = (int32_t)L;
        B_left -= L;
        capped = 1;
      } else {
        keep[n_keep++] = h;
      }
    }
    if (!capped) return 0;
    for (int a = 0; a < n_keep; ++a) active[a] = keep[a];
    n_act = n_keep;
  }
}

/* S [n_layers][H]; L per sequence; b [n_seq][n_layers][H]. */
int orc_allocate(int n_seq, const int64_t* L, int n_layers, int H, int w, int budget_pct, float r,
                 const float* S, int32_t* b) {
  if (H > 1024) return 1;
  for (int s = 0; s < n_seq; ++s) {
    int64_t B = ((int64_t)budget_pct * L[s] * H) / 100;
    for (int l = 0; l < n_layers; ++l) {
      int st = alloc_layer(H, L[s], w, B, (double)r, S + (size_t)l * H, b + ((size_t)s * n_layers + l) * H);
      if (st) return st;
    }
  }
  return 0;
}

/* Variant of step 3: one allocation over every (layer, head) of a sequence   */
/* ([AudioKV] §2.1: the audio-critical heads concentrate in some layers, so a */
/* budget shared across layers can follow them).                               */
/* READINGS: the same total as the per-layer allocation,                        */
/* B = n_layers * floor(pct L H / 100), split by the same formula, rounding,    */
/* remainder and capping rule over the n_layers * H heads in (layer, head)      */
/* order (H in the formula becomes n_layers * H).                               */
int orc_allocate_global(int n_seq, const int64_t* L, int n_layers, int H, int w, int budget_pct, float r,
                        const float* S, int32_t* b) {
  const int Hg = n_layers * H;
  if (Hg > 1024) return 1;
  for (int s = 0; s < n_seq; ++s) {
    int64_t B = (int64_t)n_layers * (((int64_t)budget_pct * L[s] * H) / 100);
    int st = alloc_layer(Hg, L[s], w, B, (double)r, S, b + (size_t)s * Hg);
    if (st) return st;
  }
  return 0;
}

/* ------------------------------------------------------------------------- */
/* Step 4. Per-head selection ([AudioKV] §3.1 keeps a basic local context     */
/* window; the rest goes by smoothed score).                                   */
/* READINGS: the last w of the L positions are always kept and count toward b;*/
/* the other b - w are the largest s_hat over [0, L - w), ties to the lower    */
/* index (a full sort on (-s_hat, j)); b >= L keeps all ([C3] bypass);         */
/* output ascending.                                                            */
/* ------------------------------------------------------------------------- */
typedef struct {
  double v;
  int32_t j;
} keyed;

static int cmp_desc_then_index(const void* pa, const void* pb) {
  const keyed* a = (const keyed*)pa;
  const keyed* b = (const keyed*)pb;
  if (a->v > b->v) return -1;
  if (a->v < b->v) return 1;
  return (a->j > b->j) - (a->j < b->j);
}

static int cmp_int32(const void* pa, const void* pb) {
  int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
  return (a > b) - (a < b);
}

void orc_select_row(const double* s_hat, int64_t L, int w, int64_t b, int32_t* idx) {
  if (b >= L) {
    for (int64_t j = 0; j < L; ++j) idx[j] = (int32_t)j;
    return;
  }
  int64_t n = L - w;
  keyed* k = (keyed*)malloc(sizeof(keyed) * (size_t)(n > 0 ? n : 1));
  for (int64_t j = 0; j < n; ++j) {
    k[j].v = s_hat[j] == 0.0 ? 0.0 : s_hat[j]; /* -0 == +0 */
    k[j].j = (int32_t)j;
  }
  qsort(k, (size_t)n, sizeof(keyed), cmp_desc_then_index);
  int64_t top = b - w;
  for (int64_t i = 0; i < top; ++i) idx[i] = k[i].j;
  for (int64_t i = 0; i < w; ++i) idx[top + i] = (int32_t)(n + i);
  qsort(idx, (size_t)b, sizeof(int32_t), cmp_int32);
  free(k);
}

/* Variant of step 4: segment-wise selection ([WnW] fixed heads keep a static */
/* subset chosen per segment rather than by one top-k over the whole row, so   */
/* that no stretch of a long recording is left without cache).                 */
/* READINGS: the candidates [0, L - w) are cut into nseg segments with bounds  */
/* e_i = floor(i (L - w) / nseg); segment i keeps q_i of the b - w positions,   */
/* q_i = floor(k len_i / (L - w)) plus one for the (k - sum q) segments with    */
/* the largest remainders (k len_i mod (L - w)), ties to the lower segment; in  */
/* each segment the top-q_i by s_hat (ties to the lower index, a full sort);   */
/* the window and the b >= L bypass are as in step 4. Output ascending.        */
void orc_select_row_seg(const double* s_hat, int64_t L, int w, int64_t b, int nseg, int32_t* idx) {
  if (b >= L) {
    for (int64_t j = 0; j < L; ++j) idx[j] = (int32_t)j;
    return;
  }
  const int64_t n = L - w, k = b - w;
  int64_t* q = (int64_t*)malloc(sizeof(int64_t) * (size_t)nseg);
  int64_t* fr = (int64_t*)malloc(sizeof(int64_t) * (size_t)nseg);
  char* got = (char*)calloc((size_t)nseg, 1);
  int64_t sum_q = 0;
  for (int i = 0; i < nseg; ++i) {
    const int64_t len = (int64_t)(i + 1) * n / nseg - (int64_t)i * n / nseg;
    q[i] = k * len / n;
    fr[i] = k * len % n;
    sum_q += q[i];
  }
  for (int64_t t = 0; t < k - sum_q; ++t) { /* the largest remainders, lower segment first */
    int best = -1;
    for (int i = 0; i < nseg; ++i)
      if (!got[i] && (best < 0 || fr[i] > fr[best])) best = i;
    got[best] = 1;
    q[best] += 1;
  }
  keyed* kk = (keyed*)malloc(sizeof(keyed) * (size_t)(n > 0 ? n : 1));
  int64_t at = 0;
  for (int i = 0; i < nseg; ++i) {
    const int64_t lo = (int64_t)i * n / nseg, hi = (int64_t)(i + 1) * n / nseg;
    for (int64_t j = lo; j < hi; ++j) {
      kk[j - lo].v = s_hat[j] == 0.0 ? 0.0 : s_hat[j]; /* -0 == +0 */
      kk[j - lo].j = (int32_t)j;
    }
    qsort(kk, (size_t)(hi - lo), sizeof(keyed), cmp_desc_then_index);
    for (int64_t t = 0; t < q[i]; ++t) idx[at++] = kk[t].j;
  }
  for (int64_t i = 0; i < w; ++i) idx[at++] = (int32_t)(n + i);
  qsort(idx, (size_t)b, sizeof(int32_t), cmp_int32);
  free(kk);
  free(got);
  free(fr);
  free(q);
}

typedef struct {
  const int64_t* L;
  const int64_t* off;
  const double* s_hat;
  int w;
  const int32_t* b;
  const int64_t* idx_off;
  int32_t* idx;
  int nseg; /* 0: one top-k over the row (step 4); > 0: segment-wise */
} sel_ctx;

static void sel_task(int64_t i, void* vctx) {
  sel_ctx* c = (sel_ctx*)vctx;
  if (c->nseg > 0)
    orc_select_row_seg(c->s_hat + c->off[i], c->L[i], c->w, c->b[i], c->nseg, c->idx + c->idx_off[i]);
  else
    orc_select_row(c->s_hat + c->off[i], c->L[i], c->w, c->b[i], c->idx + c->idx_off[i]);
}

void orc_select_rows(int64_t n_rows, const int64_t* L, const int64_t* off, const double* s_hat, int w,
                     const int32_t* b, const int64_t* idx_off, int32_t* idx, int n_threads) {
  sel_ctx c = {L, off, s_hat, w, b, idx_off, idx, 0};
  orc_parallel(n_rows, n_threads, sel_task, &c);
}

void orc_select_rows_seg(int64_t n_rows, const int64_t* L, const int64_t* off, const double* s_hat, int w,
                         const int32_t* b, int nseg, const int64_t* idx_off, int32_t* idx, int n_threads) {
  sel_ctx c = {L, off, s_hat, w, b, idx_off, idx, nseg};
  orc_parallel(n_rows, n_threads, sel_task, &c);
}

/* Gather: Kc[i] = K[idx[i]] (an index copy). */
void orc_gather_row(const float* K, int d, const int32_t* idx, int64_t n, float* Kc) {
  for (int64_t i = 0; i < n; ++i) memcpy(Kc + (size_t)i * d, K + (size_t)idx[i] * d, sizeof(float) * (size_t)d);
}

/* ------------------------------------------------------------------------- */
/* Step 5. One decode step of one KV head over its kept cache ([VoxZip],       */
/* second stage):                                                               */
/*   append (k_t, v_t);  p_g = softmax(q_{t,g} K_t^T / sqrt d) over the list;   */
/*   o_g = p_g V_t;  A^(t) = gamma [A^(t-1), 0] + sum_g p_g;                     */
/*   if the list holds more than b entries:                                     */
/*     K_{t+1} = Concat(K_t[:T], K_t[I_hist], K_t[-M:]), V and A likewise,       */
/*     I_hist = the top-N middle entries by A, N = b - T - M.                    */
/* READINGS: A^(0) = 0 for the prefill entries; A is carried per entry and     */
/* cropped with the same index set as K and V; the g query heads of the group  */
/* add their softmaxes into one A; the output uses the list before eviction;   */
/* ties in A keep the lower position (the higher one is evicted).              */
/* The list is in position order. Arrays hold n entries on entry and the       */
/* caller provides room for n + 1.                                              */
/* Returns the evicted position, or -1 when nothing was evicted.                */
/* ------------------------------------------------------------------------- */
typedef struct {
  double A;
  int64_t pos;
  int64_t at; /* index in the middle part */
} mid_entry;

static int cmp_mid(const void* pa, const void* pb) {
  const mid_entry* a = (const mid_entry*)pa;
  const mid_entry* b = (const mid_entry*)pb;
  if (a->A > b->A) return -1;
  if (a->A < b->A) return 1;
  return (a->pos > b->pos) - (a->pos < b->pos);
}

int64_t orc_decode_step(int64_t* n_io, int d, int g, float* Kc, float* Vc, double* A, int64_t* pos,
                        const float* q, const float* k_new, const float* v_new, int64_t pos_new, double gamma,
                        int T, int M, int64_t b, double* o) {
  int64_t n = *n_io;
  /* append */
  memcpy(Kc + (size_t)n * d, k_new, sizeof(float) * (size_t)d);
  memcpy(Vc + (size_t)n * d, v_new, sizeof(float) * (size_t)d);
  A[n] = 0.0;
  pos[n] = pos_new;
  n += 1;
  /* attention per query head, and the decayed score update */
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  double* x = (double*)malloc(sizeof(double) * (size_t)n);
  double* padd = (double*)calloc((size_t)n, sizeof(double));
  for (int gi = 0; gi < g; ++gi) {
    const float* qg = q + (size_t)gi * d;
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += (double)qg[c] * (double)Kc[(size_t)j * d + c];
      x[j] = dot * inv_sqrt_d;
      if (x[j] > m) m = x[j];
    }
    double Z = 0.0;
    for (int64_t j = 0; j < n; ++j) {
      x[j] = exp(x[j] - m);
      Z += x[j];
    }
    double* og = o + (size_t)gi * d;
    for (int c = 0; c < d; ++c) og[c] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
      double p = x[j] / Z;
      padd[j] += p;
      for (int c = 0; c < d; ++c) og[c] += p * (double)Vc[(size_t)j * d + c];
    }
  }
  for (int64_t j = 0; j < n; ++j) A[j] = gamma * A[j] + padd[j];
  free(x);
  free(padd);

  int64_t evicted = -1;
  if (n > b) {
    /* Concat(K[:T], K[I_hist], K[-M:]): keep the first T, the last M, and the
     * top-N of the middle by A; the middle keeps its original order. */
    int64_t N = b - T - M;
    int64_t mid0 = T, mid1 = n - M; /* middle = [mid0, mid1) */
    int64_t nm = mid1 - mid0;
    mid_entry* me = (mid_entry*)malloc(sizeof(mid_entry) * (size_t)(nm > 0 ? nm : 1));
    for (int64_t i = 0; i < nm; ++i) {
      me[i].A = A[mid0 + i];
      me[i].pos = pos[mid0 + i];
      me[i].at = i;
    }
    qsort(me, (size_t)nm, sizeof(mid_entry), cmp_mid);
    char* keep = (char*)calloc((size_t)(nm > 0 ? nm : 1), 1);
    for (int64_t i = 0; i < N && i < nm; ++i) keep[me[i].at] = 1;
    int64_t wr = mid0;
    for (int64_t i = 0; i < nm; ++i) {
      int64_t src = mid0 + i;
      if (!keep[i]) {
        evicted = pos[src];
        continue;
      }
      if (wr != src) {
        memmove(Kc + (size_t)wr * d, Kc + (size_t)src * d, sizeof(float) * (size_t)d);
        memmove(Vc + (size_t)wr * d, Vc + (size_t)src * d, sizeof(float) * (size_t)d);
        A[wr] = A[src];
        pos[wr] = pos[src];
      }
      ++wr;
    }
    for (int64_t src = mid1; src < n; ++src, ++wr) {
      memmove(Kc + (size_t)wr * d, Kc + (size_t)src * d, sizeof(float) * (size_t)d);
      memmove(Vc + (size_t)wr * d, Vc + (size_t)src * d, sizeof(float) * (size_t)d);
      A[wr] = A[src];
      pos[wr] = pos[src];
    }
    n = wr;
    free(me);
    free(keep);
  }
  *n_io = n;
  return evicted;
}

/* Many steps of one head (used to time the oracle as a CPU baseline).
 * q [steps][g][d], k_new/v_new [steps][d], o [steps][g][d], evicted [steps].
 * Cache arrays need room for b + 1 entries (or n + steps without eviction). */
void orc_decode_run(int64_t* n_io, int d, int g, float* Kc, float* Vc, double* A, int64_t* pos,
                    int64_t steps, const float* q, const float* k_new, const float* v_new, int64_t pos0,
                    double gamma, int T, int M, int64_t b, double* o, int64_t* evicted) {
  for (int64_t t = 0; t < steps; ++t) {
    evicted[t] = orc_decode_step(n_io, d, g, Kc, Vc, A, pos, q + (size_t)t * g * d, k_new + (size_t)t * d,
                                 v_new + (size_t)t * d, pos0 + t, gamma, T, M, b, o + (size_t)t * g * d);
  }
}

/* Independent heads in parallel (CPU baseline). Per head h the arrays start at
 * cache_off[h] * d (Kc, Vc) / cache_off[h] (A, pos); q/k/v/o/evicted are laid
 * out [steps][heads][...]. */
typedef struct {
  int64_t* n;
  int d, g;
  float* Kc;
  float* Vc;
  double* A;
  int64_t* pos;
  const int64_t* cache_off;
  int64_t heads, steps;
  const float* q;
  const float* k_new;
  const float* v_new;
  const int64_t* pos0;
  double gamma;
  int T;
  const int32_t* M;
  const int64_t* b;
  double* o;
  int64_t* evicted;
} drun_ctx;

static void drun_task(int64_t h, void* vctx) {
  drun_ctx* c = (drun_ctx*)vctx;
  int64_t off = c->cache_off[h];
  for (int64_t t = 0; t < c->steps; ++t) {
    size_t qo = ((size_t)t * c->heads + h) * c->g * c->d;
    size_t ko = ((size_t)t * c->heads + h) * c->d;
    c->evicted[t * c->heads + h] =
        orc_decode_step(&c->n[h], c->d, c->g, c->Kc + (size_t)off * c->d, c->Vc + (size_t)off * c->d,
                        c->A + off, c->pos + off, c->q + qo, c->k_new + ko, c->v_new + ko, c->pos0[h] + t,
                        c->gamma, c->T, c->M[h], c->b[h], c->o + qo);
  }
}

void orc_decode_run_heads(int64_t heads, int64_t* n, int d, int g, float* Kc, float* Vc, double* A, int64_t* pos,
                          const int64_t* cache_off, int64_t steps, const float* q, const float* k_new,
                          const float* v_new, const int64_t* pos0, double gamma, int T, const int32_t* M,
                          const int64_t* b, double* o, int64_t* evicted, int n_threads) {
  drun_ctx c = {n, d, g, Kc, Vc, A, pos, cache_off, heads, steps, q, k_new, v_new, pos0, gamma, T, M, b, o, evicted};
  orc_parallel(heads, n_threads, drun_task, &c);
}

/* ------------------------------------------------------------------------- */
/* Next row: [VoxZip] 方法概述和架构, first stage (Semantic-Anchored Audio   */
/* Compression) on one sequence of L audio feature rows E_A [L][d]:           */
/*  1. keep the ASR segments whose confidence exceeds conf_min (0.3 on the    */
/*     page) and map their timestamps to token indices,                       */
/*     idx = floor(L * tau / tau_total);                                        */
/*  2. split the segment's tokens evenly into L_t groups (L_t = its text     */
/*     tokens), take the element-wise mean of each group and add the text    */
/*     embedding of the same position;                                        */
/*  3. keep every token that no kept segment covers as it is, and concatenate */
/*     fused groups and background tokens in time order.                      */
/* READINGS: a segment covers [idx_start, idx_end) (end exclusive), indices    */
/* clamped to [0, L]; it is kept when confidence > conf_min (compared in       */
/* float32), L_t >= 1 and idx_end > idx_start; kept segments are taken in the */
/* given order and one that starts before the end of an earlier kept segment  */
/* starts at that end instead (no token is pooled twice); a segment of len    */
/* tokens forms n = min(L_t, len) groups, group j being the tokens            */
/* [floor(j len / n), floor((j + 1) len / n)) from its start, fused with text */
/* embedding row text_row + j. Output row descriptors src[r] = (first token,  */
/* token count, text row or -1 for a background token).                       */
/* ------------------------------------------------------------------------- */
static int64_t vz_index(int64_t L, double tau, double tau_total) {
  double x = floor((double)L * tau / tau_total);
  if (x < 0.0) x = 0.0;
  if (x > (double)L) x = (double)L;
  return (int64_t)x;
}

int64_t orc_voxzip_pool(int64_t L, int d, const double* E_A, double tau_total, int64_t n_seg, const double* tau,
                        const float* conf, const int32_t* n_text, const int32_t* text_row, const double* E_T,
                        float conf_min, double* out, int32_t* src) {
  int64_t* owner = (int64_t*)malloc(sizeof(int64_t) * (size_t)(L > 0 ? L : 1));
  int64_t* seg_start = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_seg > 0 ? n_seg : 1));
  int64_t* seg_len = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_seg > 0 ? n_seg : 1));
  for (int64_t t = 0; t < L; ++t) owner[t] = -1;
  /* step 1: which tokens each kept segment covers */
  int64_t covered_to = 0;
  for (int64_t i = 0; i < n_seg; ++i) {
    seg_start[i] = 0;
    seg_len[i] = 0;
    if (!(conf[i] > conf_min) || n_text[i] < 1) continue;
    int64_t a = vz_index(L, tau[2 * i], tau_total);
    const int64_t e = vz_index(L, tau[2 * i + 1], tau_total);
    if (e <= a) continue;
    if (a < covered_to) a = covered_to;
    for (int64_t t = a; t < e; ++t) owner[t] = i;
    if (e > a) {
      seg_start[i] = a;
      seg_len[i] = e - a;
    }
    if (e > covered_to) covered_to = e;
  }
  /* steps 2 and 3: walk the sequence in time order */
  int64_t r = 0, t = 0;
  while (t < L) {
    const int64_t i = owner[t];
    if (i < 0) {
      for (int c = 0; c < d; ++c) out[(size_t)r * d + c] = E_A[(size_t)t * d + c];
      src[3 * r] = (int32_t)t;
      src[3 * r + 1] = 1;
      src[3 * r + 2] = -1;
      ++r;
      ++t;
      continue;
    }
    const int64_t len = seg_len[i];
    const int64_t n = n_text[i] < len ? n_text[i] : len;
    for (int64_t j = 0; j < n; ++j) {
      const int64_t lo = seg_start[i] + j * len / n, hi = seg_start[i] + (j + 1) * len / n;
      for (int c = 0; c < d; ++c) {
        double sum = 0.0;
        for (int64_t k = lo; k < hi; ++k) sum += E_A[(size_t)k * d + c];
        double v = sum / (double)(hi - lo);
        if (E_T) v += E_T[((size_t)text_row[i] + (size_t)j) * d + c];
        out[(size_t)r * d + c] = v;
      }
      src[3 * r] = (int32_t)lo;
      src[3 * r + 1] = (int32_t)(hi - lo);
      src[3 * r + 2] = (int32_t)(text_row[i] + j);
      ++r;
    }
    t = seg_start[i] + len;
  }
  free(seg_len);
  free(seg_start);
  free(owner);
  return r;
}

/* ------------------------------------------------------------------------- */
/* Next row: [WnW] anchor heads and tidal heads ("WnW: Waxing-and-Waning KV   */
/* Cache for Long-Form Speech LLMs", 方法概述和架构 and 细节详述): at every  */
/* decode step the anchor heads' attention over the audio positions is summed */
/* into the importance of overlapping time chunks (4 s long, 2 s apart); the  */
/* top 3 chunks are selected; a chunk leaves the GPU only after 3 steps in a  */
/* row without being selected; the tidal heads' GPU copy holds the resident   */
/* chunks, recalled from the full copy in host memory.                        */
/* READINGS: chunk m covers positions [m S, min(m S + C, L)) (C = chunk_len,  */
/* S = chunk_stride, C a multiple of S), m = 0 .. M - 1 with M = 1 when        */
/* L <= C, else ceil((L - C) / S) + 1; its score is the sum over the anchor   */
/* rows, then over its positions, of the anchors' attention mass s (float64, */
/* in that order); the top_c largest scores are selected (ties to the lower   */
/* chunk; all chunks when M <= top_c); a selected chunk's idle count becomes  */
/* 0, a resident unselected one's grows by 1 and it is released when the      */
/* count reaches release_after (-1 = not resident). Storage is kept per block */
/* [b S, min((b + 1) S, L)): a block is resident while a resident chunk holds */
/* it; blocks that stop being resident free their slots, then the new blocks, */
/* in ascending order, take the lowest free slots.                            */
/* ------------------------------------------------------------------------- */
int64_t orc_wnw_chunks(int64_t L, int64_t chunk_len, int64_t stride) {
  if (L <= chunk_len) return 1;
  return (L - chunk_len + stride - 1) / stride + 1;
}

/* One step of one sequence. idle [M], block_slot [nb], slot_block [n_slots]  */
/* are the state (updated); score [M], selected [min(top_c, M)], fetch and    */
/* release [..][2] (block, slot) and their counts are outputs. Returns 0, or  */
/* 1 when the slots run out (never when n_slots >= top_c * release_after *    */
/* chunk_len / chunk_stride).                                                 */
int orc_wnw_step(int64_t L, int n_anchor, const float* s, int chunk_len, int stride, int top_c, int release_after,
                 int n_slots, int32_t* idle, int32_t* block_slot, int32_t* slot_block, double* score,
                 int32_t* selected, int32_t* fetch, int32_t* n_fetch, int32_t* release, int32_t* n_release) {
  const int64_t M = orc_wnw_chunks(L, chunk_len, stride);
  const int64_t nb = (L + stride - 1) / stride;
  /* chunk importance */
  for (int64_t m = 0; m < M; ++m) {
    const int64_t lo = m * stride, hi = lo + chunk_len < L ? lo + chunk_len : L;
    double acc = 0.0;
    for (int a = 0; a < n_anchor; ++a)
      for (int64_t j = lo; j < hi; ++j) acc += (double)s[(size_t)a * (size_t)L + (size_t)j];
    score[m] = acc;
  }
  /* top_c selection: repeatedly the largest unselected score, lower chunk first */
  const int64_t n_sel = top_c < M ? top_c : M;
  char* chosen = (char*)calloc((size_t)(M > 0 ? M : 1), 1);
  for (int64_t k = 0; k < n_sel; ++k) {
    int64_t best = -1;
    for (int64_t m = 0; m < M; ++m)
      if (!chosen[m] && (best < 0 || score[m] > score[best])) best = m;
    chosen[best] = 1;
    selected[k] = (int32_t)best;
  }
  /* hysteresis */
  for (int64_t m = 0; m < M; ++m) {
    if (chosen[m]) {
      idle[m] = 0;
    } else if (idle[m] >= 0) {
      idle[m] += 1;
      if (idle[m] >= release_after) idle[m] = -1;
    }
  }
  /* block residency, releases, then fetches into the lowest free slots */
  const int64_t q = chunk_len / stride;
  int st = 0;
  *n_fetch = 0;
  *n_release = 0;
  char* resident = (char*)calloc((size_t)(nb > 0 ? nb : 1), 1);
  for (int64_t m = 0; m < M; ++m)
    if (idle[m] >= 0)
      for (int64_t b = m; b < m + q && b < nb; ++b) resident[b] = 1;
  for (int64_t b = 0; b < nb; ++b) {
    if (block_slot[b] >= 0 && !resident[b]) {
      release[2 * *n_release] = (int32_t)b;
      release[2 * *n_release + 1] = block_slot[b];
      ++*n_release;
      slot_block[block_slot[b]] = -1;
      block_slot[b] = -1;
    }
  }
  for (int64_t b = 0; b < nb; ++b) {
    if (resident[b] && block_slot[b] < 0) {
      int slot = -1;
      for (int k = 0; k < n_slots; ++k)
        if (slot_block[k] < 0) {
          slot = k;
          break;
        }
      if (slot < 0) {
        st = 1;
        break;
      }
      slot_block[slot] = (int32_t)b;
      block_slot[b] = slot;
      fetch[2 * *n_fetch] = (int32_t)b;
      fetch[2 * *n_fetch + 1] = slot;
      ++*n_fetch;
    }
  }
  free(resident);
  free(chosen);
  return st;
}

/* ------------------------------------------------------------------------- */
/* Next row: [C3] ("C3: Speech-Guided KV Retrieval for Long-Context SpeechLLM */
/* Inference"), the key-space index, shared-GQA competition and adaptive     */
/* resolution, per (layer, KV head) row of L audio keys K [L][d]:            */
/*  - prefill: recursive bisecting 2-means over the keys (8 iterations per    */
/*    split, seed 0); every node's centroid is the mean of its keys;          */
/*  - the active frontier starts at the cut of mean node size about 16 and    */
/*    always partitions the L positions;                                      */
/*  - step t: sigma_n = max over the G query heads of cos(q_g, c_n); clusters */
/*    in descending sigma give their keys until B are taken; exact attention  */
/*    over those keys; e_n = lambda e_n + (1 - lambda) sigma_n; R exchanges,  */
/*    each splitting the highest-e node into its children (which inherit e)   */
/*    and merging the lowest sibling pair into its parent (max of the two).   */
/* READINGS: a node with more than leaf_max (4) keys is split; the 2-means    */
/* starts from two distinct member keys picked by SplitMix64 (outputs 2n and  */
/* 2n + 1 of the generator seeded with `seed`, n = node id), assigns by       */
/* squared Euclidean distance (ties to the left child) and recomputes means  */
/* (an empty side keeps its centroid), 8 times; a split that leaves a side    */
/* empty falls back to halving the members; node ids are given breadth-first  */
/* (a split node's children get the next two ids); a node's members, in      */
/* index order, are its left child's then its right child's (a leaf's in     */
/* ascending position): centroids sum in that order, and a cluster that does  */
/* not fit the budget gives its first members in it. The initial frontier is */
/* every node at depth D0 = round(log2(L / granularity)) (the largest D with  */
/* (granularity 2^D)^2 <= 2 L^2) plus the leaves above it. Cosine with a zero */
/* vector is 0. Clusters are ranked by sigma, ties to the lower node id. e    */
/* starts at 0. An exchange picks the split node by largest e (ties to the    */
/* lower id) among frontier nodes with children, and the merge pair by        */
/* smallest max(e) (ties to the lower parent id) among sibling pairs both on  */
/* the frontier and not containing the split node; nodes created earlier in   */
/* the same step are not candidates; an exchange without both candidates is   */
/* skipped. L <= B bypasses retrieval (all keys, no update). iters >= 1.      */
/* ------------------------------------------------------------------------- */
uint64_t orc_splitmix64(uint64_t seed, uint64_t k) {
  uint64_t z = seed + (k + 1) * 0x9e3779b97f4a7c15ull;
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  return z ^ (z >> 31);
}

/* The tree: node n owns perm[lo[n] .. lo[n] + cnt[n]) (positions, index order), */
/* children left[n], left[n] + 1 (or -1), parent[n], depth[n], centroid        */
/* cent[n][d]. Arrays sized 2 L. Returns the node count.                       */
int64_t orc_c3_build(int64_t L, int d, const float* K, int leaf_max, int iters, uint64_t seed, int32_t* perm,
                     int32_t* lo, int32_t* cnt, int32_t* left, int32_t* parent, int32_t* depth, double* cent) {
  for (int64_t j = 0; j < L; ++j) perm[j] = (int32_t)j;
  int64_t n_nodes = 1;
  lo[0] = 0;
  cnt[0] = (int32_t)L;
  parent[0] = -1;
  depth[0] = 0;
  int32_t* side = (int32_t*)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
  int32_t* tmp = (int32_t*)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
  double* c = (double*)malloc(sizeof(double) * 2 * (size_t)d);
  double* acc = (double*)malloc(sizeof(double) * 2 * (size_t)d);
  for (int64_t nd = 0; nd < n_nodes; ++nd) { /* breadth first: children are appended */
    left[nd] = -1;
    const int32_t n = cnt[nd];
    const int32_t* m = perm + lo[nd];
    if (n <= leaf_max || n < 2) continue;
    const int64_t i0 = (int64_t)(orc_splitmix64(seed, 2 * (uint64_t)nd) % (uint64_t)n);
    const int64_t i1 = (i0 + 1 + (int64_t)(orc_splitmix64(seed, 2 * (uint64_t)nd + 1) % (uint64_t)(n - 1))) % n;
    for (int k = 0; k < d; ++k) {
      c[k] = K[(size_t)m[i0] * d + k];
      c[d + k] = K[(size_t)m[i1] * d + k];
    }
    for (int it = 0; it < iters; ++it) {
      int64_t n1 = 0;
      for (int32_t j = 0; j < n; ++j) {
        double d0 = 0.0, d1 = 0.0;
        for (int k = 0; k < d; ++k) {
          const double x = K[(size_t)m[j] * d + k];
          d0 += (x - c[k]) * (x - c[k]);
          d1 += (x - c[d + k]) * (x - c[d + k]);
        }
        side[j] = d1 < d0 ? 1 : 0;
        n1 += side[j];
      }
      for (int k = 0; k < 2 * d; ++k) acc[k] = 0.0;
      for (int32_t j = 0; j < n; ++j)
        for (int k = 0; k < d; ++k) acc[side[j] * d + k] += K[(size_t)m[j] * d + k];
      if (n - n1 > 0)
        for (int k = 0; k < d; ++k) c[k] = acc[k] / (double)(n - n1);
      if (n1 > 0)
        for (int k = 0; k < d; ++k) c[d + k] = acc[d + k] / (double)n1;
    }
    int32_t n0 = 0;
    for (int32_t j = 0; j < n; ++j) n0 += side[j] == 0;
    if (n0 == 0 || n0 == n) { /* fall back to halving in position order */
      n0 = (n + 1) / 2;
      for (int32_t j = 0; j < n; ++j) side[j] = j >= n0;
    }
    int32_t a = 0, b = n0;
    for (int32_t j = 0; j < n; ++j) tmp[side[j] ? b++ : a++] = m[j];
    memcpy(perm + lo[nd], tmp, sizeof(int32_t) * (size_t)n);
    const int64_t l = n_nodes, r = n_nodes + 1;
    left[nd] = (int32_t)l;
    lo[l] = lo[nd];
    cnt[l] = n0;
    lo[r] = lo[nd] + n0;
    cnt[r] = n - n0;
    parent[l] = parent[r] = (int32_t)nd;
    depth[l] = depth[r] = depth[nd] + 1;
    n_nodes += 2;
  }
  /* centroids: the mean of every node's keys, summed in index order */
  for (int64_t nd = 0; nd < n_nodes; ++nd) {
    for (int k = 0; k < d; ++k) {
      double s = 0.0;
      for (int32_t j = 0; j < cnt[nd]; ++j) s += K[(size_t)perm[lo[nd] + j] * d + k];
      cent[(size_t)nd * d + k] = s / (double)cnt[nd];
    }
  }
  free(acc);
  free(c);
  free(tmp);
  free(side);
  return n_nodes;
}

/* The initial frontier (node ids, ascending) into front; returns its size. */
int64_t orc_c3_frontier(int64_t n_nodes, int64_t L, int granularity, const int32_t* left, const int32_t* depth,
                        int32_t* front) {
  int D0 = 0; /* the cut whose mean node size is nearest granularity (log scale) */
  while (D0 < 40) {
    const double next = (double)granularity * (double)((int64_t)1 << (D0 + 1));
    if (next * next > 2.0 * (double)L * (double)L) break;
    ++D0;
  }
  int64_t A = 0;
  for (int64_t nd = 0; nd < n_nodes; ++nd)
    if (depth[nd] == D0 || (depth[nd] < D0 && left[nd] < 0)) front[A++] = (int32_t)nd;
  return A;
}

static double cosine(const double* a, const double* b, int d) {
  double ab = 0.0, aa = 0.0, bb = 0.0;
  for (int k = 0; k < d; ++k) {
    ab += a[k] * b[k];
    aa += a[k] * a[k];
    bb += b[k] * b[k];
  }
  if (aa == 0.0 || bb == 0.0) return 0.0;
  return ab / (sqrt(aa) * sqrt(bb));
}

/* One decode step of one row. front [A] and e [n_nodes] are updated.        */
/* sigma [A] (scores of the frontier at entry, in its order), sel [min(B, L)] */
/* (positions, ascending) and o [G][d] are outputs. Returns the number of     */
/* selected positions.                                                        */
int64_t orc_c3_step(int64_t L, int d, int G, const float* K, const float* V, const float* q, int64_t n_nodes,
                    const int32_t* perm, const int32_t* lo, const int32_t* cnt, const int32_t* left,
                    const double* cent, int64_t A, int32_t* front, double* e, int64_t B,
                    double lambda, int R, double* sigma, int32_t* sel, double* o) {
  int64_t n_sel = 0;
  char* taken = (char*)calloc((size_t)(L > 0 ? L : 1), 1);
  const int bypass = L <= B;
  if (bypass) {
    for (int64_t j = 0; j < L; ++j) taken[j] = 1;
  } else {
    double* qv = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t i = 0; i < A; ++i) {
      double best = -INFINITY;
      for (int g = 0; g < G; ++g) {
        for (int k = 0; k < d; ++k) qv[k] = q[(size_t)g * d + k];
        const double cs = cosine(qv, cent + (size_t)front[i] * d, d);
        if (cs > best) best = cs;
      }
      sigma[i] = best;
    }
    free(qv);
    /* clusters in descending sigma (ties: lower node id) give their keys */
    char* used = (char*)calloc((size_t)(A > 0 ? A : 1), 1);
    int64_t got = 0;
    while (got < B) {
      int64_t bi = -1;
      for (int64_t i = 0; i < A; ++i)
        if (!used[i] && (bi < 0 || sigma[i] > sigma[bi] || (sigma[i] == sigma[bi] && front[i] < front[bi]))) bi = i;
      if (bi < 0) break;
      used[bi] = 1;
      const int32_t nd = front[bi];
      /* a cluster that does not fit gives its first members in index order */
      for (int32_t j = 0; j < cnt[nd] && got < B; ++j, ++got) taken[perm[lo[nd] + j]] = 1;
    }
    free(used);
  }
  for (int64_t j = 0; j < L; ++j)
    if (taken[j]) sel[n_sel++] = (int32_t)j;
  /* exact attention over the selected keys */
  const double scale = 1.0 / sqrt((double)d);
  double* lg = (double*)malloc(sizeof(double) * (size_t)(n_sel > 0 ? n_sel : 1));
  for (int g = 0; g < G; ++g) {
    double mx = -INFINITY;
    for (int64_t i = 0; i < n_sel; ++i) {
      double dot = 0.0;
      for (int k = 0; k < d; ++k) dot += (double)q[(size_t)g * d + k] * (double)K[(size_t)sel[i] * d + k];
      lg[i] = dot * scale;
      if (lg[i] > mx) mx = lg[i];
    }
    double den = 0.0;
    for (int64_t i = 0; i < n_sel; ++i) den += exp(lg[i] - mx);
    for (int k = 0; k < d; ++k) {
      double acc = 0.0;
      for (int64_t i = 0; i < n_sel; ++i) acc += exp(lg[i] - mx) / den * (double)V[(size_t)sel[i] * d + k];
      o[(size_t)g * d + k] = acc;
    }
  }
  free(lg);
  free(taken);
  if (bypass) return n_sel;
  /* relevance EMA of the frontier */
  for (int64_t i = 0; i < A; ++i) e[front[i]] = lambda * e[front[i]] + (1.0 - lambda) * sigma[i];
  /* R exchanges: split the most relevant node, merge the least relevant sibling pair */
  char* on = (char*)calloc((size_t)n_nodes, 1);
  char* fresh = (char*)calloc((size_t)n_nodes, 1);
  for (int64_t i = 0; i < A; ++i) on[front[i]] = 1;
  for (int r = 0; r < R; ++r) {
    int64_t s = -1;
    for (int64_t nd = 0; nd < n_nodes; ++nd)
      if (on[nd] && !fresh[nd] && left[nd] >= 0 && (s < 0 || e[nd] > e[s])) s = nd;
    if (s < 0) break;
    int64_t p = -1;
    double pv = 0.0;
    for (int64_t nd = 0; nd < n_nodes; ++nd) {
      if (left[nd] < 0) continue;
      const int64_t a = left[nd], b = left[nd] + 1;
      if (!on[a] || !on[b] || fresh[a] || fresh[b] || a == s || b == s) continue;
      const double v = e[a] > e[b] ? e[a] : e[b];
      if (p < 0 || v < pv) {
        p = nd;
        pv = v;
      }
    }
    if (p < 0) break;
    const int64_t c0 = left[s];
    on[s] = 0;
    on[c0] = on[c0 + 1] = 1;
    fresh[c0] = fresh[c0 + 1] = 1;
    e[c0] = e[c0 + 1] = e[s];
    on[left[p]] = on[left[p] + 1] = 0;
    on[p] = 1;
    fresh[p] = 1;
    e[p] = pv;
  }
  int64_t a = 0;
  for (int64_t nd = 0; nd < n_nodes; ++nd)
    if (on[nd]) front[a++] = (int32_t)nd;
  free(fresh);
  free(on);
  return n_sel;
}
