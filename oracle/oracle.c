/*
 * oracle.c - plain fp64 CPU reference ("oracle") for exact attention forward.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library. The CUDA product path
 * never links, loads or calls it, and this file shares no code, header, table
 * or helper with the CUDA path.
 *
 * What it computes is the three-step definition of attention given in
 * "A Deep Dive into Flash Attention" (section "Key-Value Attention: The
 * Backbone of Transformers"): score every query against every key, turn the
 * scores into probabilities with a softmax, and take the probability-weighted
 * sum of the value rows. Each score row is materialised in full, in double
 * precision, from the bf16 inputs widened exactly; there is no tiling and no
 * online rescaling. The masks and score modifiers are the FlexAttention hooks
 * ("FlexAttention + FlashAttention-4" talk; attention-gym issue 101 repro:
 * causal mask_mod q_idx >= kv_idx, score_mod(score, b, h, q_idx, kv_idx)), the
 * window / ALiBi / softcap options of flash_attn_func (FlashAttention overview,
 * "Examples"), and GQA follows the repeat_kv head map (transformers issue
 * 36218): KV head j serves query heads j*g .. j*g+g-1, g = Hq / Hkv.
 *
 * Readings where the pages are silent (all stated here and in the design notes):
 *   - the score modifier receives the scaled score: s = mod(scale * q.k);
 *   - softcap: s -> c * tanh(s / c);
 *   - ALiBi: s -> s + slope[b][h] * (kv_pos - q_pos);
 *   - LSE is the natural log-sum-exp of the modified scores over allowed keys;
 *   - a row with no allowed key has O = 0 and LSE = -inf;
 *   - query i sits at position i + q_offset for the causal / window masks;
 *   - window (left, right), -1 = unbounded: allowed iff
 *       q_pos - kv <= left and kv - q_pos <= right;
 *   - document mask: allowed iff doc[q] == doc[kv] and kv <= q;
 *   - ReLU activation wrapper (the talk's example of undoing the softmax
 *     normalisation and applying a pointwise activation instead):
 *     O = sum over allowed keys of max(scale * q.k, 0) * v, unnormalised,
 *     and the LSE slot holds ln of the summed weights (-inf when they sum
 *     to 0 or no key is allowed).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { O_MASK_NONE = 0, O_MASK_CAUSAL = 1, O_MASK_WINDOW = 2, O_MASK_DOCUMENT = 3 };
enum { O_MOD_NONE = 0, O_MOD_SOFTCAP = 1, O_MOD_ALIBI = 2, O_MOD_RELU = 3 };

static double widen_bf16(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ------------------------------------------------------------ prefill */

typedef struct {
  const uint16_t *q, *k, *v;         /* bf16 bit patterns, last dim contiguous */
  int64_t q_sb, q_ss, q_sh;          /* element strides: batch, sequence, head */
  int64_t k_sb, k_ss, k_sh;
  int64_t v_sb, v_ss, v_sh;
  int B, Hq, Hkv, Sq, Skv, D;
  double scale;
  int mask, window_left, window_right, q_offset;
  const int32_t *doc_id;             /* document mask only: row b ([Sq] == [Skv]) at doc_id + b * doc_bstride */
  int64_t doc_bstride;               /* 0: one row shared by every batch */
  int mod;
  double softcap;
  const float *alibi;                /* alibi[b * alibi_bstride + h] */
  int64_t alibi_bstride;
  int kv_begin, kv_end;              /* keys restricted to [kv_begin, kv_end) */
} oracle_attn_args;

static int mask_allows(int mask, int wl, int wr, int64_t q_pos, int64_t kv, const int32_t *doc, int64_t qi) {
  switch (mask) {
    case O_MASK_NONE:
      return 1;
    case O_MASK_CAUSAL:
      return kv <= q_pos;
    case O_MASK_WINDOW:
      return (wl < 0 || q_pos - kv <= wl) && (wr < 0 || kv - q_pos <= wr);
    case O_MASK_DOCUMENT:
      return kv <= q_pos && doc[qi] == doc[kv];
    default:
      return 0;
  }
}

static double apply_mod(const oracle_attn_args *a, double s, int b, int h, int64_t q_pos, int64_t kv) {
  if (a->mod == O_MOD_SOFTCAP) return a->softcap * tanh(s / a->softcap);
  if (a->mod == O_MOD_ALIBI) return s + (double)a->alibi[b * a->alibi_bstride + h] * (double)(kv - q_pos);
  return s;
}

/* One output row: O[b, i, h, :] and LSE[b, h, i]. s is scratch of Skv doubles. */
static void attn_row(const oracle_attn_args *a, int b, int h, int i, double *o, double *lse, double *s) {
  const int g = a->Hq / a->Hkv;
  const int hk = h / g;
  const int64_t q_pos = (int64_t)i + a->q_offset;
  const uint16_t *qr = a->q + b * a->q_sb + (int64_t)i * a->q_ss + (int64_t)h * a->q_sh;
  /* the mask_mod sees the batch index: batch b has its own document row */
  const int32_t *doc = a->doc_id ? a->doc_id + (int64_t)b * a->doc_bstride : NULL;
  double m = -INFINITY;
  int any = 0;
  for (int j = a->kv_begin; j < a->kv_end; ++j) {
    if (!mask_allows(a->mask, a->window_left, a->window_right, q_pos, j, doc, i)) {
      s[j] = -INFINITY;
      continue;
    }
    const uint16_t *kr = a->k + b * a->k_sb + (int64_t)j * a->k_ss + (int64_t)hk * a->k_sh;
    double dot = 0.0;
    for (int d = 0; d < a->D; ++d) dot += widen_bf16(qr[d]) * widen_bf16(kr[d]);
    s[j] = apply_mod(a, a->scale * dot, b, h, q_pos, j);
    if (s[j] > m) m = s[j];
    any = 1;
  }
  for (int d = 0; d < a->D; ++d) o[d] = 0.0;
  if (!any) {
    *lse = -INFINITY;
    return;
  }
  if (a->mod == O_MOD_RELU) {
    double w = 0.0;
    for (int j = a->kv_begin; j < a->kv_end; ++j) {
      if (s[j] == -INFINITY || !(s[j] > 0.0)) continue;
      w += s[j];
      const uint16_t *vr = a->v + b * a->v_sb + (int64_t)j * a->v_ss + (int64_t)hk * a->v_sh;
      for (int d = 0; d < a->D; ++d) o[d] += s[j] * widen_bf16(vr[d]);
    }
    *lse = w > 0.0 ? log(w) : -INFINITY;
    return;
  }
  double l = 0.0;
  for (int j = a->kv_begin; j < a->kv_end; ++j) {
    if (s[j] == -INFINITY) continue;
    const double p = exp(s[j] - m);
    l += p;
    const uint16_t *vr = a->v + b * a->v_sb + (int64_t)j * a->v_ss + (int64_t)hk * a->v_sh;
    for (int d = 0; d < a->D; ++d) o[d] += p * widen_bf16(vr[d]);
  }
  for (int d = 0; d < a->D; ++d) o[d] /= l;
  *lse = m + log(l);
}

typedef struct {
  const oracle_attn_args *a;
  const int32_t *rows; /* nrows x (b, h, i) or NULL: all rows in (b, h, i) order */
  int64_t r0, r1;
  double *o, *lse;
} attn_job;

static void *attn_worker(void *p) {
  attn_job *job = (attn_job *)p;
  const oracle_attn_args *a = job->a;
  double *s = (double *)malloc(sizeof(double) * (size_t)(a->Skv > 0 ? a->Skv : 1));
  for (int64_t r = job->r0; r < job->r1; ++r) {
    int b, h, i;
    if (job->rows) {
      b = job->rows[3 * r];
      h = job->rows[3 * r + 1];
      i = job->rows[3 * r + 2];
    } else {
      i = (int)(r % a->Sq);
      h = (int)((r / a->Sq) % a->Hq);
      b = (int)(r / ((int64_t)a->Sq * a->Hq));
    }
    attn_row(a, b, h, i, job->o + r * a->D, job->lse + r, s);
  }
  free(s);
  return NULL;
}

static void run_jobs(void *(*fn)(void *), void *jobs, size_t job_size, int n) {
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n);
  for (int t = 0; t < n; ++t) pthread_create(&th[t], NULL, fn, (char *)jobs + job_size * (size_t)t);
  for (int t = 0; t < n; ++t) pthread_join(th[t], NULL);
  free(th);
}

/* Returns 0 on success, -1 on bad arguments. */
int oracle_attn(const oracle_attn_args *a, const int32_t *rows, int64_t nrows, double *o, double *lse, int nthreads) {
  if (a->Hkv <= 0 || a->Hq % a->Hkv != 0 || a->D <= 0) return -1;
  if (a->kv_begin < 0 || a->kv_end > a->Skv || a->kv_begin > a->kv_end) return -1;
  if (a->mask == O_MASK_DOCUMENT && (a->doc_id == NULL || a->Sq != a->Skv || a->q_offset != 0)) return -1;
  if (a->mod == O_MOD_ALIBI && a->alibi == NULL) return -1;
  if (a->mod == O_MOD_SOFTCAP && !(a->softcap > 0.0)) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nrows < nthreads) nthreads = nrows > 0 ? (int)nrows : 1;
  attn_job *jobs = (attn_job *)malloc(sizeof(attn_job) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].a = a;
    jobs[t].rows = rows;
    jobs[t].r0 = nrows * t / nthreads;
    jobs[t].r1 = nrows * (t + 1) / nthreads;
    jobs[t].o = o;
    jobs[t].lse = lse;
  }
  run_jobs(attn_worker, jobs, sizeof(attn_job), nthreads);
  free(jobs);
  return 0;
}

/* ------------------------------------------------------------ LSE combine */

/* Merge partial results computed over disjoint key sets: the combined LSE is
 * ln(sum_i exp(lse_i)) and the combined output is the exp(lse_i - lse)-weighted
 * sum of the partial outputs (the "combine the results" step of the online
 * softmax in "A Deep Dive into Flash Attention", section "2. Online Softmax").
 * The largest lse_i is factored out of the sum; that changes no value.
 */
void oracle_lse_combine(int n, const double *lse_parts, const double *o_parts, int D, double *o, double *lse) {
  double mx = -INFINITY;
  for (int i = 0; i < n; ++i)
    if (lse_parts[i] > mx) mx = lse_parts[i];
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (mx == -INFINITY) {
    *lse = -INFINITY;
    return;
  }
  double sum = 0.0;
  for (int i = 0; i < n; ++i) sum += exp(lse_parts[i] - mx);
  *lse = mx + log(sum);
  for (int i = 0; i < n; ++i) {
    if (lse_parts[i] == -INFINITY) continue;
    const double w = exp(lse_parts[i] - *lse);
    for (int d = 0; d < D; ++d) o[d] += w * o_parts[(int64_t)i * D + d];
  }
}

/* ------------------------------------------------------------ paged decode */

typedef struct {
  const uint16_t *q;                 /* [B][Hq][D] with strides */
  int64_t q_sb, q_sh;
  const uint16_t *k_cache, *v_cache; /* [num_pages][page_size][Hkv][D] with strides */
  int64_t c_sp, c_ss, c_sh;
  const int32_t *block_table;        /* [B][bt_stride] logical page -> physical page */
  int64_t bt_stride;
  const int32_t *seqlens;            /* [B] */
  int B, Hq, Hkv, D, page_size, num_pages;
  double scale;
  int mod;
  double softcap;
  const float *alibi;
  int64_t alibi_bstride;
} oracle_decode_args;

typedef struct {
  const oracle_decode_args *a;
  int64_t r0, r1;
  double *o, *lse;
  int err;
} decode_job;

/* Key t of sequence b lives in physical page block_table[b][t / page_size] at
 * slot t % page_size (flash_attn_with_kvcache with block_table, FlashAttention
 * overview, "Examples"). The single query sits at position seqlen - 1. */
static void *decode_worker(void *p) {
  decode_job *job = (decode_job *)p;
  const oracle_decode_args *a = job->a;
  const int g = a->Hq / a->Hkv;
  for (int64_t r = job->r0; r < job->r1; ++r) {
    const int b = (int)(r / a->Hq), h = (int)(r % a->Hq), hk = h / g;
    const int n = a->seqlens[b];
    const uint16_t *qr = a->q + b * a->q_sb + (int64_t)h * a->q_sh;
    double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double *o = job->o + r * a->D;
    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
      const int page = a->block_table[b * a->bt_stride + t / a->page_size];
      if (page < 0 || page >= a->num_pages) {
        job->err = 1;
        s[t] = -INFINITY;
        continue;
      }
      const uint16_t *kr = a->k_cache + page * a->c_sp + (int64_t)(t % a->page_size) * a->c_ss + (int64_t)hk * a->c_sh;
      double dot = 0.0;
      for (int d = 0; d < a->D; ++d) dot += widen_bf16(qr[d]) * widen_bf16(kr[d]);
      double sc = a->scale * dot;
      if (a->mod == O_MOD_SOFTCAP) sc = a->softcap * tanh(sc / a->softcap);
      if (a->mod == O_MOD_ALIBI) sc += (double)a->alibi[b * a->alibi_bstride + h] * (double)(t - (n - 1));
      s[t] = sc;
      if (sc > m) m = sc;
    }
    for (int d = 0; d < a->D; ++d) o[d] = 0.0;
    if (m == -INFINITY) {
      job->lse[r] = -INFINITY;
      free(s);
      continue;
    }
    double l = 0.0;
    for (int t = 0; t < n; ++t) {
      if (s[t] == -INFINITY) continue;
      const double pr = exp(s[t] - m);
      l += pr;
      const int page = a->block_table[b * a->bt_stride + t / a->page_size];
      const uint16_t *vr = a->v_cache + page * a->c_sp + (int64_t)(t % a->page_size) * a->c_ss + (int64_t)hk * a->c_sh;
      for (int d = 0; d < a->D; ++d) o[d] += pr * widen_bf16(vr[d]);
    }
    for (int d = 0; d < a->D; ++d) o[d] /= l;
    job->lse[r] = m + log(l);
    free(s);
  }
  return NULL;
}

/* o: [B][Hq][D], lse: [B][Hq]. Returns 0, or -1 on bad arguments / page ids. */
int oracle_decode(const oracle_decode_args *a, double *o, double *lse, int nthreads) {
  if (a->Hkv <= 0 || a->Hq % a->Hkv != 0 || a->page_size <= 0) return -1;
  if (a->mod == O_MOD_ALIBI && a->alibi == NULL) return -1;
  if (a->mod == O_MOD_SOFTCAP && !(a->softcap > 0.0)) return -1;
  const int64_t nrows = (int64_t)a->B * a->Hq;
  if (nthreads < 1) nthreads = 1;
  if (nrows < nthreads) nthreads = nrows > 0 ? (int)nrows : 1;
  decode_job *jobs = (decode_job *)malloc(sizeof(decode_job) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].a = a;
    jobs[t].r0 = nrows * t / nthreads;
    jobs[t].r1 = nrows * (t + 1) / nthreads;
    jobs[t].o = o;
    jobs[t].lse = lse;
    jobs[t].err = 0;
  }
  run_jobs(decode_worker, jobs, sizeof(decode_job), nthreads);
  int err = 0;
  for (int t = 0; t < nthreads; ++t) err |= jobs[t].err;
  free(jobs);
  return err ? -1 : 0;
}

/* ------------------------------------------------------------ block mask */

/* FlexAttention block mask (create_block_mask with BLOCK_SIZE (blk_q, blk_kv),
 * attention-gym issue 101; block-sparse tiles in the FA4 talk): each
 * (q-tile, kv-tile) is empty (0) when no in-range pair is allowed, full (2)
 * when every in-range pair is allowed, partial (1) otherwise. Per q-tile the
 * partial and full kv-tile indices are listed in ascending order. Decided by
 * evaluating the mask on every in-range pair of the tile.
 * cls: [nQ][nK]; *_cnt: [nQ]; *_idx: [nQ][nK] (unused tail left untouched). */
int oracle_block_mask(int mask, int window_left, int window_right, int q_offset, const int32_t *doc_id, int Sq,
                      int Skv, int blk_q, int blk_kv, uint8_t *cls, int32_t *part_cnt, int32_t *part_idx,
                      int32_t *full_cnt, int32_t *full_idx) {
  if (blk_q <= 0 || blk_kv <= 0 || Sq < 0 || Skv < 0) return -1;
  if (mask == O_MASK_DOCUMENT && (doc_id == NULL || Sq != Skv || q_offset != 0)) return -1;
  const int nQ = (Sq + blk_q - 1) / blk_q, nK = (Skv + blk_kv - 1) / blk_kv;
  for (int qt = 0; qt < nQ; ++qt) {
    int np = 0, nf = 0;
    for (int kt = 0; kt < nK; ++kt) {
      int64_t allowed = 0, total = 0;
      for (int i = qt * blk_q; i < (qt + 1) * blk_q && i < Sq; ++i)
        for (int j = kt * blk_kv; j < (kt + 1) * blk_kv && j < Skv; ++j) {
          ++total;
          allowed += mask_allows(mask, window_left, window_right, (int64_t)i + q_offset, j, doc_id, i);
        }
      const uint8_t c = allowed == 0 ? 0 : (allowed == total ? 2 : 1);
      cls[(int64_t)qt * nK + kt] = c;
      if (c == 1) part_idx[(int64_t)qt * nK + np++] = kt;
      if (c == 2) full_idx[(int64_t)qt * nK + nf++] = kt;
    }
    part_cnt[qt] = np;
    full_cnt[qt] = nf;
  }
  return 0;
}

/* Number of allowed (q, kv) pairs for one (b, h): used for FLOP accounting. */
int64_t oracle_count_pairs(int mask, int window_left, int window_right, int q_offset, const int32_t *doc_id, int Sq,
                           int Skv) {
  int64_t n = 0;
  for (int i = 0; i < Sq; ++i)
    for (int j = 0; j < Skv; ++j) n += mask_allows(mask, window_left, window_right, (int64_t)i + q_offset, j, doc_id, i);
  return n;
}

/* ------------------------------------------------------------ fp64-input forward and backward */

/* The same attention in double precision on double inputs (no bf16 step):
 * the forward exists so that the backward can be checked against central
 * finite differences of it. Layouts as in oracle_attn_args (element strides
 * of batch, sequence, head; last dimension contiguous). */
typedef struct {
  const double *q, *k, *v, *dout;    /* dout: upstream gradient dL/dO, laid out like q */
  int64_t q_sb, q_ss, q_sh;
  int64_t k_sb, k_ss, k_sh;
  int64_t v_sb, v_ss, v_sh;
  int B, Hq, Hkv, Sq, Skv, D;
  double scale;
  int mask, window_left, window_right, q_offset;
  const int32_t *doc_id;
  int64_t doc_bstride;
  int mod;
  double softcap;
  const float *alibi;
  int64_t alibi_bstride;
} oracle_f64_args;

static double f64_score(const oracle_f64_args *a, int b, int h, int i, int j, double *dmod) {
  /* z = scale * q.k; s = mod(z); *dmod = ds/dz */
  const int g = a->Hq / a->Hkv, hk = h / g;
  const double *qr = a->q + b * a->q_sb + (int64_t)i * a->q_ss + (int64_t)h * a->q_sh;
  const double *kr = a->k + b * a->k_sb + (int64_t)j * a->k_ss + (int64_t)hk * a->k_sh;
  double dot = 0.0;
  for (int d = 0; d < a->D; ++d) dot += qr[d] * kr[d];
  const double z = a->scale * dot;
  if (a->mod == O_MOD_SOFTCAP) {
    const double t = tanh(z / a->softcap);
    *dmod = 1.0 - t * t;
    return a->softcap * t;
  }
  *dmod = 1.0;
  if (a->mod == O_MOD_ALIBI) {
    const int64_t q_pos = (int64_t)i + a->q_offset;
    return z + (double)a->alibi[b * a->alibi_bstride + h] * (double)(j - q_pos);
  }
  return z;
}

static int f64_allowed(const oracle_f64_args *a, int b, int i, int j) {
  const int32_t *doc = a->doc_id ? a->doc_id + (int64_t)b * a->doc_bstride : NULL;
  return mask_allows(a->mask, a->window_left, a->window_right, (int64_t)i + a->q_offset, j, doc, i);
}

/* Row (b, h, i): p[j] = softmax probabilities (0 where masked), returns LSE
 * (-inf for a row with no allowed key, then p = 0). */
static double f64_row_probs(const oracle_f64_args *a, int b, int h, int i, double *p, double *dm) {
  double m = -INFINITY;
  for (int j = 0; j < a->Skv; ++j) {
    if (!f64_allowed(a, b, i, j)) {
      p[j] = -INFINITY;
      continue;
    }
    p[j] = f64_score(a, b, h, i, j, &dm[j]);
    if (p[j] > m) m = p[j];
  }
  if (m == -INFINITY) {
    for (int j = 0; j < a->Skv; ++j) p[j] = 0.0;
    return -INFINITY;
  }
  double l = 0.0;
  for (int j = 0; j < a->Skv; ++j) {
    p[j] = p[j] == -INFINITY ? 0.0 : exp(p[j] - m);
    l += p[j];
  }
  for (int j = 0; j < a->Skv; ++j) p[j] /= l;
  return m + log(l);
}

/* o: [B][Sq][Hq][D] contiguous, lse: [B][Hq][Sq]. Returns 0 or -1. */
int oracle_attn_f64(const oracle_f64_args *a, double *o, double *lse) {
  if (a->Hkv <= 0 || a->Hq % a->Hkv != 0 || a->D <= 0) return -1;
  double *p = (double *)malloc(sizeof(double) * (size_t)(a->Skv > 0 ? a->Skv : 1));
  double *dm = (double *)malloc(sizeof(double) * (size_t)(a->Skv > 0 ? a->Skv : 1));
  const int g = a->Hq / a->Hkv;
  for (int b = 0; b < a->B; ++b)
    for (int h = 0; h < a->Hq; ++h)
      for (int i = 0; i < a->Sq; ++i) {
        const double L = f64_row_probs(a, b, h, i, p, dm);
        lse[((int64_t)b * a->Hq + h) * a->Sq + i] = L;
        double *orow = o + (((int64_t)b * a->Sq + i) * a->Hq + h) * a->D;
        for (int d = 0; d < a->D; ++d) orow[d] = 0.0;
        for (int j = 0; j < a->Skv; ++j) {
          if (p[j] == 0.0) continue;
          const double *vr = a->v + b * a->v_sb + (int64_t)j * a->v_ss + (int64_t)(h / g) * a->v_sh;
          for (int d = 0; d < a->D; ++d) orow[d] += p[j] * vr[d];
        }
      }
  free(p);
  free(dm);
  return 0;
}

/* Backward of the forward above by the chain rule (FlashAttention overview,
 * "Examples": the backward pass and its deterministic option): with
 * p = softmax row, dp_ij = dO_i . v_j, ds_ij = p_ij (dp_ij - sum_j' p_ij' dp_ij'),
 * dz_ij = ds_ij * mod'(z_ij),
 *   dV_j += p_ij dO_i,  dQ_i = scale sum_j dz_ij k_j,  dK_j += scale dz_ij q_i,
 * summed over every query head of a KV head's group (GQA) and every row.
 * One thread per (batch, KV head) owns that head's dK / dV rows.
 * dq: [B][Sq][Hq][D], dk / dv: [B][Skv][Hkv][D], all contiguous. */
typedef struct {
  const oracle_f64_args *a;
  int bh0, bh1;
  double *dq, *dk, *dv;
} bwd_job;

static void *bwd_worker(void *ptr) {
  bwd_job *job = (bwd_job *)ptr;
  const oracle_f64_args *a = job->a;
  const int g = a->Hq / a->Hkv;
  const size_t n = (size_t)(a->Skv > 0 ? a->Skv : 1);
  double *p = (double *)malloc(sizeof(double) * n);
  double *dm = (double *)malloc(sizeof(double) * n);
  double *dp = (double *)malloc(sizeof(double) * n);
  for (int bh = job->bh0; bh < job->bh1; ++bh) {
    const int b = bh / a->Hkv, hk = bh % a->Hkv;
    for (int h = hk * g; h < hk * g + g; ++h)
      for (int i = 0; i < a->Sq; ++i) {
        const double L = f64_row_probs(a, b, h, i, p, dm);
        double *dqr = job->dq + (((int64_t)b * a->Sq + i) * a->Hq + h) * a->D;
        for (int d = 0; d < a->D; ++d) dqr[d] = 0.0;
        if (L == -INFINITY) continue;
        const double *dor = a->dout + b * a->q_sb + (int64_t)i * a->q_ss + (int64_t)h * a->q_sh;
        const double *qr = a->q + b * a->q_sb + (int64_t)i * a->q_ss + (int64_t)h * a->q_sh;
        double Di = 0.0;
        for (int j = 0; j < a->Skv; ++j) {
          dp[j] = 0.0;
          if (p[j] == 0.0) continue;
          const double *vr = a->v + b * a->v_sb + (int64_t)j * a->v_ss + (int64_t)hk * a->v_sh;
          for (int d = 0; d < a->D; ++d) dp[j] += dor[d] * vr[d];
          Di += p[j] * dp[j];
        }
        for (int j = 0; j < a->Skv; ++j) {
          if (p[j] == 0.0) continue;
          const double dz = p[j] * (dp[j] - Di) * dm[j];
          const double *kr = a->k + b * a->k_sb + (int64_t)j * a->k_ss + (int64_t)hk * a->k_sh;
          double *dkr = job->dk + (((int64_t)b * a->Skv + j) * a->Hkv + hk) * a->D;
          double *dvr = job->dv + (((int64_t)b * a->Skv + j) * a->Hkv + hk) * a->D;
          for (int d = 0; d < a->D; ++d) {
            dqr[d] += a->scale * dz * kr[d];
            dkr[d] += a->scale * dz * qr[d];
            dvr[d] += p[j] * dor[d];
          }
        }
      }
  }
  free(p);
  free(dm);
  free(dp);
  return NULL;
}

int oracle_attn_bwd_f64(const oracle_f64_args *a, double *dq, double *dk, double *dv, int nthreads) {
  if (a->Hkv <= 0 || a->Hq % a->Hkv != 0 || a->D <= 0 || a->dout == NULL) return -1;
  if (a->mask == O_MASK_DOCUMENT && (a->doc_id == NULL || a->Sq != a->Skv || a->q_offset != 0)) return -1;
  if (a->mod == O_MOD_ALIBI && a->alibi == NULL) return -1;
  if (a->mod == O_MOD_SOFTCAP && !(a->softcap > 0.0)) return -1;
  const size_t nkv = (size_t)a->B * a->Skv * a->Hkv * a->D;
  for (size_t x = 0; x < nkv; ++x) dk[x] = dv[x] = 0.0;
  const int nbh = a->B * a->Hkv;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nbh) nthreads = nbh > 0 ? nbh : 1;
  bwd_job *jobs = (bwd_job *)malloc(sizeof(bwd_job) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].a = a;
    jobs[t].bh0 = nbh * t / nthreads;
    jobs[t].bh1 = nbh * (t + 1) / nthreads;
    jobs[t].dq = dq;
    jobs[t].dk = dk;
    jobs[t].dv = dv;
  }
  run_jobs(bwd_worker, jobs, sizeof(bwd_job), nthreads);
  free(jobs);
  return 0;
}
