/*
 * pa_oracle.c — fp64 CPU oracle for causal GQA prefill attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the correctness reference that the CUDA path is
 * checked against. Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference leg may load it. It shares no code, header, table or helper with the CUDA
 * library under paged_kv_long_b200/, and includes none of its files.
 *
 * What it computes (the plain definition, no blocking, no online softmax, no splits):
 *   "Metal: paged-KV prefill is 4.43x slower than contiguous KV at 32K" (BaseRT issue #51),
 *   section "Reproduction"/"Scaling characteristic": prefill attention that reads its K/V
 *   through a paged cache must give what the contiguous cache gives.
 *   "perf: scale prefill attention splits with GPU cores on Apple7/8" (splash PR #33),
 *   section "Testing": the split kernel is verified by comparison with a CPU implementation;
 *   splitting the history changes only rounding.
 *   Shapes: 24 Q / 4 KV heads, D256 ("KVarN V-store per-call latency ..." issue #163, Setup);
 *   16 Q / 2 KV heads, head_dim 256 (BaseRT issue #51, "Model provenance").
 *
 * For query row i of the chunk (absolute position H+i) and Q head h, with G = Hq/Hkv and
 * KV head g = floor(h/G):
 *   K[j] = k_pool[page_table[j / PS]][j % PS][g][:]   (paged)   or  k[j][g][:] (contiguous)
 *   s_j  = scale * sum_d q[i][h][d] * K[j][d]            for 0 <= j <= H+i  (others skipped)
 *   m    = max_j s_j;  p_j = exp(s_j - m);  l = sum_j p_j
 *   out  = sum_j (p_j / l) * V[j][:];        lse = m + ln(l)
 * Readings where the pages are silent: scale 1/sqrt(D) unless given; contiguous GQA groups
 * (g = floor(h/G)); the chunk's own keys are already in the cache; row i sees 0..H+i.
 *
 * The 16-bit inputs are decoded exactly to double (binary16 and bfloat16 are subsets of
 * binary64), so the only rounding in the oracle is fp64 arithmetic.
 *
 * Mutation hooks: when compiled with -DORC_MUTANT=n the oracle carries one deliberate
 * mistake (used by the pin tests to show that the pins catch it). The default build has none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORC_MUTANT
#define ORC_MUTANT 0
#endif

enum { ORC_F16 = 0, ORC_BF16 = 1 };
enum { ORC_OK = 0, ORC_ERR_ARG = -1, ORC_ERR_PAGE = -2, ORC_ERR_NOMEM = -3 };

/* IEEE 754 binary16: sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double orc_decode_f16(uint16_t h) {
  int sign = h >> 15, e = (h >> 10) & 0x1f, f = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24);                 /* subnormal: f * 2^-14 * 2^-10 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f | 0x400), e - 25);    /* (1 + f/1024) * 2^(e-15) */
  return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE 754 binary32. */
double orc_decode_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

double orc_decode(int dtype, uint16_t x) {
  return dtype == ORC_BF16 ? orc_decode_bf16(x) : orc_decode_f16(x);
}

typedef struct {
  int32_t dtype;        /* ORC_F16 or ORC_BF16 */
  int32_t paged;        /* 1: k/v are pools [num_pages][PS][Hkv][D]; 0: [H+R][Hkv][D] */
  int32_t page_size;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int64_t num_pages;    /* pool pages (paged) */
  int64_t table_len;    /* entries in page_table (paged) */
  int64_t hist_len;     /* H: keys already in the cache before the chunk */
  int64_t chunk_rows;   /* R: query rows of the chunk */
  double scale;         /* softmax scale; <= 0 means 1/sqrt(D) */
  const uint16_t* q;    /* [R][Hq][D] */
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* page_table;
} orc_problem;

static double eff_scale(const orc_problem* p) {
#if ORC_MUTANT == 3
  return 1.0; /* mutant: scale dropped */
#else
  return p->scale > 0 ? p->scale : 1.0 / sqrt((double)p->head_dim);
#endif
}

/* Pointer to the D values of logical key j for KV head g, or NULL if the page-table entry
 * is out of range. */
static const uint16_t* kv_row(const orc_problem* p, const uint16_t* base, int64_t j, int g) {
  const int64_t D = p->head_dim, Hkv = p->n_kv_heads;
  if (!p->paged) return base + (j * Hkv + g) * D;
  const int64_t PS = p->page_size;
#if ORC_MUTANT == 4
  const int64_t lp = j % PS, slot = j / PS;  /* mutant: page and slot swapped */
  if (lp >= p->table_len || slot >= PS) return NULL;
#else
  const int64_t lp = j / PS, slot = j % PS;
  if (lp >= p->table_len) return NULL;
#endif
  const int64_t phys = p->page_table[lp];
  if (phys < 0 || phys >= p->num_pages) return NULL;
  return base + ((phys * PS + slot) * Hkv + g) * D;
}

static int kv_head_of(const orc_problem* p, int h) {
#if ORC_MUTANT == 2
  return h % p->n_kv_heads; /* mutant: interleaved instead of grouped heads */
#else
  return h / (p->n_q_heads / p->n_kv_heads);
#endif
}

/* Last key (inclusive) visible to chunk row i. */
static int64_t last_visible(const orc_problem* p, int64_t i) {
#if ORC_MUTANT == 1
  return p->hist_len + i + 1; /* mutant: causal limit one too far */
#else
  return p->hist_len + i;
#endif
}

/* Softmax weights of one (row, head) over keys [lo, hi) intersected with the causal range.
 * w has room for hi - lo values; invisible keys get 0. Returns the number of visible keys
 * (0: w all zero, *m = -inf), or a negative error. Also returns m (max score) and l. */
static int64_t row_weights(const orc_problem* p, const double* lut, int64_t i, int h, int64_t lo,
                           int64_t hi, double* w, double* m_out, double* l_out) {
  const int D = p->head_dim, g = kv_head_of(p, h);
  const double scale = eff_scale(p);
  const uint16_t* qrow = p->q + ((int64_t)i * p->n_q_heads + h) * D;
  int64_t end = last_visible(p, i) + 1;
  if (end > hi) end = hi;
  double m = -INFINITY;
  for (int64_t j = lo; j < hi; ++j) w[j - lo] = 0.0;
  for (int64_t j = lo; j < end; ++j) {
    const uint16_t* krow = kv_row(p, p->k, j, g);
    if (!krow) return ORC_ERR_PAGE;
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += lut[qrow[d]] * lut[krow[d]];
    const double s = scale * dot;
    w[j - lo] = s;
    if (s > m) m = s;
  }
  double l = 0.0;
  for (int64_t j = lo; j < end; ++j) {
    const double e = exp(w[j - lo] - m);
    w[j - lo] = e;
    l += e;
  }
  *m_out = m;
  *l_out = l;
  return end > lo ? end - lo : 0;
}

static double* make_lut(int dtype) {
  double* lut = (double*)malloc(65536 * sizeof(double));
  if (!lut) return NULL;
  for (uint32_t x = 0; x < 65536; ++x) lut[x] = orc_decode(dtype, (uint16_t)x);
  return lut;
}

static int check_problem(const orc_problem* p) {
  if (!p || !p->q || !p->k || !p->v) return ORC_ERR_ARG;
  if (p->n_q_heads <= 0 || p->n_kv_heads <= 0 || p->n_q_heads % p->n_kv_heads) return ORC_ERR_ARG;
  if (p->head_dim <= 0 || p->hist_len < 0 || p->chunk_rows < 0) return ORC_ERR_ARG;
  if (p->paged && (p->page_size <= 0 || !p->page_table)) return ORC_ERR_ARG;
  return ORC_OK;
}

/*
 * Attention of sampled (row, head) pairs restricted to keys [key_lo, key_hi) (clipped to
 * the causal range). With key_lo = 0 and key_hi >= H+R this is the full result. For each
 * sample n: out[n][0..D) and lse[n] (natural log). A sample that sees no key gets out = 0
 * and lse = -inf. rows[n] is the chunk-relative row (0..R-1).
 */
int orc_attend(const orc_problem* p, int64_t key_lo, int64_t key_hi, int64_t n_samples,
               const int64_t* rows, const int32_t* heads, double* out, double* lse,
               int n_threads) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (key_lo < 0 || key_hi < key_lo) return ORC_ERR_ARG;
  for (int64_t n = 0; n < n_samples; ++n)
    if (rows[n] < 0 || rows[n] >= p->chunk_rows || heads[n] < 0 || heads[n] >= p->n_q_heads)
      return ORC_ERR_ARG;
  double* lut = make_lut(p->dtype);
  if (!lut) return ORC_ERR_NOMEM;
  const int D = p->head_dim;
  int status = ORC_OK;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t n = 0; n < n_samples; ++n) {
    const int64_t i = rows[n];
    const int h = heads[n];
    int64_t hi = key_hi;
    if (hi > last_visible(p, i) + 1) hi = last_visible(p, i) + 1;
    if (hi < key_lo) hi = key_lo;
    double* o = out + n * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    double* w = (double*)malloc((size_t)(hi - key_lo + 1) * sizeof(double));
    if (!w) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      status = ORC_ERR_NOMEM;
      continue;
    }
    double m, l;
    const int64_t nvis = row_weights(p, lut, i, h, key_lo, hi, w, &m, &l);
    if (nvis < 0) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      status = (int)nvis;
    } else if (nvis == 0) {
      lse[n] = -INFINITY;
    } else {
      const int g = kv_head_of(p, h);
      for (int64_t j = key_lo; j < hi; ++j) {
        const double wj = w[j - key_lo] / l;
        const uint16_t* vrow = kv_row(p, p->v, j, g);
        for (int d = 0; d < D; ++d) o[d] += wj * lut[vrow[d]];
      }
#if ORC_MUTANT == 5
      lse[n] = log(l); /* mutant: max term dropped from the log-sum-exp */
#else
      lse[n] = m + log(l);
#endif
    }
    free(w);
  }
  free(lut);
  return status;
}

/* Normalised softmax weights of one (row, head) over all keys 0..H+R-1 (invisible keys 0). */
int orc_weights(const orc_problem* p, int64_t row, int32_t head, double* w) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (row < 0 || row >= p->chunk_rows || head < 0 || head >= p->n_q_heads) return ORC_ERR_ARG;
  double* lut = make_lut(p->dtype);
  if (!lut) return ORC_ERR_NOMEM;
  const int64_t total = p->hist_len + p->chunk_rows;
  double m, l;
  const int64_t nvis = row_weights(p, lut, row, head, 0, total, w, &m, &l);
  free(lut);
  if (nvis < 0) return (int)nvis;
  for (int64_t j = 0; j < total; ++j) w[j] /= l;
  return ORC_OK;
}

/* Log-sum-exp merge of S partial results of one (row, head): each partial is normalised
 * over its own key range (o_s) with log-sum-exp lse_s; the whole is
 *   out = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M),  lse = M + ln sum_s exp(lse_s - M),
 * with M = max_s lse_s. Partials with lse_s = -inf carry no weight. */
void orc_merge(int n_parts, int D, const double* lse_parts, const double* o_parts, double* out,
               double* lse_out) {
  double M = -INFINITY;
  for (int s = 0; s < n_parts; ++s)
    if (lse_parts[s] > M) M = lse_parts[s];
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (M == -INFINITY) {
    *lse_out = -INFINITY;
    return;
  }
  double wsum = 0.0;
  for (int s = 0; s < n_parts; ++s) {
    if (lse_parts[s] == -INFINITY) continue;
    const double w = exp(lse_parts[s] - M);
    wsum += w;
    for (int d = 0; d < D; ++d) out[d] += w * o_parts[(int64_t)s * D + d];
  }
  for (int d = 0; d < D; ++d) out[d] /= wsum;
  *lse_out = M + log(wsum);
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
