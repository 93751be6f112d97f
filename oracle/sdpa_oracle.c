/*
 * CPU oracle for multi-head scaled-dot-product attention — TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the CPU-baseline leg of the benchmark may load
 * this file's library. The CUDA library never includes, links or calls it, and it shares
 * no code, header, table or constant with the CUDA library.
 *
 * What it computes is the plain definition from the Flux.jl page "Neural Network
 * primitives from NNlib.jl", entry NNlib.scaled_dot_product_attention:
 *
 *   out = softmax(scale * query' * key + bias, masked) * value        (first paragraph)
 *
 * in float64, one output row at a time, with a two-pass softmax and no tiling. Each
 * step below names the argument of that entry which defines it.
 *
 * Layout. The page's arrays are column-major (head_dim, nheads, seq_len, batch), which is
 * the same memory as row-major [batch][seq][head][dim]; this file indexes row-major:
 *   q[b][i][h][c]   (batch, q_len, nheads, qk_head_dim)
 *   k[b][j][g][c]   (batch, kv_len, nkvheads, qk_head_dim)
 *   v[b][j][g][e]   (batch, kv_len, nkvheads, v_head_dim)
 *   out[b][i][h][e] (batch, q_len, nheads, v_head_dim)
 * The bias and the mask are broadcastable to the page's (kv_len, q_len, nheads, batch);
 * they are addressed through four element strides in that order (key j, query i, head h,
 * batch b), a stride of 0 meaning the array is broadcast along that axis.
 *
 * Readings where the page leaves a step open (each also listed in the design notes):
 *  - GQA head sharing: query head h uses key/value head h / (nheads/nkvheads) (contiguous
 *    groups). The other grouping, h % nkvheads, is selectable for tests.
 *  - A masked logit is -infinity, so its weight is exactly zero; the bias is added first.
 *  - The bias is not multiplied by the scale.
 *  - A query row that attends to no key is NaN; a query row at or past q_lengths[b] is 0,
 *    and the zero wins when both hold.
 *  - :bottom_right takes q_offset[b] = kv_len[b] - q_len[b], with the array sizes where the
 *    lengths are not given; a negative offset is allowed.
 *
 * Parity pins: every function here is pinned by the CPU tests (closed forms, the stated
 * equivalences of the entry, PyTorch's float64 CPU routine on the special cases it can
 * express, brute force on tiny inputs).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_RANGE 2
#define ORACLE_ERR_NOMEM 3

typedef struct {
  int64_t batch, q_len, kv_len, nheads, nkvheads, dqk, dv;
  double scale;               /* NaN: 1/sqrt(dqk) (argument `scale`) */
  int32_t causal;             /* 0 false, 1 true (top-left), 2 :bottom_right */
  int32_t kv_head_rule;       /* 0: h / (nheads/nkvheads); 1: h % nkvheads */
  int64_t q_offset_scalar;    /* used when q_offset == NULL */
  const int64_t* q_offset;    /* [batch] or NULL */
  const int64_t* q_lengths;   /* [batch] or NULL (= q_len for every batch element) */
  const int64_t* kv_lengths;  /* [batch] or NULL (= kv_len for every batch element) */
  const double* bias;         /* NULL or broadcast array */
  int64_t bias_stride[4];     /* (j, i, h, b) element strides */
  const uint8_t* mask;        /* NULL or broadcast boolean array (0 = not attended) */
  int64_t mask_stride[4];     /* (j, i, h, b) element strides */
} oracle_sdpa_problem;

/* Checks the shape rules the entry states: nheads divisible by nkvheads (GQA paragraph). */
static int check_problem(const oracle_sdpa_problem* p) {
  if (!p) return ORACLE_ERR_ARG;
  if (p->batch < 0 || p->q_len < 0 || p->kv_len < 0) return ORACLE_ERR_ARG;
  if (p->nheads <= 0 || p->nkvheads <= 0 || p->dqk <= 0 || p->dv <= 0) return ORACLE_ERR_ARG;
  if (p->nheads % p->nkvheads != 0) return ORACLE_ERR_ARG;
  if (p->causal < 0 || p->causal > 2) return ORACLE_ERR_ARG;
  if (p->kv_head_rule < 0 || p->kv_head_rule > 1) return ORACLE_ERR_ARG;
  return ORACLE_OK;
}

/* One output row: batch b, query head h, query position i. `s` is scratch of kv_len doubles.
 * With `lse` not NULL it also receives the row's log-sum-exp, log sum_j exp(logit_j) over the
 * attended keys (the softmax's normaliser), +inf for a row with no key or past q_lengths. */
static void sdpa_row(const oracle_sdpa_problem* p, const double* q, const double* k,
                     const double* v, double* out, int64_t b, int64_t h, int64_t i,
                     double* s, unsigned char* allowed, double* lse) {
  const int64_t Lq = p->q_len, Lk = p->kv_len, H = p->nheads, Hkv = p->nkvheads;
  const int64_t D = p->dqk, Dv = p->dv;
  double* o = out + ((b * Lq + i) * H + h) * Dv;

  /* Argument `q_lengths`: the output is zero at the queries past q_lengths[b]. */
  const int64_t qlen_b = p->q_lengths ? p->q_lengths[b] : Lq;
  if (i >= qlen_b) {
    for (int64_t e = 0; e < Dv; ++e) o[e] = 0.0;
    if (lse) *lse = INFINITY;
    return;
  }
  /* Argument `kv_lengths`: the keys past kv_lengths[b] are not attended to. */
  const int64_t kvlen_b = p->kv_lengths ? p->kv_lengths[b] : Lk;

  /* GQA paragraph: key/value heads are shared across query heads. */
  const int64_t group = H / Hkv;
  const int64_t g = (p->kv_head_rule == 0) ? (h / group) : (h % Hkv);

  /* Argument `is_causal` / `q_offset`: query i attends keys j <= q_offset + i. */
  int64_t off = 0;
  if (p->causal == 1) off = p->q_offset ? p->q_offset[b] : p->q_offset_scalar;
  if (p->causal == 2) off = kvlen_b - qlen_b;

  /* Argument `scale`: default 1/sqrt(qk_head_dim). */
  const double scale = isnan(p->scale) ? 1.0 / sqrt((double)D) : p->scale;

  const double* qi = q + ((b * Lq + i) * H + h) * D;
  int64_t n_allowed = 0;
  double m = -INFINITY;
  for (int64_t j = 0; j < Lk; ++j) {
    /* `mask`, `is_causal` and `kv_lengths` combine: attended only where all allow it. */
    int ok = (j < kvlen_b);
    if (p->causal != 0 && !(j <= off + i)) ok = 0;
    if (p->mask) {
      const uint8_t mv = p->mask[j * p->mask_stride[0] + i * p->mask_stride[1] +
                                 h * p->mask_stride[2] + b * p->mask_stride[3]];
      if (!mv) ok = 0;
    }
    allowed[j] = (unsigned char)ok;
    if (!ok) continue;
    const double* kj = k + ((b * Lk + j) * Hkv + g) * D;
    double dot = 0.0;
    for (int64_t c = 0; c < D; ++c) dot += qi[c] * kj[c];
    double x = scale * dot;
    /* Argument `bias`: added to the logits before the softmax (not scaled). */
    if (p->bias)
      x += p->bias[j * p->bias_stride[0] + i * p->bias_stride[1] + h * p->bias_stride[2] +
                   b * p->bias_stride[3]];
    s[j] = x;
    if (x > m) m = x;
    ++n_allowed;
  }

  /* A query attending to no key has a NaN output (fused-implementation paragraph). */
  if (n_allowed == 0) {
    for (int64_t e = 0; e < Dv; ++e) o[e] = NAN;
    if (lse) *lse = INFINITY;
    return;
  }

  /* Softmax over the attended keys, then the weighted sum of the values. */
  double denom = 0.0;
  for (int64_t j = 0; j < Lk; ++j) {
    if (!allowed[j]) continue;
    s[j] = exp(s[j] - m);
    denom += s[j];
  }
  if (lse) *lse = m + log(denom);
  for (int64_t e = 0; e < Dv; ++e) o[e] = 0.0;
  for (int64_t j = 0; j < Lk; ++j) {
    if (!allowed[j]) continue;
    const double w = s[j] / denom;
    const double* vj = v + ((b * Lk + j) * Hkv + g) * Dv;
    for (int64_t e = 0; e < Dv; ++e) o[e] += w * vj[e];
  }
}

/* scaled_dot_product_attention(query, key, value, [bias]; mask, scale, is_causal, q_offset,
 * q_lengths, kv_lengths): every (b, h, i) row of the output, and with `lse` not NULL each row's
 * log-sum-exp, [batch][nheads][q_len]. */
int oracle_sdpa_forward_lse(const oracle_sdpa_problem* p, const double* q, const double* k,
                            const double* v, double* out, double* lse) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (p->batch == 0 || p->q_len == 0) return ORACLE_OK;
  const int64_t rows = p->batch * p->nheads * p->q_len;
  int failed = 0;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(p->kv_len > 0 ? p->kv_len : 1));
    unsigned char* allowed = (unsigned char*)malloc((size_t)(p->kv_len > 0 ? p->kv_len : 1));
    if (!s || !allowed) {
#pragma omp atomic write
      failed = 1;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (int64_t r = 0; r < rows; ++r) {
        const int64_t b = r / (p->nheads * p->q_len);
        const int64_t h = (r / p->q_len) % p->nheads;
        const int64_t i = r % p->q_len;
        sdpa_row(p, q, k, v, out, b, h, i, s, allowed, lse ? lse + (b * p->nheads + h) * p->q_len + i : NULL);
      }
    }
    free(s);
    free(allowed);
  }
  return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

int oracle_sdpa_forward(const oracle_sdpa_problem* p, const double* q, const double* k,
                        const double* v, double* out) {
  return oracle_sdpa_forward_lse(p, q, k, v, out, NULL);
}

/* Rotary position embedding of query or key rows (the Keras thread "MultiHeadAttention is
 * missing a position_bias call argument": rotary embeddings applied to the key and query after
 * the dense projections; the thread leaves the exact form open). Reading taken here, the common
 * form: the head dimension d (even) is split in halves, and the pair (c, c + d/2),
 * c < d/2, of row t is rotated by the angle positions[t] * base^(-2c/d):
 *   out[c]       = x[c] cos a - x[c + d/2] sin a
 *   out[c + d/2] = x[c + d/2] cos a + x[c] sin a
 * x and out are [rows][nheads][d]; positions has one entry per row. */
int oracle_rope(const double* x, int64_t rows, int64_t nheads, int64_t d, const int64_t* positions,
                double base, double* out) {
  if (!x || !out || !positions || rows < 0 || nheads <= 0 || d <= 0 || d % 2 || !(base > 0.0))
    return ORACLE_ERR_ARG;
  const int64_t half = d / 2;
  for (int64_t t = 0; t < rows; ++t)
    for (int64_t h = 0; h < nheads; ++h) {
      const double* xr = x + (t * nheads + h) * d;
      double* o = out + (t * nheads + h) * d;
      for (int64_t c = 0; c < half; ++c) {
        const double a = (double)positions[t] * pow(base, -2.0 * (double)c / (double)d);
        const double x0 = xr[c], x1 = xr[c + half];
        o[c] = x0 * cos(a) - x1 * sin(a);
        o[c + half] = x1 * cos(a) + x0 * sin(a);
      }
    }
  return ORACLE_OK;
}

/* Counter-based dropout draw: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014). Its n-th output (n = 1, 2, ...) from state `seed` is the
 * mixing function applied to seed + n * gamma, gamma = 0x9e3779b97f4a7c15. The weights' linear
 * indices (b, h, i, j), row-major, are taken four at a time: group g = index / 4 gets output
 * n = g + 1, and the weight at `index` takes its 16-bit field number index % 4 (lowest first)
 * as an integer u in [0, 2^16). The weight is kept when u >= threshold = ceil(drop_p * 2^16):
 * with probability 1 - threshold / 2^16, within 2^-16 of 1 - drop_p. */
static uint64_t splitmix64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}
static int dropout_keep(uint64_t seed, uint64_t index, uint32_t threshold) {
  const uint64_t r = splitmix64_mix(seed + ((index >> 2) + 1) * 0x9e3779b97f4a7c15ULL);
  const uint32_t u = (uint32_t)(r >> (16 * (index & 3))) & 0xFFFFu;
  return u >= threshold;
}

/* scaled_dot_product_attention_with_weights (the entry's "See also": the attention weights too)
 * with an fdrop that is dropout of probability drop_p (argument fdrop: applied to the weights
 * right after the softmax). The weights are materialized (paragraph "Fused implementation":
 * any call with an fdrop takes the materialized implementation):
 *   w_ij = softmax_j(scale q_i.k_j + bias_ij, masked)
 *   w'_ij = w_ij / (1 - drop_p) where the draw of (b, h, i, j) keeps it, else 0
 *   out_i = sum_j w'_ij v_j
 * and `weights` receives w' in the page's (kv_len, q_len, nheads, batch) order, which is
 * row-major [batch][nheads][q_len][kv_len]. A row with no attended key has NaN weights and a
 * NaN output; a row past q_lengths has zero weights and a zero output. drop_p must be in
 * [0, 1). */
int oracle_sdpa_forward_with_weights(const oracle_sdpa_problem* p, const double* q, const double* k,
                                     const double* v, double drop_p, uint64_t seed, double* out,
                                     double* weights) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (!(drop_p >= 0.0 && drop_p < 1.0)) return ORACLE_ERR_ARG;
  const int64_t B = p->batch, Lq = p->q_len, Lk = p->kv_len, H = p->nheads, Hkv = p->nkvheads;
  const int64_t D = p->dqk, Dv = p->dv, group = H / Hkv;
  const double scale = isnan(p->scale) ? 1.0 / sqrt((double)D) : p->scale;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < B * H * Lq; ++r) {
    const int64_t b = r / (H * Lq), h = (r / Lq) % H, i = r % Lq;
    double* wrow = weights + ((b * H + h) * Lq + i) * Lk;
    double* o = out + ((b * Lq + i) * H + h) * Dv;
    const int64_t qlen_b = p->q_lengths ? p->q_lengths[b] : Lq;
    const int64_t kvlen_b = p->kv_lengths ? p->kv_lengths[b] : Lk;
    for (int64_t j = 0; j < Lk; ++j) wrow[j] = 0.0;
    for (int64_t e = 0; e < Dv; ++e) o[e] = 0.0;
    if (i >= qlen_b) continue;
    int64_t off = 0;
    if (p->causal == 1) off = p->q_offset ? p->q_offset[b] : p->q_offset_scalar;
    if (p->causal == 2) off = kvlen_b - qlen_b;
    const int64_t g = h / group;
    const double* qi = q + ((b * Lq + i) * H + h) * D;
    double m = -INFINITY;
    int64_t n = 0;
    for (int64_t j = 0; j < Lk; ++j) {
      int a = (j < kvlen_b);
      if (p->causal != 0 && !(j <= off + i)) a = 0;
      if (p->mask && !p->mask[j * p->mask_stride[0] + i * p->mask_stride[1] + h * p->mask_stride[2] +
                              b * p->mask_stride[3]])
        a = 0;
      if (!a) {
        wrow[j] = -INFINITY;
        continue;
      }
      const double* kj = k + ((b * Lk + j) * Hkv + g) * D;
      double dot = 0.0;
      for (int64_t c = 0; c < D; ++c) dot += qi[c] * kj[c];
      double x = scale * dot;
      if (p->bias)
        x += p->bias[j * p->bias_stride[0] + i * p->bias_stride[1] + h * p->bias_stride[2] +
                     b * p->bias_stride[3]];
      wrow[j] = x;
      if (x > m) m = x;
      ++n;
    }
    if (n == 0) {
      for (int64_t j = 0; j < Lk; ++j) wrow[j] = NAN;
      for (int64_t e = 0; e < Dv; ++e) o[e] = NAN;
      continue;
    }
    double z = 0.0;
    for (int64_t j = 0; j < Lk; ++j) {
      wrow[j] = (wrow[j] == -INFINITY) ? 0.0 : exp(wrow[j] - m);
      z += wrow[j];
    }
    const uint64_t base = (uint64_t)(((b * H + h) * Lq + i) * Lk);
    const uint32_t thr = (uint32_t)ceil(drop_p * 65536.0);
    for (int64_t j = 0; j < Lk; ++j) {
      double w = wrow[j] / z;
      if (drop_p > 0.0)
        w = dropout_keep(seed, base + (uint64_t)j, thr) ? w / (1.0 - drop_p) : 0.0;
      wrow[j] = w;
      if (w == 0.0) continue;
      const double* vj = v + ((b * Lk + j) * Hkv + g) * Dv;
      for (int64_t e = 0; e < Dv; ++e) o[e] += w * vj[e];
    }
  }
  return ORACLE_OK;
}

/* The gradient of the fused implementation (paragraph "Fused implementation": the fused
 * implementation has a gradient with respect to query, key, value and scale, and a query that
 * attends to no key, whose output is NaN, takes no part in it). For the loss
 * L = sum over output elements of dout * out, with w_j the softmax weights of a row and
 * x_j = scale * q.k_j its attended logits:
 *   dv_j    += w_j * dout_i
 *   dw_j     = dout_i . v_j
 *   dx_j     = w_j * (dw_j - sum_l w_l dw_l)
 *   dq_i     = scale * sum_j dx_j k_j
 *   dk_j    += scale * dx_j q_i
 *   dscale  += sum_j dx_j (q_i . k_j)
 * summed over the query heads that share a key/value head. Rows past q_lengths (constant zero)
 * and rows with no attended key contribute nothing and get dq = 0. A bias is an error: under
 * automatic differentiation a call with a bias takes the materialized implementation. */
int oracle_sdpa_backward(const oracle_sdpa_problem* p, const double* q, const double* k,
                         const double* v, const double* dout, double* dq, double* dk, double* dv,
                         double* dscale) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (p->bias || p->kv_head_rule != 0) return ORACLE_ERR_ARG;
  const int64_t B = p->batch, Lq = p->q_len, Lk = p->kv_len, H = p->nheads, Hkv = p->nkvheads;
  const int64_t D = p->dqk, Dv = p->dv, group = H / Hkv;
  const double scale = isnan(p->scale) ? 1.0 / sqrt((double)D) : p->scale;
  memset(dq, 0, sizeof(double) * (size_t)(B * Lq * H * D));
  memset(dk, 0, sizeof(double) * (size_t)(B * Lk * Hkv * D));
  memset(dv, 0, sizeof(double) * (size_t)(B * Lk * Hkv * Dv));
  int failed = 0;
  /* dscale's share of each (batch, key/value head), summed in that order after the loop, so
   * that the result does not depend on how the threads took the units */
  double* part = (double*)calloc((size_t)(B * Hkv > 0 ? B * Hkv : 1), sizeof(double));
  if (!part) return ORACLE_ERR_NOMEM;
  /* each (batch, key/value head) owns its rows of dk and dv */
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bg = 0; bg < B * Hkv; ++bg) {
    const int64_t b = bg / Hkv, g = bg % Hkv;
    double total = 0.0;
    double* x = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    double* dw = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    unsigned char* ok = (unsigned char*)malloc((size_t)(Lk > 0 ? Lk : 1));
    if (!x || !dw || !ok) {
#pragma omp atomic write
      failed = 1;
      free(x);
      free(dw);
      free(ok);
      continue;
    }
    const int64_t qlen_b = p->q_lengths ? p->q_lengths[b] : Lq;
    const int64_t kvlen_b = p->kv_lengths ? p->kv_lengths[b] : Lk;
    int64_t off = 0;
    if (p->causal == 1) off = p->q_offset ? p->q_offset[b] : p->q_offset_scalar;
    if (p->causal == 2) off = kvlen_b - qlen_b;
    for (int64_t h = g * group; h < (g + 1) * group; ++h) {
      for (int64_t i = 0; i < qlen_b && i < Lq; ++i) {
        const double* qi = q + ((b * Lq + i) * H + h) * D;
        const double* doi = dout + ((b * Lq + i) * H + h) * Dv;
        double m = -INFINITY;
        int64_t n = 0;
        for (int64_t j = 0; j < Lk; ++j) {
          int a = (j < kvlen_b);
          if (p->causal != 0 && !(j <= off + i)) a = 0;
          if (p->mask && !p->mask[j * p->mask_stride[0] + i * p->mask_stride[1] +
                                  h * p->mask_stride[2] + b * p->mask_stride[3]])
            a = 0;
          ok[j] = (unsigned char)a;
          if (!a) continue;
          const double* kj = k + ((b * Lk + j) * Hkv + g) * D;
          double dot = 0.0;
          for (int64_t c = 0; c < D; ++c) dot += qi[c] * kj[c];
          x[j] = scale * dot;
          if (x[j] > m) m = x[j];
          ++n;
        }
        if (n == 0) continue; /* NaN row: no part in the gradient */
        double z = 0.0;
        for (int64_t j = 0; j < Lk; ++j)
          if (ok[j]) {
            x[j] = exp(x[j] - m);
            z += x[j];
          }
        double wdw = 0.0;
        for (int64_t j = 0; j < Lk; ++j) {
          if (!ok[j]) continue;
          x[j] /= z; /* now the weight w_j */
          const double* vj = v + ((b * Lk + j) * Hkv + g) * Dv;
          double t = 0.0;
          for (int64_t e = 0; e < Dv; ++e) t += doi[e] * vj[e];
          dw[j] = t;
          wdw += x[j] * t;
        }
        double* dqi = dq + ((b * Lq + i) * H + h) * D;
        for (int64_t j = 0; j < Lk; ++j) {
          if (!ok[j]) continue;
          const double dx = x[j] * (dw[j] - wdw);
          const double* kj = k + ((b * Lk + j) * Hkv + g) * D;
          double* dkj = dk + ((b * Lk + j) * Hkv + g) * D;
          double* dvj = dv + ((b * Lk + j) * Hkv + g) * Dv;
          double dot = 0.0;
          for (int64_t c = 0; c < D; ++c) {
            dot += qi[c] * kj[c];
            dqi[c] += scale * dx * kj[c];
            dkj[c] += scale * dx * qi[c];
          }
          for (int64_t e = 0; e < Dv; ++e) dvj[e] += x[j] * doi[e];
          total += dx * dot;
        }
      }
    }
    part[bg] = total;
    free(x);
    free(dw);
    free(ok);
  }
  double total = 0.0;
  for (int64_t bg = 0; bg < B * Hkv; ++bg) total += part[bg];
  free(part);
  if (failed) return ORACLE_ERR_NOMEM;
  if (dscale) *dscale = total;
  return ORACLE_OK;
}

/* Packed sequences (the entry's keywords q_segments, kv_segments, maxlen and its paragraph
 * "Packed sequences"): query holds nseg sequences of q_segments[s] rows one after the other,
 * key and value nseg sequences of kv_segments[s] rows; the s-th query segment attends to the
 * s-th key/value segment only, exactly as batch element s of a padded batch would. Here p
 * describes the packed arrays: batch = 1, q_len / kv_len the total lengths, and q_offset,
 * q_lengths, kv_lengths (when given) hold one entry per segment. The segment lengths must add
 * up to the total lengths, no length may be negative, and maxlen (when >= 0) must be at least
 * every segment; a bias or a mask is an error. */
int oracle_sdpa_forward_packed(const oracle_sdpa_problem* p, int64_t nseg,
                               const int64_t* q_segments, const int64_t* kv_segments,
                               int64_t maxlen, const double* q, const double* k,
                               const double* v, double* out) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (p->batch != 1 || nseg < 0 || (nseg > 0 && !q_segments)) return ORACLE_ERR_ARG;
  if (p->bias || p->mask) return ORACLE_ERR_ARG;
  const int64_t* kvs = kv_segments ? kv_segments : q_segments; /* kv_segments defaults */
  int64_t q_tot = 0, kv_tot = 0;
  for (int64_t s = 0; s < nseg; ++s) {
    if (q_segments[s] < 0 || kvs[s] < 0) return ORACLE_ERR_ARG;
    if (maxlen >= 0 && (q_segments[s] > maxlen || kvs[s] > maxlen)) return ORACLE_ERR_RANGE;
    q_tot += q_segments[s];
    kv_tot += kvs[s];
  }
  if (q_tot != p->q_len || kv_tot != p->kv_len) return ORACLE_ERR_ARG;
  const int64_t H = p->nheads, Hkv = p->nkvheads;
  int64_t q0 = 0, k0 = 0;
  for (int64_t s = 0; s < nseg; ++s) {
    oracle_sdpa_problem ps = *p;
    ps.q_len = q_segments[s];
    ps.kv_len = kvs[s];
    ps.q_offset = p->q_offset ? p->q_offset + s : NULL;
    ps.q_lengths = p->q_lengths ? p->q_lengths + s : NULL;
    ps.kv_lengths = p->kv_lengths ? p->kv_lengths + s : NULL;
    rc = oracle_sdpa_forward(&ps, q + q0 * H * p->dqk, k + k0 * Hkv * p->dqk,
                             v + k0 * Hkv * p->dv, out + q0 * H * p->dv);
    if (rc) return rc;
    q0 += q_segments[s];
    k0 += kvs[s];
  }
  return ORACLE_OK;
}

/* Writing new keys/values into a KV cache at a per-sequence position (the Keras issue
 * "MultiHeadAttention is missing a position_bias call argument": `cache_update_index`; the
 * Flax discussion's cached_key/cached_value, shaped (batch, len, heads, head_dim)):
 *   cache[b][index[b] + t][g][c] = new[b][t][g][c]   for t < n_new.
 * An index outside [0, capacity - n_new] is an error and nothing is written. */
int oracle_cache_update_at_index(double* cache, const double* new_rows, int64_t batch,
                                 int64_t capacity, int64_t n_new, int64_t nkvheads, int64_t d,
                                 const int64_t* index) {
  if (batch < 0 || capacity < 0 || n_new < 0 || nkvheads <= 0 || d <= 0 || !index)
    return ORACLE_ERR_ARG;
  for (int64_t b = 0; b < batch; ++b)
    if (index[b] < 0 || index[b] + n_new > capacity) return ORACLE_ERR_RANGE;
  const int64_t row = nkvheads * d;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t t = 0; t < n_new; ++t)
      memcpy(cache + (b * capacity + index[b] + t) * row, new_rows + (b * n_new + t) * row,
             sizeof(double) * (size_t)row);
  return ORACLE_OK;
}

/* Decoding with a KV cache (the entry's example "decoding with a KV cache"): write the new
 * keys/values at index[b], then attend with is_causal=:bottom_right and
 * kv_lengths[b] = index[b] + n_new, the n_new queries being the last positions. */
int oracle_sdpa_decode_with_cache(const oracle_sdpa_problem* p_in, const double* q,
                                  const double* k_new, const double* v_new, double* k_cache,
                                  double* v_cache, const int64_t* index, double* out) {
  if (!p_in || !index) return ORACLE_ERR_ARG;
  oracle_sdpa_problem p = *p_in; /* q_len = n_new, kv_len = capacity */
  int rc = oracle_cache_update_at_index(k_cache, k_new, p.batch, p.kv_len, p.q_len, p.nkvheads,
                                        p.dqk, index);
  if (rc) return rc;
  rc = oracle_cache_update_at_index(v_cache, v_new, p.batch, p.kv_len, p.q_len, p.nkvheads, p.dv,
                                    index);
  if (rc) return rc;
  int64_t* kvl = (int64_t*)malloc(sizeof(int64_t) * (size_t)(p.batch > 0 ? p.batch : 1));
  if (!kvl) return ORACLE_ERR_NOMEM;
  for (int64_t b = 0; b < p.batch; ++b) kvl[b] = index[b] + p.q_len;
  p.kv_lengths = kvl;
  p.q_lengths = NULL;
  p.causal = 2;
  rc = oracle_sdpa_forward(&p, q, k_cache, v_cache, out);
  free(kvl);
  return rc;
}

/* Block classification of a boolean mask, after the splash-attention mask info of the JAX
 * pull request "Support dynamic masks in splash attention": the mask is cut into blocks of
 * bq queries x bk keys, and each block is empty (no key attended), full (every key
 * attended) or partial. A block at the ragged edge counts only its in-range cells.
 *
 * Outputs, for mask heads h < nheads (the mask's own head extent) and block rows qb:
 *  - cls[h][qb][kb]: 0 empty, 1 partial, 2 full (this library's own encoding);
 *  - count[h][qb]: the number of non-empty blocks of the row;
 *  - list[h][qb][n] for n < count: the non-empty kb in increasing order, with the class in
 *    the top two bits: kb | (cls << 30);
 *  - bits: for each partial block, at block slot (h*nqb + qb)*nkb + kb, bq rows of
 *    ceil(bk/32) 32-bit words, bit c of word w of row r = mask(h, qb*bq + r, kb*bk + 32w + c);
 *    out-of-range cells are 0. Slots of non-partial blocks are left untouched.
 * The mask is read as mask[j*ms[0] + i*ms[1] + h*ms[2]] (key j, query i, head h). */
int oracle_block_mask_info(const uint8_t* mask, const int64_t ms[3], int64_t nheads,
                           int64_t q_len, int64_t kv_len, int64_t bq, int64_t bk, uint8_t* cls,
                           int32_t* count, uint32_t* list, uint32_t* bits) {
  if (!mask || !ms || nheads <= 0 || q_len <= 0 || kv_len <= 0 || bq <= 0 || bk <= 0)
    return ORACLE_ERR_ARG;
  const int64_t nqb = (q_len + bq - 1) / bq, nkb = (kv_len + bk - 1) / bk;
  const int64_t words = (bk + 31) / 32;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t hq = 0; hq < nheads * nqb; ++hq) {
    const int64_t h = hq / nqb, qb = hq % nqb;
    int32_t n = 0;
    for (int64_t kb = 0; kb < nkb; ++kb) {
      int64_t cells = 0, set = 0;
      for (int64_t r = 0; r < bq; ++r) {
        const int64_t i = qb * bq + r;
        if (i >= q_len) break;
        for (int64_t c = 0; c < bk; ++c) {
          const int64_t j = kb * bk + c;
          if (j >= kv_len) break;
          ++cells;
          if (mask[j * ms[0] + i * ms[1] + h * ms[2]]) ++set;
        }
      }
      const uint8_t cl = (set == 0) ? 0 : (set == cells ? 2 : 1);
      cls[(h * nqb + qb) * nkb + kb] = cl;
      if (cl != 0) list[(h * nqb + qb) * nkb + (n++)] = (uint32_t)kb | ((uint32_t)cl << 30);
      if (cl == 1) {
        uint32_t* blk = bits + ((h * nqb + qb) * nkb + kb) * bq * words;
        for (int64_t r = 0; r < bq; ++r)
          for (int64_t w = 0; w < words; ++w) {
            uint32_t word = 0;
            for (int64_t c = 0; c < 32; ++c) {
              const int64_t i = qb * bq + r, jc = w * 32 + c, j = kb * bk + jc;
              if (i < q_len && jc < bk && j < kv_len && mask[j * ms[0] + i * ms[1] + h * ms[2]])
                word |= (1u << c);
            }
            blk[r * words + w] = word;
          }
      }
    }
    count[h * nqb + qb] = n;
  }
  return ORACLE_OK;
}

/* Number of host threads the OpenMP loops above use (reported beside timings). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
