/*
 * s2_oracle.c -- plain float64 CPU oracle for shifted sparse attention (S²-Attn).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the package smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * library: it is written directly from the method's definition, slowly and
 * obviously, so that the GPU kernels can be checked against it.
 *
 * Sources (page title, section):
 *   [PT]  "4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" (PaperTrace notes)
 *         §1 "S²-Attn的计算图": group index b(i)=floor(i/G); shifted heads use
 *             b'(i)=floor((i-G/2)/G) and exclude wrapped positions; the visible
 *             sets N_0(i) and N_1(i); the rolled scheme's last group [6,7,0,1];
 *             the strict variant with separate short head/tail groups; the
 *             second half of the heads Q[:, H/2:] is the shifted half; pad to
 *             whole groups and mask invalid K/V.
 *         §3 "稀疏训练与full推理之间的目标偏移": o_i = softmax over S_i of
 *             q_i·k_j/sqrt(D), applied to v_j; dL/dz_j = a_j g^T (v_j - o_i).
 *   [LN]  "精读笔记：LongLoRA — 长上下文大模型的高效微调", §3.2.2: pattern 2's
 *         first group of an 8192-token context with G=2048 spans tokens
 *         1025..3072 (1-indexed).
 *
 * Readings taken where the pages leave a step open (all 0-indexed):
 *   - variant 0 (STRICT): shifted heads group by floor((x - s)/G) with floor
 *     division, s = G/2; this yields the short head group [0,s), the full
 *     groups [s+kG, s+kG+G) and the short tail group [N-s, N); visibility
 *     also needs j <= i, so no wrapped edge exists.
 *   - variant 1 (ROLLED): rolled index r(x) = (x - s) mod N (a left roll by s);
 *     j visible from i iff floor(r(i)/G) == floor(r(j)/G) and r(j) <= r(i).
 *   - variant 2 (DENSE_CAUSAL): every head sees j <= i (the inference graph).
 *   - a position x is valid iff x < n_valid; invalid keys are never visible and
 *     invalid query rows see nothing: o = 0, lse = -inf, and their output
 *     gradient is treated as 0 (loss mask).
 *   - lse is the natural log of sum_j exp(scale q_i·k_j); scale = 1/sqrt(D).
 *   - document mask ([PT] §1.1 "因果mask与样本packing"): when several documents
 *     are packed into one sequence, j is visible from i only if, in addition,
 *     doc(i) == doc(j); the same constraint applies to the original and the
 *     shifted grouping.  doc is a per-position ID array [B, N] (NULL: one
 *     document); IDs need not be contiguous runs here.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define S2O_STRICT 0
#define S2O_ROLLED 1
#define S2O_DENSE_CAUSAL 2

/* floor division for possibly negative numerators (positive divisor). */
static int64_t floor_div(int64_t a, int64_t b) {
  int64_t q = a / b;
  if ((a % b != 0) && (a < 0)) q -= 1;
  return q;
}

static int64_t pos_mod(int64_t a, int64_t n) {
  int64_t r = a % n;
  return r < 0 ? r + n : r;
}

/* The visibility predicate A^(c)[i][j] of [PT] §1.  Returns 1 if key j is
 * visible from query i for a head of class c (0: heads [0,H/2), 1: heads
 * [H/2,H)), else 0. */
int s2o_visible(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class,
                int64_t i, int64_t j) {
  if (i < 0 || j < 0 || i >= N || j >= N) return 0;
  if (i >= n_valid || j >= n_valid) return 0;
  if (variant == S2O_DENSE_CAUSAL) return j <= i;
  if (head_class == 0) {
    /* N_0(i) = { j : G floor(i/G) <= j <= i } */
    return (j <= i) && (i / G == j / G);
  }
  int64_t s = G / 2;
  if (variant == S2O_STRICT) {
    /* b'(x) = floor((x - s)/G), no wrap: N_1(i) with short head/tail groups */
    return (j <= i) && (floor_div(i - s, G) == floor_div(j - s, G));
  }
  if (variant == S2O_ROLLED) {
    /* roll left by s, then the in-group triangular mask of the rolled order */
    int64_t ri = pos_mod(i - s, N), rj = pos_mod(j - s, N);
    return (ri / G == rj / G) && (rj <= ri);
  }
  return 0;
}

/* Explicit boolean matrix A (row-major N x N, 1 byte per entry). */
void s2o_adjacency(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class,
                   uint8_t* out) {
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < N; ++j)
      out[i * N + j] = (uint8_t)s2o_visible(N, G, n_valid, variant, head_class, i, j);
}

/* One row of A: out[j] = A[i][j] for j in [0, N). */
void s2o_adjacency_row(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class, int64_t i,
                       uint8_t* out) {
  for (int64_t j = 0; j < N; ++j) out[j] = (uint8_t)s2o_visible(N, G, n_valid, variant, head_class, i, j);
}

/* Number of visible (i, j) pairs, by enumeration. */
int64_t s2o_pair_count(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class) {
  int64_t c = 0;
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < N; ++j)
      c += s2o_visible(N, G, n_valid, variant, head_class, i, j);
  return c;
}

/* Number of visible (i, j) pairs under a document mask (doc: [N] IDs of one
 * batch row), by enumeration. */
int64_t s2o_pair_count_docs(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class,
                            const int32_t* doc) {
  int64_t c = 0;
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < N; ++j)
      c += s2o_visible(N, G, n_valid, variant, head_class, i, j) && doc[i] == doc[j];
  return c;
}

/* Explicit boolean matrix under a document mask (doc: [N] IDs of one batch
 * row): out[i*N + j] = A^(c)[i][j] and doc[i] == doc[j]. */
void s2o_adjacency_docs(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class,
                        const int32_t* doc, uint8_t* out) {
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < N; ++j)
      out[i * N + j] = (uint8_t)(s2o_visible(N, G, n_valid, variant, head_class, i, j) && doc[i] == doc[j]);
}

/* One row of the document-masked matrix: out[j] = A^(c)[i][j] and doc[i] == doc[j]. */
void s2o_adjacency_row_docs(int64_t N, int64_t G, int64_t n_valid, int variant, int head_class,
                            const int32_t* doc, int64_t i, uint8_t* out) {
  for (int64_t j = 0; j < N; ++j)
    out[j] = (uint8_t)(s2o_visible(N, G, n_valid, variant, head_class, i, j) && doc[i] == doc[j]);
}

/* bf16 bit pattern -> double (exact). */
static double bf16_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* element (b, i, h, d) of a [B, N, H, D] tensor */
static size_t at(int64_t N, int64_t H, int64_t D, int64_t b, int64_t i, int64_t h, int64_t d) {
  return (size_t)(((b * N + i) * H + h) * D + d);
}

/*
 * Masked softmax attention and its gradients over the visibility matrix.
 *
 *   q, k, v, dout : bf16 bit patterns, [B, N, H, D] contiguous.  dout may be
 *                   NULL, in which case only the forward is computed.
 *   rows          : query rows [row_begin, row_end) are processed.
 *   heads         : list of flattened (b*H + h) heads to process, or NULL for
 *                   all B*H heads.
 *   doc           : per-position document IDs [B, N], or NULL (one document).
 *   o, dq         : [B, N, H, D] float64, written for the processed rows.
 *   lse           : [B, H, N] float64, written for the processed rows.
 *   dk, dv        : [B, N, H, D] float64, ACCUMULATED (+=) with the
 *                   contributions of the processed rows; the caller zeroes
 *                   them.  With all rows processed they are the full
 *                   gradients.
 * Returns 0, or -1 on an invalid argument.
 *
 * Forward, per visible set S_i ([PT] §3):
 *   z_j = scale q_i·k_j,  m = max z,  l = sum exp(z_j - m),
 *   o_i = sum exp(z_j - m) v_j / l,  lse_i = m + ln l.
 * Backward ([PT] §3, dL/dz_j = a_j g^T (v_j - o_i) with g = dL/do_i):
 *   a_ij = exp(z_ij - lse_i),  Delta_i = g_i·o_i,
 *   dS_ij = a_ij (g_i·v_j - Delta_i) = dL/dz_ij,
 *   dq_i = scale sum_j dS_ij k_j,  dk_j += scale dS_ij q_i,  dv_j += a_ij g_i.
 */
int s2o_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                  const int32_t* doc, int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid,
                  int variant, int64_t row_begin, int64_t row_end,
                  const int64_t* heads, int64_t n_heads,
                  double* o, double* lse, double* dq, double* dk, double* dv) {
  if (B < 1 || N < 1 || H < 2 || D < 1 || G < 2 || (H % 2) || (G % 2) || (N % G)) return -1;
  if (n_valid < 0 || n_valid > N || row_begin < 0 || row_end > N || row_begin > row_end) return -1;
  if (variant < 0 || variant > 2) return -1;
  const double scale = 1.0 / sqrt((double)D);
  const int64_t nh = heads ? n_heads : B * H;

#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < nh; ++t) {
    const int64_t bh = heads ? heads[t] : t;
    const int64_t b = bh / H, h = bh % H;
    const int head_class = (h >= H / 2) ? 1 : 0;
    double* qi = (double*)malloc(sizeof(double) * D);
    double* gi = (double*)malloc(sizeof(double) * D);
    double* oi = (double*)malloc(sizeof(double) * D);
    double* dqi = (double*)malloc(sizeof(double) * D);
    double* z = (double*)malloc(sizeof(double) * N);
    int64_t* js = (int64_t*)malloc(sizeof(int64_t) * N);

    for (int64_t i = row_begin; i < row_end; ++i) {
      /* S_i: the visible keys of row i */
      int64_t ns = 0;
      for (int64_t j = 0; j < N; ++j)
        if (s2o_visible(N, G, n_valid, variant, head_class, i, j) && (!doc || doc[b * N + i] == doc[b * N + j]))
          js[ns++] = j;

      for (int64_t d = 0; d < D; ++d) qi[d] = bf16_to_double(q[at(N, H, D, b, i, h, d)]);

      if (ns == 0) { /* only rows i >= n_valid: empty set */
        for (int64_t d = 0; d < D; ++d) {
          o[at(N, H, D, b, i, h, d)] = 0.0;
          if (dout) dq[at(N, H, D, b, i, h, d)] = 0.0;
        }
        lse[(b * H + h) * N + i] = -INFINITY;
        continue;
      }

      double m = -INFINITY;
      for (int64_t t2 = 0; t2 < ns; ++t2) {
        const int64_t j = js[t2];
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += qi[d] * bf16_to_double(k[at(N, H, D, b, j, h, d)]);
        z[t2] = scale * acc;
        if (z[t2] > m) m = z[t2];
      }
      double l = 0.0;
      for (int64_t t2 = 0; t2 < ns; ++t2) l += exp(z[t2] - m);
      for (int64_t d = 0; d < D; ++d) oi[d] = 0.0;
      for (int64_t t2 = 0; t2 < ns; ++t2) {
        const double p = exp(z[t2] - m) / l;
        const int64_t j = js[t2];
        for (int64_t d = 0; d < D; ++d) oi[d] += p * bf16_to_double(v[at(N, H, D, b, j, h, d)]);
      }
      const double lse_i = m + log(l);
      for (int64_t d = 0; d < D; ++d) o[at(N, H, D, b, i, h, d)] = oi[d];
      lse[(b * H + h) * N + i] = lse_i;

      if (!dout) continue;
      /* loss mask: rows >= n_valid carry no gradient (they have ns == 0 anyway) */
      for (int64_t d = 0; d < D; ++d)
        gi[d] = (i < n_valid) ? bf16_to_double(dout[at(N, H, D, b, i, h, d)]) : 0.0;
      double delta = 0.0;
      for (int64_t d = 0; d < D; ++d) delta += gi[d] * oi[d];
      for (int64_t d = 0; d < D; ++d) dqi[d] = 0.0;
      for (int64_t t2 = 0; t2 < ns; ++t2) {
        const int64_t j = js[t2];
        const double a = exp(z[t2] - lse_i);
        double gv = 0.0;
        for (int64_t d = 0; d < D; ++d) gv += gi[d] * bf16_to_double(v[at(N, H, D, b, j, h, d)]);
        const double ds = a * (gv - delta);
        for (int64_t d = 0; d < D; ++d) {
          dqi[d] += scale * ds * bf16_to_double(k[at(N, H, D, b, j, h, d)]);
          dk[at(N, H, D, b, j, h, d)] += scale * ds * qi[d];
          dv[at(N, H, D, b, j, h, d)] += a * gi[d];
        }
      }
      for (int64_t d = 0; d < D; ++d) dq[at(N, H, D, b, i, h, d)] = dqi[d];
    }
    free(qi); free(gi); free(oi); free(dqi); free(z); free(js);
  }
  return 0;
}

/*
 * The same computation on a window of query rows [r0, r1) of selected heads,
 * with compact outputs (for large inputs whose full-size float64 outputs
 * would not fit in memory):
 *   o_w, dq_w  [n_heads][r1 - r0][D]   rows r0..r1-1
 *   lse_w      [n_heads][r1 - r0]
 *   dk_w, dv_w [n_heads][r1 - r0][D]   keys r0..r1-1, ACCUMULATED from the
 *              window's rows only (exact for keys whose visible-from rows
 *              all lie inside the window; the caller zeroes them)
 * heads: flattened (b*H + h) list.  dout may be NULL (forward only); doc as
 * for s2o_attention.
 */
int s2o_attention_window(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                         const int32_t* doc, int64_t B, int64_t N, int64_t H, int64_t D, int64_t G, int64_t n_valid,
                         int variant, int64_t r0, int64_t r1, const int64_t* heads, int64_t n_heads,
                         double* o_w, double* lse_w, double* dq_w, double* dk_w, double* dv_w) {
  if (B < 1 || N < 1 || H < 2 || D < 1 || G < 2 || (H % 2) || (G % 2) || (N % G)) return -1;
  if (n_valid < 0 || n_valid > N || r0 < 0 || r1 > N || r0 > r1 || !heads) return -1;
  if (variant < 0 || variant > 2) return -1;
  const double scale = 1.0 / sqrt((double)D);
  const int64_t W = r1 - r0;

#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < n_heads; ++t) {
    const int64_t bh = heads[t];
    const int64_t b = bh / H, h = bh % H;
    const int head_class = (h >= H / 2) ? 1 : 0;
    double* qi = (double*)malloc(sizeof(double) * D);
    double* gi = (double*)malloc(sizeof(double) * D);
    double* oi = (double*)malloc(sizeof(double) * D);
    double* dqi = (double*)malloc(sizeof(double) * D);
    double* z = (double*)malloc(sizeof(double) * N);
    int64_t* js = (int64_t*)malloc(sizeof(int64_t) * N);
    for (int64_t i = r0; i < r1; ++i) {
      const size_t wi = (size_t)(t * W + (i - r0));
      int64_t ns = 0;
      for (int64_t j = 0; j < N; ++j)
        if (s2o_visible(N, G, n_valid, variant, head_class, i, j) && (!doc || doc[b * N + i] == doc[b * N + j]))
          js[ns++] = j;
      for (int64_t d = 0; d < D; ++d) qi[d] = bf16_to_double(q[at(N, H, D, b, i, h, d)]);
      if (ns == 0) {
        for (int64_t d = 0; d < D; ++d) {
          o_w[wi * D + d] = 0.0;
          if (dout) dq_w[wi * D + d] = 0.0;
        }
        lse_w[wi] = -INFINITY;
        continue;
      }
      double m = -INFINITY;
      for (int64_t t2 = 0; t2 < ns; ++t2) {
        const int64_t j = js[t2];
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += qi[d] * bf16_to_double(k[at(N, H, D, b, j, h, d)]);
        z[t2] = scale * acc;
        if (z[t2] > m) m = z[t2];
      }
      double l = 0.0;
      for (int64_t t2 = 0; t2 < ns; ++t2) l += exp(z[t2] - m);
      for (int64_t d = 0; d < D; ++d) oi[d] = 0.0;
      for (int64_t t2 = 0; t2 < ns; ++t2) {
        const double p = exp(z[t2] - m) / l;
        const int64_t j = js[t2];
        for (int64_t d = 0; d < D; ++d) oi[d] += p * bf16_to_double(v[at(N, H, D, b, j, h, d)]);
      }
      const double lse_i = m + log(l);
      for (int64_t d = 0; d < D; ++d) o_w[wi * D + d] = oi[d];
      lse_w[wi] = lse_i;
      if (!dout) continue;
      for (int64_t d = 0; d < D; ++d)
        gi[d] = (i < n_valid) ? bf16_to_double(dout[at(N, H, D, b, i, h, d)]) : 0.0;
      double delta = 0.0;
      for (int64_t d = 0; d < D; ++d) delta += gi[d] * oi[d];
      for (int64_t d = 0; d < D; ++d) dqi[d] = 0.0;
      for (int64_t t2 = 0; t2 < ns; ++t2) {
        const int64_t j = js[t2];
        const double a = exp(z[t2] - lse_i);
        double gv = 0.0;
        for (int64_t d = 0; d < D; ++d) gv += gi[d] * bf16_to_double(v[at(N, H, D, b, j, h, d)]);
        const double ds = a * (gv - delta);
        const int in_window = (j >= r0 && j < r1);
        const size_t wj = (size_t)(t * W + (j - r0));
        for (int64_t d = 0; d < D; ++d) {
          dqi[d] += scale * ds * bf16_to_double(k[at(N, H, D, b, j, h, d)]);
          if (in_window) {
            dk_w[wj * D + d] += scale * ds * qi[d];
            dv_w[wj * D + d] += a * gi[d];
          }
        }
      }
      for (int64_t d = 0; d < D; ++d) dq_w[wi * D + d] = dqi[d];
    }
    free(qi); free(gi); free(oi); free(dqi); free(z); free(js);
  }
  return 0;
}

/* Number of threads the OpenMP runtime will use for s2o_attention. */
int s2o_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
