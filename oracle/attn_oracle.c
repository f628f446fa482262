/*
 * Test infrastructure only: the fp64 CPU oracle for segment-masked
 * multi-head softmax attention (bidirectional, with an optional causal limit
 * or 3D neighbourhood window, both described below).  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg load this file's library; the product
 * path never calls it, and it shares no code with the CUDA library.
 *
 * What it computes (vidax: A Unified JAX Framework for Video Generative Models
 * on Accelerator Meshes, §2 "3D RoPE, 3D VAEs, and flash attention": exact
 * attention whose query-key matrix is never stored; Appendix A, Table 4, group
 * 2 "Sharding, Parallelism & Custom Kernels", row "HunyuanVideo-1.5:
 * RESOURCE_EXHAUSTED at 720p": segment ids instead of a dense (B,H,Sq,Sk)
 * mask).  Flash attention (reference [2] of that paper) reaches the plain
 * softmax-attention result exactly up to rounding order, so this oracle is
 * that plain definition written out, row by row:
 *
 *   A_i   = { j : 0 <= j < S_kv and seg_q[b,i] == seg_kv[b,j] }  (all j when no ids)
 *   s_ij  = scale * sum_d q[b,h,i,d] * k[b,h,j,d]
 *   m_i   = max_{j in A_i} s_ij
 *   l_i   = sum_{j in A_i} exp(s_ij - m_i)
 *   out_i = sum_{j in A_i} exp(s_ij - m_i) * v[b,h,j,:] / l_i
 *   lse_i = m_i + ln(l_i)                 (natural log of sum exp(s_ij))
 *   A_i empty  =>  out_i = 0, lse_i = -inf
 *
 * Inputs are bf16 bit patterns (uint16); each is widened exactly to double.
 * Everything after that is double precision, in the order written above.
 * Subtracting m_i only keeps exp() in range; it does not change the result.
 *
 * Readings taken where the pages are silent: a query sees a key iff their
 * segment ids are equal; a row that sees no key gets out = 0 and lse = -inf;
 * lse is the natural log over the scaled logits of the allowed keys.
 *
 * Causal variant (same paper, §3.1, Cosmos paragraph: a backbone whose
 * "understanding" pathway attends causally): with causal != 0 a key is
 * allowed only if, in addition, j <= i + (S_kv - S_q), i.e. query i sees
 * the keys up to its own position, the last query aligned with the last
 * key.  The set A_i above gains this condition; nothing else changes.
 *
 * Windowed variant (same paper, Appendix A, Table 4, group 4 "Memory, Tiling
 * & Execution Graphs", rows on the LTX-2.5 VAE decoder: 3D neighbourhood
 * attention with an 11 x 11 x 11 window; the paper gives no formula).  Each
 * token carries (t, h, w) coordinates in a T x Hg x Wg volume, packed as
 * t << 22 | h << 11 | w.  On each axis, a window of odd size k starts at
 * c - (k - 1) / 2 for a query at coordinate c (centred; keys outside the
 * volume do not exist), or, "clamped", at that start pushed into
 * [0, extent - k], so that a query near a border still sees k keys on that
 * axis (the neighbourhood attention of Hassani et al., "Neighborhood
 * Attention Transformer", CVPR 2023).  Key j is in query i's window iff, on
 * every axis, start <= c_j <= start + k - 1.  The set A_i gains this
 * condition; nothing else changes.
 *
 * Parallelism: OpenMP over independent rows only; the arithmetic of a row is
 * the serial loop above.  Build without -ffast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* exact widening of a bf16 bit pattern: bf16 is the top half of an fp32 */
static double bf16_bits_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* A 3D neighbourhood window: per-token packed coordinates ([B,S_q] and
 * [B,S_kv]), the window size and the volume extent on each axis (t, h, w). */
struct window3 {
  const int32_t* coord_q;
  const int32_t* coord_kv;
  long size[3];
  long extent[3];
  int clamped;
};

static void unpack_coord(int32_t packed, long c[3]) {
  uint32_t u = (uint32_t)packed;
  c[0] = (long)(u >> 22);
  c[1] = (long)((u >> 11) & 2047u);
  c[2] = (long)(u & 2047u);
}

/* First coordinate of the window of a query at c, on one axis. */
static long window_start(long c, long size, long extent, int clamped) {
  long start = c - (size - 1) / 2;
  if (clamped) {
    if (start > extent - size) start = extent - size;
    if (start < 0) start = 0;
  }
  return start;
}

static int in_window(const struct window3* w, long S_q, long S_kv, long b, long i, long j) {
  long cq[3], ck[3];
  unpack_coord(w->coord_q[b * S_q + i], cq);
  unpack_coord(w->coord_kv[b * S_kv + j], ck);
  for (int a = 0; a < 3; ++a) {
    long start = window_start(cq[a], w->size[a], w->extent[a], w->clamped);
    if (ck[a] < start || ck[a] > start + w->size[a] - 1) return 0;
  }
  return 1;
}

/* Is key j visible to query i?  (segment equality; causal limit; window) */
static int key_allowed(const int32_t* seg_q, const int32_t* seg_kv, long S_q, long S_kv,
                       long b, long i, long j, int causal, const struct window3* win) {
  if (seg_q != NULL && seg_kv[b * S_kv + j] != seg_q[b * S_q + i]) return 0;
  if (causal && j > i + (S_kv - S_q)) return 0;
  if (win != NULL && !in_window(win, S_q, S_kv, b, i, j)) return 0;
  return 1;
}

/* One output row (b, h, i).  s_scratch holds S_kv doubles. */
static void oracle_row(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       const int32_t* seg_q, const int32_t* seg_kv,
                       long H, long S_q, long S_kv, long D, double scale, int causal,
                       const struct window3* win, long b, long h, long i, double* s_scratch,
                       double* out_row, double* lse_out) {
  const uint16_t* qi = q + ((b * H + h) * S_q + i) * D;
  const uint16_t* kb = k + (b * H + h) * S_kv * D;
  const uint16_t* vb = v + (b * H + h) * S_kv * D;

  /* scores of the allowed keys, and their maximum */
  double m = -INFINITY;
  long n_allowed = 0;
  for (long j = 0; j < S_kv; ++j) {
    int allowed = key_allowed(seg_q, seg_kv, S_q, S_kv, b, i, j, causal, win);
    if (!allowed) { s_scratch[j] = NAN; continue; }
    double dot = 0.0;
    for (long d = 0; d < D; ++d)
      dot += bf16_bits_to_double(qi[d]) * bf16_bits_to_double(kb[j * D + d]);
    double s = scale * dot;
    s_scratch[j] = s;
    if (s > m) m = s;
    ++n_allowed;
  }

  for (long d = 0; d < D; ++d) out_row[d] = 0.0;
  if (n_allowed == 0) {       /* nothing to attend to */
    *lse_out = -INFINITY;
    return;
  }

  /* softmax weights, their sum, and the weighted sum of values */
  double l = 0.0;
  for (long j = 0; j < S_kv; ++j) {
    int allowed = key_allowed(seg_q, seg_kv, S_q, S_kv, b, i, j, causal, win);
    if (!allowed) continue;
    double e = exp(s_scratch[j] - m);
    l += e;
    for (long d = 0; d < D; ++d)
      out_row[d] += e * bf16_bits_to_double(vb[j * D + d]);
  }
  for (long d = 0; d < D; ++d) out_row[d] /= l;
  *lse_out = m + log(l);
}

static int check_shape(long B, long H, long S_q, long S_kv, long D) {
  if (B < 0 || H < 0 || S_q < 0 || S_kv < 0 || D <= 0) return 1;
  return 0;
}

/* Window arguments of the exported functions: coord_q/coord_kv both set,
 * sizes odd and >= 1, extents >= 1.  Returns 0, or 1 on bad arguments. */
static int make_window(const int32_t* coord_q, const int32_t* coord_kv, const long* size,
                       const long* extent, int clamped, struct window3* w) {
  if (coord_q == NULL || coord_kv == NULL || size == NULL || extent == NULL) return 1;
  w->coord_q = coord_q;
  w->coord_kv = coord_kv;
  w->clamped = clamped;
  for (int a = 0; a < 3; ++a) {
    if (size[a] < 1 || size[a] % 2 == 0 || extent[a] < 1) return 1;
    w->size[a] = size[a];
    w->extent[a] = extent[a];
  }
  return 0;
}

static int fwd_impl(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    const int32_t* seg_q, const int32_t* seg_kv,
                    double* out, double* lse,
                    long B, long H, long S_q, long S_kv, long D,
                    double scale, int causal, const struct window3* win, int nthreads) {
  if (check_shape(B, H, S_q, S_kv, D)) return 1;
  if ((seg_q == NULL) != (seg_kv == NULL)) return 1;
  long n_rows = B * H * S_q;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int failed = 0;
#pragma omp parallel
  {
    double* s_scratch = (double*)malloc(sizeof(double) * (size_t)(S_kv > 0 ? S_kv : 1));
    if (!s_scratch) {
#pragma omp atomic write
      failed = 1;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (long r = 0; r < n_rows; ++r) {
        long i = r % S_q;
        long h = (r / S_q) % H;
        long b = r / (S_q * H);
        oracle_row(q, k, v, seg_q, seg_kv, H, S_q, S_kv, D, scale, causal, win, b, h, i,
                   s_scratch, out + r * D, lse + r);
      }
      free(s_scratch);
    }
  }
  return failed ? 2 : 0;
}

/* All rows.  out: double[B,H,S_q,D]; lse: double[B,H,S_q].
 * seg_q and seg_kv: int32 [B,S_q] and [B,S_kv], or both NULL (one segment).
 * nthreads <= 0 uses the OpenMP default.  Returns 0, or 1 on bad arguments. */
int oracle_attn_fwd_f64(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const int32_t* seg_q, const int32_t* seg_kv,
                        double* out, double* lse,
                        long B, long H, long S_q, long S_kv, long D,
                        double scale, int causal, int nthreads) {
  return fwd_impl(q, k, v, seg_q, seg_kv, out, lse, B, H, S_q, S_kv, D, scale, causal, NULL,
                  nthreads);
}

/* All rows with a 3D neighbourhood window (coord_* int32 [B,S], packed
 * t << 22 | h << 11 | w; size[3], extent[3] per axis t, h, w). */
int oracle_attn_win_fwd_f64(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            const int32_t* seg_q, const int32_t* seg_kv,
                            const int32_t* coord_q, const int32_t* coord_kv,
                            const long* size, const long* extent, int clamped,
                            double* out, double* lse,
                            long B, long H, long S_q, long S_kv, long D,
                            double scale, int causal, int nthreads) {
  struct window3 w;
  if (make_window(coord_q, coord_kv, size, extent, clamped, &w)) return 1;
  return fwd_impl(q, k, v, seg_q, seg_kv, out, lse, B, H, S_q, S_kv, D, scale, causal, &w,
                  nthreads);
}

static int rows_impl(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const int32_t* seg_q, const int32_t* seg_kv,
                     const int64_t* rows, long n_rows,
                     double* out_rows, double* lse_rows,
                     long B, long H, long S_q, long S_kv, long D,
                     double scale, int causal, const struct window3* win, int nthreads) {
  if (check_shape(B, H, S_q, S_kv, D) || n_rows < 0) return 1;
  if ((seg_q == NULL) != (seg_kv == NULL)) return 1;
  for (long r = 0; r < n_rows; ++r) {
    if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 ||
        rows[3 * r + 1] >= H || rows[3 * r + 2] < 0 || rows[3 * r + 2] >= S_q)
      return 1;
  }
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int failed = 0;
#pragma omp parallel
  {
    double* s_scratch = (double*)malloc(sizeof(double) * (size_t)(S_kv > 0 ? S_kv : 1));
    if (!s_scratch) {
#pragma omp atomic write
      failed = 1;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (long r = 0; r < n_rows; ++r)
        oracle_row(q, k, v, seg_q, seg_kv, H, S_q, S_kv, D, scale, causal, win,
                   rows[3 * r], rows[3 * r + 1], rows[3 * r + 2], s_scratch,
                   out_rows + r * D, lse_rows + r);
      free(s_scratch);
    }
  }
  return failed ? 2 : 0;
}

/* Selected rows only.  rows: int64[n_rows][3] = (b, h, i).
 * out_rows: double[n_rows, D]; lse_rows: double[n_rows]. */
int oracle_attn_rows_f64(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const int32_t* seg_q, const int32_t* seg_kv,
                         const int64_t* rows, long n_rows,
                         double* out_rows, double* lse_rows,
                         long B, long H, long S_q, long S_kv, long D,
                         double scale, int causal, int nthreads) {
  return rows_impl(q, k, v, seg_q, seg_kv, rows, n_rows, out_rows, lse_rows, B, H, S_q, S_kv,
                   D, scale, causal, NULL, nthreads);
}

/* Selected rows with a 3D neighbourhood window. */
int oracle_attn_win_rows_f64(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const int32_t* seg_q, const int32_t* seg_kv,
                             const int32_t* coord_q, const int32_t* coord_kv,
                             const long* size, const long* extent, int clamped,
                             const int64_t* rows, long n_rows,
                             double* out_rows, double* lse_rows,
                             long B, long H, long S_q, long S_kv, long D,
                             double scale, int causal, int nthreads) {
  struct window3 w;
  if (make_window(coord_q, coord_kv, size, extent, clamped, &w)) return 1;
  return rows_impl(q, k, v, seg_q, seg_kv, rows, n_rows, out_rows, lse_rows, B, H, S_q, S_kv,
                   D, scale, causal, &w, nthreads);
}

static int probs_impl(const uint16_t* q, const uint16_t* k,
                      const int32_t* seg_q, const int32_t* seg_kv,
                      double* probs,
                      long B, long H, long S_q, long S_kv, long D, double scale,
                      int causal, const struct window3* win) {
  if (check_shape(B, H, S_q, S_kv, D)) return 1;
  if ((seg_q == NULL) != (seg_kv == NULL)) return 1;
  for (long b = 0; b < B; ++b)
    for (long h = 0; h < H; ++h)
      for (long i = 0; i < S_q; ++i) {
        const uint16_t* qi = q + ((b * H + h) * S_q + i) * D;
        const uint16_t* kb = k + (b * H + h) * S_kv * D;
        double* prow = probs + ((b * H + h) * S_q + i) * S_kv;
        double m = -INFINITY;
        for (long j = 0; j < S_kv; ++j) {
          int allowed = key_allowed(seg_q, seg_kv, S_q, S_kv, b, i, j, causal, win);
          if (!allowed) { prow[j] = -INFINITY; continue; }
          double dot = 0.0;
          for (long d = 0; d < D; ++d)
            dot += bf16_bits_to_double(qi[d]) * bf16_bits_to_double(kb[j * D + d]);
          prow[j] = scale * dot;
          if (prow[j] > m) m = prow[j];
        }
        if (m == -INFINITY) {
          for (long j = 0; j < S_kv; ++j) prow[j] = 0.0;
          continue;
        }
        double l = 0.0;
        for (long j = 0; j < S_kv; ++j)
          if (prow[j] != -INFINITY) l += exp(prow[j] - m);
        for (long j = 0; j < S_kv; ++j)
          prow[j] = (prow[j] == -INFINITY) ? 0.0 : exp(prow[j] - m) / l;
      }
  return 0;
}

/* Softmax weights P[b,h,i,j] = exp(s_ij - lse_i) for allowed j, 0 elsewhere.
 * For small inputs only (the result is B*H*S_q*S_kv doubles).  A row that sees
 * no key is all zeros.  Used by the tests to check that each row sums to 1. */
int oracle_attn_probs_f64(const uint16_t* q, const uint16_t* k,
                          const int32_t* seg_q, const int32_t* seg_kv,
                          double* probs,
                          long B, long H, long S_q, long S_kv, long D, double scale,
                          int causal) {
  return probs_impl(q, k, seg_q, seg_kv, probs, B, H, S_q, S_kv, D, scale, causal, NULL);
}

/* Softmax weights with a 3D neighbourhood window. */
int oracle_attn_win_probs_f64(const uint16_t* q, const uint16_t* k,
                              const int32_t* seg_q, const int32_t* seg_kv,
                              const int32_t* coord_q, const int32_t* coord_kv,
                              const long* size, const long* extent, int clamped,
                              double* probs,
                              long B, long H, long S_q, long S_kv, long D, double scale,
                              int causal) {
  struct window3 w;
  if (make_window(coord_q, coord_kv, size, extent, clamped, &w)) return 1;
  return probs_impl(q, k, seg_q, seg_kv, probs, B, H, S_q, S_kv, D, scale, causal, &w);
}
