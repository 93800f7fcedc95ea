/*
 * attn_oracle.c -- fp64 CPU oracle for the fused attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the tests, the package's smoke check and the bench's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA path.
 *
 * What it computes.  The PipeThreader pages (papers.lqhl.me
 * "PipeThreader-OSDI25", "实验与结果", paper Sec. 6.2 / Fig. 12) evaluate a
 * FlashAttention forward on LLaMA3-8B/70B head shapes, SEQ 512-8k, BS 1/64,
 * but never write the operator down.  The fused kernel reaches exactly (up to
 * rounding order) the plain definition of scaled dot-product attention, so the
 * oracle is that definition written out, in fp64, with no tiling, no online
 * rescaling and no fusion:
 *
 *   g       = hq / (Hq / Hkv)                  grouped-query head -> kv head
 *   s_ij    = (sum_d Q[b,hq,i,d] * K[b,g,j,d]) / sqrt(D)       j in A(i)
 *   A(i)    = {0..i} when causal, else {0..S-1}
 *   m_i     = max_{j in A(i)} s_ij
 *   l_i     = sum_{j in A(i)} exp(s_ij - m_i)
 *   P_ij    = exp(s_ij - m_i) / l_i
 *   O[..,i,d] = sum_{j in A(i)} P_ij * V[b,g,j,d]
 *   LSE[..,i] = m_i + ln(l_i)     (natural log of the sum of exp of the
 *                                  scaled logits)
 *
 * Layout: Q, O are [B, Hq, S, D]; K, V are [B, Hkv, S, D]; LSE is [B, Hq, S];
 * all dense, row-major, fp64.  The *_qk_* functions at the end take Sq query
 * rows over Sk keys, with the causal window aligned at the bottom right.  Every function returns 0 on success and a
 * negative value on a bad argument; it never aborts.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

/*
 * Probabilities of one query row: P[j] for j in [0, S), zero outside A(i).
 * q: [D]; k: [S, D] (the kv head's keys); i: the query position.
 */
int oracle_attn_probs_row_f64(const double* q, const double* k, int64_t i,
                              int64_t S, int64_t D, int causal, double* p_out,
                              double* lse_out) {
  if (!q || !k || !p_out || D <= 0 || S <= 0 || i < 0 || i >= S) return -1;
  const double inv_sqrt_d = 1.0 / sqrt((double)D);
  const int64_t n_keys = causal ? i + 1 : S; /* A(i) = {0 .. n_keys-1} */

  /* pass 1: logits and their maximum */
  double m = -INFINITY;
  for (int64_t j = 0; j < S; ++j) {
    if (j >= n_keys) { p_out[j] = 0.0; continue; }
    double dot = 0.0;
    for (int64_t d = 0; d < D; ++d) dot += q[d] * k[j * D + d];
    p_out[j] = dot * inv_sqrt_d;
    if (p_out[j] > m) m = p_out[j];
  }
  /* pass 2: exponentials, their sum, normalisation */
  double l = 0.0;
  for (int64_t j = 0; j < n_keys; ++j) {
    p_out[j] = exp(p_out[j] - m);
    l += p_out[j];
  }
  for (int64_t j = 0; j < n_keys; ++j) p_out[j] /= l;
  if (lse_out) *lse_out = m + log(l);
  return 0;
}

/*
 * One query row of the output: o[D] and its LSE, from the row's probabilities.
 * scratch: caller-provided [S] doubles.
 */
int oracle_attn_row_f64(const double* q, const double* k, const double* v,
                        int64_t i, int64_t S, int64_t D, int causal,
                        double* o, double* lse, double* scratch) {
  if (!v || !o || !scratch) return -1;
  int rc = oracle_attn_probs_row_f64(q, k, i, S, D, causal, scratch, lse);
  if (rc) return rc;
  const int64_t n_keys = causal ? i + 1 : S;
  for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
  for (int64_t j = 0; j < n_keys; ++j) {
    const double pj = scratch[j];
    for (int64_t d = 0; d < D; ++d) o[d] += pj * v[j * D + d];
  }
  return 0;
}

/*
 * Selected rows of one (b, hq) head.  q_rows: [n, D] query vectors,
 * pos: [n] their positions i; k, v: [S, D] of kv head g.  Rows are
 * independent, so a sampled row is an exact check of that row.
 * Threads: OpenMP over rows when compiled with it.
 */
int oracle_attn_rows_f64(const double* q_rows, const int64_t* pos, int64_t n,
                         const double* k, const double* v, int64_t S,
                         int64_t D, int causal, double* o, double* lse) {
  if (!q_rows || !pos || !k || !v || !o || !lse || n < 0 || S <= 0 || D <= 0)
    return -1;
  for (int64_t r = 0; r < n; ++r)
    if (pos[r] < 0 || pos[r] >= S) return -2;
  int bad = 0;
#pragma omp parallel
  {
    double* scratch = (double*)malloc(sizeof(double) * (size_t)S);
    if (!scratch) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(dynamic, 4)
      for (int64_t r = 0; r < n; ++r) {
        if (oracle_attn_row_f64(q_rows + r * D, k, v, pos[r], S, D, causal,
                                o + r * D, lse + r, scratch)) {
#pragma omp atomic write
          bad = 1;
        }
      }
      free(scratch);
    }
  }
  return bad ? -3 : 0;
}

/*
 * Whole tensors: every (b, hq, i).  The kv head of query head hq is
 * g = hq / (Hq / Hkv) (contiguous groups of Hq/Hkv query heads share one kv
 * head).
 */
int oracle_attn_fwd_f64(const double* q, const double* k, const double* v,
                        double* o, double* lse, int64_t B, int64_t Hq,
                        int64_t Hkv, int64_t S, int64_t D, int causal) {
  if (!q || !k || !v || !o || !lse) return -1;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || S <= 0 || D <= 0) return -1;
  if (Hq % Hkv != 0) return -2;
  const int64_t group = Hq / Hkv;
  int bad = 0;
#pragma omp parallel
  {
    double* scratch = (double*)malloc(sizeof(double) * (size_t)S);
    if (!scratch) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for collapse(3) schedule(dynamic, 16)
      for (int64_t b = 0; b < B; ++b)
        for (int64_t hq = 0; hq < Hq; ++hq)
          for (int64_t i = 0; i < S; ++i) {
            const int64_t g = hq / group;
            const double* kh = k + ((b * Hkv + g) * S) * D;
            const double* vh = v + ((b * Hkv + g) * S) * D;
            const int64_t row = (b * Hq + hq) * S + i;
            if (oracle_attn_row_f64(q + row * D, kh, vh, i, S, D, causal,
                                    o + row * D, lse + row, scratch)) {
#pragma omp atomic write
              bad = 1;
            }
          }
      free(scratch);
    }
  }
  return bad ? -3 : 0;
}

/*
 * Different query and key lengths: Sq query rows over Sk keys.  The causal
 * window is aligned at the bottom right -- query i sees keys
 * j <= i + (Sk - Sq) -- so the last query sees every key, and Sq == Sk is the
 * square case above.  A causal query with no visible key (Sq > Sk and
 * i < Sq - Sk) is rejected (-4): softmax over an empty set is undefined.
 * Layout: Q, O [B, Hq, Sq, D]; K, V [B, Hkv, Sk, D]; LSE [B, Hq, Sq].
 */
static int64_t qk_visible_keys(int64_t i, int64_t Sq, int64_t Sk, int causal) {
  if (!causal) return Sk;
  const int64_t last = i + (Sk - Sq); /* the last visible key */
  return last + 1 < Sk ? last + 1 : Sk;
}

/*
 * One query row i of a head: o[D] and its LSE.  k, v: [Sk, D] of the kv
 * head; scratch: caller-provided [Sk] doubles.
 */
int oracle_attn_row_qk_f64(const double* q, const double* k, const double* v,
                           int64_t i, int64_t Sq, int64_t Sk, int64_t D,
                           int causal, double* o, double* lse,
                           double* scratch) {
  if (!q || !k || !v || !o || !lse || !scratch) return -1;
  if (D <= 0 || Sq <= 0 || Sk <= 0 || i < 0 || i >= Sq) return -1;
  const int64_t nk = qk_visible_keys(i, Sq, Sk, causal);
  if (nk < 1) return -4;
  const double scale = pow((double)D, -0.5);
  /* pass 1: the scaled logits of the visible keys, and their maximum */
  double mx = -INFINITY;
  for (int64_t j = 0; j < nk; ++j) {
    double acc = 0.0;
    for (int64_t d = 0; d < D; ++d) acc += q[d] * k[D * j + d];
    scratch[j] = acc * scale;
    if (scratch[j] > mx) mx = scratch[j];
  }
  /* pass 2: weights exp(s - max), their sum, and the weighted values */
  double sum = 0.0;
  for (int64_t j = 0; j < nk; ++j) {
    scratch[j] = exp(scratch[j] - mx);
    sum += scratch[j];
  }
  for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
  for (int64_t j = 0; j < nk; ++j)
    for (int64_t d = 0; d < D; ++d) o[d] += scratch[j] * v[D * j + d];
  for (int64_t d = 0; d < D; ++d) o[d] /= sum;
  *lse = mx + log(sum);
  return 0;
}

/* Selected rows of one head (positions pos[n] in [0, Sq)). */
int oracle_attn_rows_qk_f64(const double* q_rows, const int64_t* pos, int64_t n,
                            const double* k, const double* v, int64_t Sq,
                            int64_t Sk, int64_t D, int causal, double* o,
                            double* lse) {
  if (!q_rows || !pos || !k || !v || !o || !lse || n < 0 || Sq <= 0 || Sk <= 0 ||
      D <= 0)
    return -1;
  for (int64_t r = 0; r < n; ++r)
    if (pos[r] < 0 || pos[r] >= Sq) return -2;
  int bad = 0;
#pragma omp parallel
  {
    double* scratch = (double*)malloc(sizeof(double) * (size_t)Sk);
    if (!scratch) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(dynamic, 4)
      for (int64_t r = 0; r < n; ++r) {
        const int rc = oracle_attn_row_qk_f64(q_rows + r * D, k, v, pos[r], Sq, Sk, D,
                                              causal, o + r * D, lse + r, scratch);
        if (rc) {
#pragma omp atomic write
          bad = rc;
        }
      }
      free(scratch);
    }
  }
  return bad ? (bad < 0 ? bad : -3) : 0;
}

/* Whole tensors, every (b, hq, i); kv head g = hq / (Hq / Hkv). */
int oracle_attn_fwd_qk_f64(const double* q, const double* k, const double* v,
                           double* o, double* lse, int64_t B, int64_t Hq,
                           int64_t Hkv, int64_t Sq, int64_t Sk, int64_t D,
                           int causal) {
  if (!q || !k || !v || !o || !lse) return -1;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Sk <= 0 || D <= 0) return -1;
  if (Hq % Hkv != 0) return -2;
  if (causal && Sq > Sk) return -4;
  const int64_t heads_per_kv = Hq / Hkv;
  int bad = 0;
#pragma omp parallel
  {
    double* scratch = (double*)malloc(sizeof(double) * (size_t)Sk);
    if (!scratch) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for collapse(3) schedule(dynamic, 16)
      for (int64_t b = 0; b < B; ++b)
        for (int64_t hq = 0; hq < Hq; ++hq)
          for (int64_t i = 0; i < Sq; ++i) {
            const int64_t kvh = b * Hkv + hq / heads_per_kv;
            const int64_t row = (b * Hq + hq) * Sq + i;
            if (oracle_attn_row_qk_f64(q + row * D, k + kvh * Sk * D, v + kvh * Sk * D, i, Sq,
                                       Sk, D, causal, o + row * D, lse + row, scratch)) {
#pragma omp atomic write
              bad = 1;
            }
          }
      free(scratch);
    }
  }
  return bad ? -3 : 0;
}

/* Threads the OpenMP runtime will use (1 when built without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
