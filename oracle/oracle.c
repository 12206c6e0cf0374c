/*
 * oracle.c -- plain, slow, float64 CPU reference for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the smoke check and the bench's CPU-baseline
 * leg use it.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (sources are the pages on exact IO-aware attention):
 *  - attention forward: O = softmax(scale * Q K^T) V with a per-row natural-log
 *    logsumexp.  The defining formula softmax(QK^T/sqrt(d_k))V is stated in
 *    "flash-attention-trading-models" (section "Por que la atencion esta ligada
 *    a la memoria") and in "FlashAttention (IT)" (section "Problematica
 *    dell'attention standard").  Each score row is materialised in full and the
 *    softmax takes two passes (max, then exp/sum): no tiling, no online update.
 *    Causal masking (a query attends to keys at or before its own position) is
 *    from "flash-attention-trading-models", section on causal masking.
 *  - attention backward: the derivatives of that definition, taken row by row:
 *    dV = P^T dO, dP = dO V^T, dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik),
 *    dQ = scale dS K, dK = scale dS^T Q.  The pages only say that the backward
 *    pass recomputes the scores ("Pase hacia atras"); the calculus is standard.
 *  - FP8 P-cast forward emulation ("P-Cast precision in FP8 attention", sections
 *    1-2): scores in float64 over key tiles of width Bc visited forward or in
 *    reverse, running max including the current tile, p = exp(s - m),
 *    P' = E4M3(S * p) (round to nearest even, saturating at 448), the running
 *    sum l taken from the unquantised p, accumulators rescaled by exp(m_old-m_new),
 *    and O = acc / (S * l) at the end.  It also counts how many P' flushed to
 *    zero, split into sink keys (index < n_sink) and the rest.
 *  - E4M3 rounding: 4 exponent bits (bias 7), 3 mantissa bits, subnormals down
 *    to 2^-9, largest finite 448, no infinities (same page, sections 1-2).
 *
 * All index arithmetic is on contiguous [B, H, N, d] row-major arrays.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* E4M3 (the "fn" variant: no infinities, 448 is the largest finite value)    */
/* ------------------------------------------------------------------------- */
double oracle_e4m3(double x) {
  if (x != x) return x;
  double a = fabs(x);
  double sgn = x < 0 ? -1.0 : 1.0;
  if (a == 0.0) return 0.0 * sgn;
  if (a >= 448.0) return sgn * 448.0; /* saturate to the largest finite value */
  int e;
  frexp(a, &e);             /* a = f * 2^e, f in [0.5, 1)  =>  binade 2^(e-1) */
  int binade = e - 1;
  if (binade < -6) binade = -6; /* below the smallest normal the step stays 2^-9 */
  double quantum = ldexp(1.0, binade - 3); /* 3 mantissa bits */
  double q = nearbyint(a / quantum) * quantum; /* default rounding: nearest, ties to even */
  if (q > 448.0) q = 448.0;
  return sgn * q;
}

void oracle_e4m3_array(const double* x, double* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = oracle_e4m3(x[i]);
}

/* ------------------------------------------------------------------------- */
/* Forward: one query row, two-pass softmax over the materialised score row   */
/* ------------------------------------------------------------------------- */
static void fwd_row(const double* q_i, const double* K, const double* V, int N, int d, int nkeys, double scale,
                    double* s /* scratch, N */, double* o_i, double* lse_i) {
  double m = -INFINITY;
  for (int j = 0; j < nkeys; ++j) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += q_i[c] * K[(int64_t)j * d + c];
    s[j] = scale * acc;
    if (s[j] > m) m = s[j];
  }
  double sum = 0.0;
  for (int j = 0; j < nkeys; ++j) {
    s[j] = exp(s[j] - m);
    sum += s[j];
  }
  for (int c = 0; c < d; ++c) o_i[c] = 0.0;
  for (int j = 0; j < nkeys; ++j) {
    const double p = s[j] / sum;
    const double* v_j = V + (int64_t)j * d;
    for (int c = 0; c < d; ++c) o_i[c] += p * v_j[c];
  }
  *lse_i = m + log(sum);
  (void)N;
}

/* Full forward over [B,H,N,d]. */
void oracle_attn_fwd(const double* Q, const double* K, const double* V, double* O, double* LSE, int B, int H,
                     int N, int d, int causal, double scale) {
  const int64_t BH = (int64_t)B * H;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 16)
    for (int64_t t = 0; t < BH * N; ++t) {
      const int64_t bh = t / N;
      const int i = (int)(t % N);
      const int64_t base = bh * (int64_t)N * d;
      const int nkeys = causal ? i + 1 : N;
      fwd_row(Q + base + (int64_t)i * d, K + base, V + base, N, d, nkeys, scale, s, O + base + (int64_t)i * d,
              LSE + bh * N + i);
    }
    free(s);
  }
}

/* Forward on a list of sampled rows: rows[2*r] = flattened (b*H+h), rows[2*r+1]
 * = query index.  O_rows is [nrows, d], LSE_rows is [nrows]. */
void oracle_attn_fwd_rows(const double* Q, const double* K, const double* V, const int64_t* rows, int64_t nrows,
                          double* O_rows, double* LSE_rows, int N, int d, int causal, double scale) {
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; ++r) {
      const int64_t bh = rows[2 * r];
      const int i = (int)rows[2 * r + 1];
      const int64_t base = bh * (int64_t)N * d;
      const int nkeys = causal ? i + 1 : N;
      fwd_row(Q + base + (int64_t)i * d, K + base, V + base, N, d, nkeys, scale, s, O_rows + r * d, LSE_rows + r);
    }
    free(s);
  }
}

/* Decode step: one query row per query head against all Nk keys of its
 * key/value head (head h uses key/value head h / (Hq / Hkv)).  Q, O [B*Hq, d];
 * K, V [B*Hkv, Nk, d]; LSE [B*Hq]. */
void oracle_attn_decode(const double* Q, const double* K, const double* V, double* O, double* LSE, int B, int Hq,
                        int Hkv, int Nk, int d, double scale) {
  const int g = Hq / Hkv;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < (int64_t)B * Hq; ++t) {
      const int64_t b = t / Hq, h = t % Hq;
      const int64_t kv = b * Hkv + h / g;
      fwd_row(Q + t * d, K + kv * (int64_t)Nk * d, V + kv * (int64_t)Nk * d, Nk, d, Nk, scale, s, O + t * d,
              LSE + t);
    }
    free(s);
  }
}

/* ------------------------------------------------------------------------- */
/* Backward: derivatives of the definition, one query row at a time           */
/* ------------------------------------------------------------------------- */
void oracle_attn_bwd(const double* Q, const double* K, const double* V, const double* dO, double* dQ, double* dK,
                     double* dV, int B, int H, int N, int d, int causal, double scale) {
  const int64_t BH = (int64_t)B * H;
  const int64_t per = (int64_t)N * d;
  memset(dK, 0, sizeof(double) * (size_t)(BH * per));
  memset(dV, 0, sizeof(double) * (size_t)(BH * per));
#pragma omp parallel
  {
    double* p = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    double* dp = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
      const double* q = Q + bh * per;
      const double* k = K + bh * per;
      const double* v = V + bh * per;
      const double* g = dO + bh * per;
      double* gq = dQ + bh * per;
      double* gk = dK + bh * per;
      double* gv = dV + bh * per;
      for (int i = 0; i < N; ++i) {
        const int nkeys = causal ? i + 1 : N;
        const double* q_i = q + (int64_t)i * d;
        const double* g_i = g + (int64_t)i * d;
        /* P row: two-pass softmax of the materialised scores */
        double m = -INFINITY;
        for (int j = 0; j < nkeys; ++j) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += q_i[c] * k[(int64_t)j * d + c];
          p[j] = scale * acc;
          if (p[j] > m) m = p[j];
        }
        double sum = 0.0;
        for (int j = 0; j < nkeys; ++j) {
          p[j] = exp(p[j] - m);
          sum += p[j];
        }
        for (int j = 0; j < nkeys; ++j) p[j] /= sum;
        /* dP = dO V^T and the row term sum_k P_ik dP_ik */
        double rowdot = 0.0;
        for (int j = 0; j < nkeys; ++j) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += g_i[c] * v[(int64_t)j * d + c];
          dp[j] = acc;
          rowdot += p[j] * acc;
        }
        /* dV += P^T dO ; dS = P o (dP - rowdot) ; dQ_i = scale dS K ; dK += scale dS^T q_i */
        double* gq_i = gq + (int64_t)i * d;
        for (int c = 0; c < d; ++c) gq_i[c] = 0.0;
        for (int j = 0; j < nkeys; ++j) {
          const double ds = p[j] * (dp[j] - rowdot);
          double* gv_j = gv + (int64_t)j * d;
          double* gk_j = gk + (int64_t)j * d;
          const double* k_j = k + (int64_t)j * d;
          for (int c = 0; c < d; ++c) {
            gv_j[c] += p[j] * g_i[c];
            gk_j[c] += scale * ds * q_i[c];
            gq_i[c] += scale * ds * k_j[c];
          }
        }
      }
    }
    free(p);
    free(dp);
  }
}

/* ------------------------------------------------------------------------- */
/* FP8 P-cast forward emulation                                              */
/* ------------------------------------------------------------------------- */
/* counts[0] = sink P' that flushed to zero, counts[1] = sink P total,
 * counts[2] = non-sink flushed, counts[3] = non-sink total.  A key is a sink
 * when its index is < n_sink.  kv_order 0 visits tiles 0..T-1, 1 visits
 * T-1..0.  Tiles are [j*Bc, min(N,(j+1)*Bc)); causal keeps keys <= i. */
void oracle_attn_fwd_fp8p(const double* Q, const double* K, const double* V, double* O, double* LSE, int B, int H,
                          int N, int d, int causal, double scale, double S, int kv_order, int Bc, int n_sink,
                          int64_t* counts) {
  const int64_t BH = (int64_t)B * H;
  const int T = (N + Bc - 1) / Bc;
  int64_t c0 = 0, c1 = 0, c2 = 0, c3 = 0;
#pragma omp parallel reduction(+ : c0, c1, c2, c3)
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(Bc));
    double* acc = (double*)malloc(sizeof(double) * (size_t)(d));
#pragma omp for schedule(dynamic, 16)
    for (int64_t t = 0; t < BH * N; ++t) {
      const int64_t bh = t / N;
      const int i = (int)(t % N);
      const int64_t base = bh * (int64_t)N * d;
      const double* q_i = Q + base + (int64_t)i * d;
      const int nkeys = causal ? i + 1 : N;
      double m = -INFINITY, l = 0.0;
      for (int c = 0; c < d; ++c) acc[c] = 0.0;
      for (int step = 0; step < T; ++step) {
        const int jt = kv_order ? (T - 1 - step) : step;
        const int j0 = jt * Bc;
        int j1 = j0 + Bc;
        if (j1 > nkeys) j1 = nkeys;
        if (j0 >= j1) continue; /* tile entirely masked for this row */
        double tmax = -INFINITY;
        for (int j = j0; j < j1; ++j) {
          double a = 0.0;
          for (int c = 0; c < d; ++c) a += q_i[c] * K[base + (int64_t)j * d + c];
          s[j - j0] = scale * a;
          if (s[j - j0] > tmax) tmax = s[j - j0];
        }
        const double m_new = tmax > m ? tmax : m;
        const double alpha = exp(m - m_new); /* exp(-inf) = 0 on the first tile */
        l *= alpha;
        for (int c = 0; c < d; ++c) acc[c] *= alpha;
        m = m_new;
        for (int j = j0; j < j1; ++j) {
          const double p = exp(s[j - j0] - m);
          l += p;
          const double pq = oracle_e4m3(S * p);
          const int sink = j < n_sink;
          if (sink) { c1++; if (pq == 0.0) c0++; }
          else { c3++; if (pq == 0.0) c2++; }
          const double* v_j = V + base + (int64_t)j * d;
          for (int c = 0; c < d; ++c) acc[c] += pq * v_j[c];
        }
      }
      double* o_i = O + base + (int64_t)i * d;
      for (int c = 0; c < d; ++c) o_i[c] = acc[c] / (S * l);
      LSE[bh * N + i] = m + log(l);
    }
    free(s);
    free(acc);
  }
  counts[0] = c0;
  counts[1] = c1;
  counts[2] = c2;
  counts[3] = c3;
}

/* ------------------------------------------------------------------------- */
/* FP8 operands with incoherent processing ("flash-attention-trading-models", */
/* section "FA3", item 3): rows are multiplied by a random orthogonal matrix   */
/* (random signs, then the normalised Walsh-Hadamard matrix) before block     */
/* quantisation to E4M3, which spreads an outlier's magnitude over the row.   */
/* ------------------------------------------------------------------------- */
/* y = x diag(signs) H / sqrt(d) for one row, H the Sylvester Hadamard matrix,
 * H[i][j] = (-1)^popcount(i & j); written as the definition, O(d^2). */
static void rotate_row(const double* x, const double* signs, double* y, int d) {
  const double norm = 1.0 / sqrt((double)d);
  for (int j = 0; j < d; ++j) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) {
      const int par = __builtin_popcount((unsigned)(i & j)) & 1;
      acc += (par ? -1.0 : 1.0) * signs[i] * x[i];
    }
    y[j] = acc * norm;
  }
}

/* The rotation alone, for `rows` rows of length d. */
void oracle_hadamard_rotate(const double* X, const double* signs, double* Y, int64_t rows, int d) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) rotate_row(X + r * d, signs, Y + r * d, d);
}

/* Quantise [BH, N, d] to E4M3 with one scale per block of `block_rows` rows
 * of each (b,h) (block_rows >= N gives one scale per head).  signs == NULL
 * means no rotation.  Outputs: xq (the dequantised values code * scale, fp64)
 * and scales [BH, ceil(N/block_rows)] with scale = amax / 448 (1 for an
 * all-zero block). */
void oracle_fp8_quantize(const double* X, const double* signs, double* XQ, double* scales, int BH, int N, int d,
                         int block_rows) {
  const int nb = (N + block_rows - 1) / block_rows;
#pragma omp parallel
  {
    double* y = (double*)malloc(sizeof(double) * (size_t)d * (size_t)block_rows);
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < (int64_t)BH * nb; ++t) {
      const int64_t bh = t / nb;
      const int blk = (int)(t % nb);
      const int r0 = blk * block_rows;
      int r1 = r0 + block_rows;
      if (r1 > N) r1 = N;
      double amax = 0.0;
      for (int r = r0; r < r1; ++r) {
        const double* x = X + (bh * N + r) * (int64_t)d;
        double* yr = y + (int64_t)(r - r0) * d;
        if (signs) rotate_row(x, signs, yr, d);
        else for (int c = 0; c < d; ++c) yr[c] = x[c];
        for (int c = 0; c < d; ++c) if (fabs(yr[c]) > amax) amax = fabs(yr[c]);
      }
      const double sc = amax > 0.0 ? amax / 448.0 : 1.0;
      scales[bh * nb + blk] = sc;
      for (int r = r0; r < r1; ++r) {
        const double* yr = y + (int64_t)(r - r0) * d;
        double* q = XQ + (bh * N + r) * (int64_t)d;
        for (int c = 0; c < d; ++c) q[c] = oracle_e4m3(yr[c] / sc) * sc;
      }
    }
    free(y);
  }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
