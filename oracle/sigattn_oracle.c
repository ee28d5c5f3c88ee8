/*
 * sigattn_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct fp64 CPU statement of bidirectional sigmoid
 * attention and its analytic gradient. It exists to check the CUDA library and
 * is never part of the product path: only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load it. It shares no code, header,
 * constant or helper with the CUDA sources.
 *
 * What it computes, per (batch b, head h), with n = lengths[b] valid tokens,
 * L = padded length, d = head dimension:
 *
 *   scale = 1/sqrt(d)                           "Better Models, Faster Training:
 *   bias  = -ln(n)                               Sigmoid Attention for single-cell
 *   S_ij  = scale * <Q_i, K_j>                   Foundation Models", sec. 2A
 *   P_ij  = sigma(S_ij + bias)  if i<n and j<n   (the SigmoidAttn equation and the
 *         = 0                   otherwise         bias term b = -log(n))
 *   O_i   = sum_j P_ij V_j                      (rows i >= n are exactly 0)
 *
 * and for the backward pass (same page, sec. 2B: sigma' = sigma(1 - sigma);
 * sec. 2C: gradients with respect to Q and to K/V, activations recomputed):
 *
 *   dP_ij = <dO_i, V_j>
 *   dS_ij = dP_ij * P_ij * (1 - P_ij)
 *   dQ_i  = scale * sum_j dS_ij K_j
 *   dK_j  = scale * sum_i dS_ij Q_i
 *   dV_j  = sum_i P_ij dO_i
 *
 * Readings where the pages are silent (each listed in the design notes):
 * n is the sequence's valid length and log is natural; padding is applied on
 * both the query and the key side by an exact select to zero; the bias is a
 * constant (no gradient); the attention is bidirectional (no causal mask);
 * n = 0 gives all-zero outputs.
 *
 * Layout: every tensor is a contiguous double array [B][H][L][d] holding the
 * exact values of the bf16 inputs. Outputs are fully written (padded rows get
 * zeros). No blocking, fusion or reordering beyond a loop over rows: the full
 * forward/backward are loops over the single-row functions below, so the
 * sampled-row checks and the full checks run the same arithmetic.
 */
#include <math.h>
#include <stddef.h>
#include <string.h>

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static double dot(const double* a, const double* b, int d) {
  double s = 0.0;
  for (int c = 0; c < d; ++c) s += a[c] * b[c];
  return s;
}

/* sigma(x) itself, exported so the tests can pin it against closed forms. */
double oracle_sigmoid(double x) { return sigmoid(x); }

/* The attention weight P_ij of one (b,h) slice; 0 outside the valid square. */
double oracle_weight(const double* q, const double* k, int n, int d, int i, int j) {
  if (i >= n || j >= n) return 0.0;
  const double scale = 1.0 / sqrt((double)d);
  const double bias = -log((double)n);
  return sigmoid(scale * dot(q + (size_t)i * d, k + (size_t)j * d, d) + bias);
}

/* O_i for one (b,h) slice. q,k,v point at the slice's [L][d] block. */
void oracle_fwd_row(const double* q, const double* k, const double* v, int n, int d,
                    int i, double* o_row) {
  for (int c = 0; c < d; ++c) o_row[c] = 0.0;
  if (i >= n) return;
  for (int j = 0; j < n; ++j) {
    const double p = oracle_weight(q, k, n, d, i, j);
    const double* vj = v + (size_t)j * d;
    for (int c = 0; c < d; ++c) o_row[c] += p * vj[c];
  }
}

/* dQ_i for one (b,h) slice. */
void oracle_dq_row(const double* q, const double* k, const double* v, const double* dout,
                   int n, int d, int i, double* dq_row) {
  for (int c = 0; c < d; ++c) dq_row[c] = 0.0;
  if (i >= n) return;
  const double scale = 1.0 / sqrt((double)d);
  const double* doi = dout + (size_t)i * d;
  for (int j = 0; j < n; ++j) {
    const double p = oracle_weight(q, k, n, d, i, j);
    const double dp = dot(doi, v + (size_t)j * d, d);
    const double ds = dp * p * (1.0 - p);
    const double* kj = k + (size_t)j * d;
    for (int c = 0; c < d; ++c) dq_row[c] += ds * kj[c];
  }
  for (int c = 0; c < d; ++c) dq_row[c] *= scale;
}

/* dK_j and dV_j for one (b,h) slice (a sum over the query index i). */
void oracle_dkdv_row(const double* q, const double* k, const double* v, const double* dout,
                     int n, int d, int j, double* dk_row, double* dv_row) {
  for (int c = 0; c < d; ++c) { dk_row[c] = 0.0; dv_row[c] = 0.0; }
  if (j >= n) return;
  const double scale = 1.0 / sqrt((double)d);
  const double* vj = v + (size_t)j * d;
  for (int i = 0; i < n; ++i) {
    const double p = oracle_weight(q, k, n, d, i, j);
    const double* doi = dout + (size_t)i * d;
    const double dp = dot(doi, vj, d);
    const double ds = dp * p * (1.0 - p);
    const double* qi = q + (size_t)i * d;
    for (int c = 0; c < d; ++c) {
      dv_row[c] += p * doi[c];
      dk_row[c] += ds * qi[c];
    }
  }
  for (int c = 0; c < d; ++c) dk_row[c] *= scale;
}

static int valid_len(const int* lengths, int b, int L) {
  int n = lengths[b];
  if (n < 0) n = 0;
  if (n > L) n = L;
  return n;
}

/* Full forward over [B][H][L][d]; parallel over (b,h,i) rows only. */
void oracle_fwd(const double* q, const double* k, const double* v, double* o,
                const int* lengths, int B, int H, int L, int d) {
  const long long rows = (long long)B * H * L;
#pragma omp parallel for schedule(dynamic, 16)
  for (long long r = 0; r < rows; ++r) {
    const long long bh = r / L;
    const int i = (int)(r % L);
    const int b = (int)(bh / H);
    const size_t off = (size_t)bh * L * d;
    oracle_fwd_row(q + off, k + off, v + off, valid_len(lengths, b, L), d, i,
                   o + off + (size_t)i * d);
  }
}

/* Full backward over [B][H][L][d]; parallel over rows only. */
void oracle_bwd(const double* q, const double* k, const double* v, const double* dout,
                double* dq, double* dk, double* dv, const int* lengths, int B, int H, int L,
                int d) {
  const long long rows = (long long)B * H * L;
#pragma omp parallel for schedule(dynamic, 16)
  for (long long r = 0; r < rows; ++r) {
    const long long bh = r / L;
    const int t = (int)(r % L);
    const int b = (int)(bh / H);
    const int n = valid_len(lengths, b, L);
    const size_t off = (size_t)bh * L * d;
    oracle_dq_row(q + off, k + off, v + off, dout + off, n, d, t, dq + off + (size_t)t * d);
    oracle_dkdv_row(q + off, k + off, v + off, dout + off, n, d, t, dk + off + (size_t)t * d,
                    dv + off + (size_t)t * d);
  }
}

/*
 * Sampled rows: out[s][d] = the requested output row for sample s, where
 * sample s names (bh[s], row[s]). which = 0: O, 1: dQ, 2: dK, 3: dV.
 */
void oracle_rows(const double* q, const double* k, const double* v, const double* dout,
                 const int* lengths, int B, int H, int L, int d, int which, const int* bh,
                 const int* row, int nsamp, double* out) {
  (void)B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int s = 0; s < nsamp; ++s) {
    const int b = bh[s] / H;
    const int n = valid_len(lengths, b, L);
    const size_t off = (size_t)bh[s] * L * d;
    double* dst = out + (size_t)s * d;
    if (which == 0) {
      oracle_fwd_row(q + off, k + off, v + off, n, d, row[s], dst);
    } else if (which == 1) {
      oracle_dq_row(q + off, k + off, v + off, dout + off, n, d, row[s], dst);
    } else {
      double tmp_k[512], tmp_v[512];
      oracle_dkdv_row(q + off, k + off, v + off, dout + off, n, d, row[s], tmp_k, tmp_v);
      memcpy(dst, which == 2 ? tmp_k : tmp_v, sizeof(double) * (size_t)d);
    }
  }
}

/*
 * The active tile list ("block-sparse computation that skips blocks padded on
 * both the query and the key side", same page, sec. 2C). Work item = one block
 * of `block` consecutive rows of one (b,h) slice that holds at least one valid
 * token, i.e. block index m with m*block < n_b. Items are listed in canonical
 * order (b, h, m ascending) as int32 triples (b, h, m). Returns the number of
 * items; writes at most `cap` of them.
 */
int oracle_tiles(const int* lengths, int B, int H, int L, int block, int* out, int cap) {
  int count = 0;
  for (int b = 0; b < B; ++b) {
    const int n = valid_len(lengths, b, L);
    for (int h = 0; h < H; ++h) {
      for (int m = 0; m * block < n; ++m) {
        if (count < cap) {
          out[3 * count + 0] = b;
          out[3 * count + 1] = h;
          out[3 * count + 2] = m;
        }
        ++count;
      }
    }
  }
  return count;
}

/*
 * The softmax counterpart, against which the sigmoid kernels are compared on
 * the same scheduler ("Better Models, Faster Training: Sigmoid Attention for
 * single-cell Foundation Models", sec. 4A, compares the sigmoid kernel with
 * softmax attention's FlashAttention-2 at 25% padding; sec. 2A contrasts the
 * two weightings; "Transformer Attention機構の効率化と最新派生モデル" states
 * softmax attention in its "Vanilla Self-Attention" pseudo code example). For one
 * (b,h) slice and a valid row i < n, over the valid keys j < n only:
 *
 *   S_ij  = <Q_i, K_j> / sqrt(d)             (no bias: softmax normalises)
 *   m_i   = max_{j<n} S_ij
 *   O_i   = sum_j exp(S_ij - m_i) V_j / sum_j exp(S_ij - m_i)
 *   lse_i = m_i + ln sum_j exp(S_ij - m_i)
 *
 * Rows i >= n are 0 (O and lse), as for the sigmoid path.
 */
void oracle_softmax_fwd_row(const double* q, const double* k, const double* v, int n, int d, int i,
                            double* o_row, double* lse) {
  for (int c = 0; c < d; ++c) o_row[c] = 0.0;
  *lse = 0.0;
  if (i >= n) return;
  const double scale = 1.0 / sqrt((double)d);
  const double* qi = q + (size_t)i * d;
  double m = -INFINITY;
  for (int j = 0; j < n; ++j) {
    const double s = scale * dot(qi, k + (size_t)j * d, d);
    if (s > m) m = s;
  }
  double l = 0.0;
  for (int j = 0; j < n; ++j) {
    const double p = exp(scale * dot(qi, k + (size_t)j * d, d) - m);
    l += p;
    const double* vj = v + (size_t)j * d;
    for (int c = 0; c < d; ++c) o_row[c] += p * vj[c];
  }
  for (int c = 0; c < d; ++c) o_row[c] /= l;
  *lse = m + log(l);
}

/* Full softmax forward over [B][H][L][d] (lse: [B][H][L]); parallel over rows. */
void oracle_softmax_fwd(const double* q, const double* k, const double* v, double* o, double* lse,
                        const int* lengths, int B, int H, int L, int d) {
  const long long rows = (long long)B * H * L;
#pragma omp parallel for schedule(dynamic, 16)
  for (long long r = 0; r < rows; ++r) {
    const long long bh = r / L;
    const int i = (int)(r % L);
    const int b = (int)(bh / H);
    const size_t off = (size_t)bh * L * d;
    oracle_softmax_fwd_row(q + off, k + off, v + off, valid_len(lengths, b, L), d, i, o + off + (size_t)i * d,
                           lse + (size_t)bh * L + i);
  }
}
