/*
 * csa_oracle.c - plain, slow FP64 CPU oracle for the CSA / HCA attention
 * layer of DeepSeek-V4.
 *
 * TEST INFRASTRUCTURE. This file is the independent reference that the CUDA
 * library is checked against. Only the tests, the package's smoke() entry
 * and the benchmark's CPU-baseline leg load it; the product path never does.
 * It shares no code, header, table or helper with the CUDA path.
 *
 * Every function evaluates the definition written in its comment, in IEEE
 * double precision, with plain loops and no blocking, fusion or streaming.
 * OpenMP splits only independent outer iterations (blocks, queries); the
 * arithmetic of one output never depends on the thread count.
 *
 * Sources (page title, then section / equation):
 *   [EL] "Evidence Ledger": CSA Eqs 9-19, HCA Eqs 20-26, Shared attention
 *        details (Sec 2.3.3, Eq 27), Sec 2.3.4 mixed KV storage.
 *   [SY] "DeepSeek-V4" study: 03 Two resolutions of history (pooling formula
 *        c_block = sum_t softmax_t(z_t + b_t) * v_t; index score
 *        score(t,s) = sum_h w_{t,h} ReLU(q^I_{t,h} . k^I_s)).
 *   [CA] "DeepSeek-V4: What Remains After Compressing History?": Sec 1 (one
 *        normalisation shared by local, compressed and sink terms), Sec 3
 *        (completed-entry count (p+1)//m).
 *
 * Readings where the pages are silent are the ones the library header
 * states (visibility offset, absent b-series for block 0, bias row order,
 * RMSNorm, interleaved RoPE with entry position i*m, 1/sqrt(c) scale, sink
 * without value, FP8 row scale).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR 1

/* RMSNorm over c values: y = x / sqrt(mean(x^2) + eps) * gain.
 * [EL] Shared attention details (Sec 2.3.3). gain NULL means ones. */
static void orc_rmsnorm(const double* x, int c, const double* gain, double eps, double* y) {
  double ss = 0.0;
  for (int i = 0; i < c; ++i) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss / (double)c + eps);
  for (int i = 0; i < c; ++i) y[i] = x[i] * inv * (gain ? gain[i] : 1.0);
}

/* Partial RoPE, in place: the last r dims of x (width c) as interleaved
 * pairs (c-r+2i, c-r+2i+1), pair i rotated by angle pos * base^(-2i/r).
 * [EL] Shared attention details: RoPE on the last 64 dims; a negative pos
 * gives the inverse rotation applied to attention outputs. */
static void orc_rope(double* x, int c, int r, double base, double pos) {
  for (int i = 0; i < r / 2; ++i) {
    double theta = pow(base, -2.0 * (double)i / (double)r);
    double a = pos * theta;
    double cs = cos(a), sn = sin(a);
    double x0 = x[c - r + 2 * i], x1 = x[c - r + 2 * i + 1];
    x[c - r + 2 * i] = x0 * cs - x1 * sn;
    x[c - r + 2 * i + 1] = x0 * sn + x1 * cs;
  }
}

/* Exported wrappers, so tests can pin the two building blocks directly. */
void orc_rmsnorm_rows(const double* x, int64_t rows, int c, const double* gain, double eps,
                      double* y) {
  for (int64_t r = 0; r < rows; ++r) orc_rmsnorm(x + r * c, c, gain, eps, y + r * c);
}

void orc_rope_rows(double* x, int64_t rows, int c, int r, double base, const double* pos) {
  for (int64_t i = 0; i < rows; ++i) orc_rope(x + i * c, c, r, base, pos[i]);
}

/* y = RoPE_pos(RMSNorm(x) * gain) per row: the preparation of window rows
 * and compressed entries for core attention ([EL] Sec 2.3.3). */
void orc_rmsnorm_rope_rows(const double* x, int64_t rows, int c, int r, double base,
                           double eps, const double* gain, const double* pos, double* y) {
  for (int64_t i = 0; i < rows; ++i) {
    orc_rmsnorm(x + i * c, c, gain, eps, y + i * c);
    orc_rope(y + i * c, c, r, base, pos[i]);
  }
}

/* Dot product of row t of H [T,d] with column ch of W [d,c]: one element of
 * the projections C = H W, Z = H W ([EL] CSA Eqs 9-10). */
static double orc_proj(const double* H, int d, const double* W, int c, int64_t t, int ch) {
  double acc = 0.0;
  for (int k = 0; k < d; ++k) acc += H[t * (int64_t)d + k] * W[(int64_t)k * c + ch];
  return acc;
}

/*
 * Compressed entries for the listed blocks ([EL] CSA Eqs 9-12, HCA Eqs
 * 20-26; [SY] 03). For block i and channel ch the candidates are
 *   overlap = 1: r = 0..m-1, token (i-1)m + r, values C^b = H W_bKV,
 *                logits Z^b = H W_bZ plus bias[r] (absent when i = 0);
 *                r = m..2m-1, token im + r - m, C^a = H W_aKV,
 *                Z^a = H W_aZ plus bias[r].
 *   overlap = 0: r = 0..m-1, token im + r, C = H W_aKV, Z = H W_aZ, bias[r].
 * pooled[ch] = sum_r softmax_r(Z + bias)[r] * C[r]; the entry is
 * RoPE_{i*m}(RMSNorm(pooled) * gain).
 * pooled_out (may be NULL) receives the pre-normalisation pooled vectors.
 * A bias of -INFINITY removes a candidate from the softmax.
 */
int orc_compress_blocks(int64_t T, int d, int c, int m, int overlap, const double* H,
                        const double* WaKV, const double* WbKV, const double* WaZ,
                        const double* WbZ, const double* bias, const double* gain, double eps,
                        int r, double base, const int64_t* blocks, int64_t nb, double* E_out,
                        double* pooled_out) {
  if (m <= 0 || c <= 0 || d <= 0 || T < 0) return ORC_ERR;
  if (overlap && (!WbKV || !WbZ)) return ORC_ERR;
  for (int64_t bi = 0; bi < nb; ++bi)
    if (blocks[bi] < 0 || blocks[bi] >= T / m) return ORC_ERR;
  const int ncand = overlap ? 2 * m : m;
  int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bi = 0; bi < nb; ++bi) {
    const int64_t i = blocks[bi];
    double* val = (double*)malloc(sizeof(double) * (size_t)ncand * c);
    double* lg = (double*)malloc(sizeof(double) * (size_t)ncand * c);
    int* present = (int*)malloc(sizeof(int) * (size_t)ncand);
    double* pooled = (double*)malloc(sizeof(double) * (size_t)c);
    if (!val || !lg || !present || !pooled) {
#pragma omp atomic write
      fail = 1;
    } else {
      for (int rr = 0; rr < ncand; ++rr) {
        int64_t tok;
        const double *Wv, *Wz;
        if (overlap && rr < m) { /* preceding block, b-series */
          tok = (i - 1) * m + rr;
          Wv = WbKV;
          Wz = WbZ;
          present[rr] = (i >= 1);
        } else { /* own block, a-series */
          tok = i * m + (overlap ? rr - m : rr);
          Wv = WaKV;
          Wz = WaZ;
          present[rr] = 1;
        }
        if (!present[rr]) continue;
        for (int ch = 0; ch < c; ++ch) {
          val[(size_t)rr * c + ch] = orc_proj(H, d, Wv, c, tok, ch);
          lg[(size_t)rr * c + ch] = orc_proj(H, d, Wz, c, tok, ch) + bias[(size_t)rr * c + ch];
        }
      }
      for (int ch = 0; ch < c; ++ch) {
        double mx = -INFINITY;
        for (int rr = 0; rr < ncand; ++rr)
          if (present[rr] && lg[(size_t)rr * c + ch] > mx) mx = lg[(size_t)rr * c + ch];
        double den = 0.0, num = 0.0;
        for (int rr = 0; rr < ncand; ++rr) {
          if (!present[rr]) continue;
          double e = exp(lg[(size_t)rr * c + ch] - mx);
          den += e;
          num += e * val[(size_t)rr * c + ch];
        }
        pooled[ch] = num / den;
      }
      if (pooled_out) memcpy(pooled_out + bi * c, pooled, sizeof(double) * (size_t)c);
      orc_rmsnorm(pooled, c, gain, eps, E_out + bi * c);
      orc_rope(E_out + bi * c, c, r, base, (double)(i * m));
    }
    free(val);
    free(lg);
    free(present);
    free(pooled);
  }
  return fail ? ORC_ERR : ORC_OK;
}

/* Number of compressed entries visible to a query at position p:
 * floor((p + vis_offset) / m), clipped to [0, n_entries].
 * [EL] CSA: strict causality s < floor(t/m); [CA] Sec 3: (p+1)//m. */
static int64_t orc_n_vis(int64_t p, int m, int vis_offset, int64_t n_entries) {
  int64_t v = (p + vis_offset) / m;
  if (p + vis_offset < 0) v = 0;
  if (v > n_entries) v = n_entries;
  if (v < 0) v = 0;
  return v;
}

int64_t orc_visible_entries(int64_t p, int m, int vis_offset, int64_t n_entries) {
  return orc_n_vis(p, m, vis_offset, n_entries);
}

typedef struct {
  double score;
  int64_t s;
} orc_scored;

/* Order by descending score, then ascending index (ties keep the lower s). */
static int orc_cmp_desc(const void* a, const void* b) {
  const orc_scored* x = (const orc_scored*)a;
  const orc_scored* y = (const orc_scored*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->s < y->s) ? -1 : (x->s > y->s);
}

static int orc_cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/*
 * Lightning indexer and top-k ([EL] CSA Eqs 13-17; [SY] 03):
 *   I[q,s] = sum_h w[q,h] * max(0, sum_j qI[q,h,j] * KI[b,s,j]), s < n_vis(q)
 * then a full sort by (-I, s) keeps k_eff = min(k, n_vis) entries, written
 * in ascending s and padded with -1.
 * Diagnostics (each may be NULL):
 *   tau_out[q]  = the k_eff-th largest score (NaN when k_eff = 0)
 *   amag_out[q] = max_s sum_h |w[q,h]| * sum_j |qI[q,h,j] * KI[b,s,j]|, the
 *                 magnitude that bounds rounding error in any evaluation order
 *   scores_out  [Q, ldK]: I[q,s] for s < n_vis(q)
 */
int orc_index_topk(int64_t Q, int HI, int cI, int k, int m, int vis_offset, const double* qI,
                   const double* w, const double* KI, int64_t ldK, const int32_t* seq_of_q,
                   const int64_t* pos, const int64_t* n_entries, int32_t* idx_out,
                   double* tau_out, double* amag_out, double* scores_out) {
  if (k <= 0 || HI <= 0 || cI <= 0 || m <= 0) return ORC_ERR;
  int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t q = 0; q < Q; ++q) {
    const int32_t b = seq_of_q[q];
    const int64_t nv = orc_n_vis(pos[q], m, vis_offset, n_entries[b]);
    orc_scored* sc = (orc_scored*)malloc(sizeof(orc_scored) * (size_t)(nv > 0 ? nv : 1));
    int32_t* kept = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    if (!sc || !kept) {
#pragma omp atomic write
      fail = 1;
      free(sc);
      free(kept);
      continue;
    }
    double amax = 0.0;
    for (int64_t s = 0; s < nv; ++s) {
      const double* ks = KI + ((int64_t)b * ldK + s) * cI;
      double I = 0.0, A = 0.0;
      for (int h = 0; h < HI; ++h) {
        const double* qh = qI + (q * HI + h) * cI;
        double dot = 0.0, mag = 0.0;
        for (int j = 0; j < cI; ++j) {
          dot += qh[j] * ks[j];
          mag += fabs(qh[j] * ks[j]);
        }
        I += w[q * HI + h] * (dot > 0.0 ? dot : 0.0);
        A += fabs(w[q * HI + h]) * mag;
      }
      sc[s].score = I;
      sc[s].s = s;
      if (A > amax) amax = A;
      if (scores_out) scores_out[q * ldK + s] = I;
    }
    qsort(sc, (size_t)nv, sizeof(orc_scored), orc_cmp_desc);
    const int64_t keff = nv < k ? nv : k;
    for (int64_t j = 0; j < keff; ++j) kept[j] = (int32_t)sc[j].s;
    qsort(kept, (size_t)keff, sizeof(int32_t), orc_cmp_i32);
    for (int64_t j = 0; j < k; ++j) idx_out[q * k + j] = j < keff ? kept[j] : -1;
    if (tau_out) tau_out[q] = keff > 0 ? sc[keff - 1].score : NAN;
    if (amag_out) amag_out[q] = amax;
    free(sc);
    free(kept);
  }
  return fail ? ORC_ERR : ORC_OK;
}

/*
 * Shared-KV MQA core attention with sliding window and sink
 * ([EL] CSA Eqs 18-19, Shared attention details Sec 2.3.3 and Eq 27;
 * [SY] 03; [CA] Sec 1). For query q (sequence b, position p), head h:
 *   qh = RoPE_p(RMSNorm(q[q,h]) * q_gain)
 *   keys: E[b, idx[q,j]] for idx >= 0 (dense = 1: E[b, s] for s < n_vis(p)),
 *         then window rows of positions j = max(0, p - n_win + 1) .. p
 *         (row j, or row j mod n_win when win_ring = 1)
 *   l_j = qh . k_j / sqrt(c)
 *   o   = sum_j exp(l_j) k_j / (exp(sink[h]) + sum_j exp(l_j))
 *   O[q,h] = RoPE_{-p}(o)
 * Every key is both key and value (shared KV). The common factor exp(-M),
 * M = max(sink, l_j), is applied to numerator and denominator alike.
 * nkeys_out[q] (may be NULL) receives |J(q)|, the main-KV reads of the query.
 */
int orc_attend(int64_t Q, int Hq, int c, int r, double base, double eps, int n_win,
               int win_ring, const double* q, const double* q_gain, const double* sink,
               const double* E, int64_t ldE, const int64_t* n_entries, const int32_t* idx,
               int k, int dense, int m, int vis_offset, const double* win, int64_t ldW,
               const int32_t* seq_of_q, const int64_t* pos, double* O, int32_t* nkeys_out) {
  if (c <= 0 || Hq <= 0 || n_win < 0 || (!dense && (!idx || k < 0))) return ORC_ERR;
  int fail = 0;
  const double scale = 1.0 / sqrt((double)c);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t qi = 0; qi < Q; ++qi) {
    const int32_t b = seq_of_q[qi];
    const int64_t p = pos[qi];
    const int64_t nv = dense ? orc_n_vis(p, m, vis_offset, n_entries[b]) : 0;
    const int64_t nsel = dense ? nv : k;
    const int64_t w0 = p - n_win + 1 > 0 ? p - n_win + 1 : 0;
    const int64_t nw = n_win > 0 ? p - w0 + 1 : 0;
    const double** keys = (const double**)malloc(sizeof(double*) * (size_t)(nsel + nw + 1));
    double* l = (double*)malloc(sizeof(double) * (size_t)(nsel + nw + 1));
    double* qh = (double*)malloc(sizeof(double) * (size_t)c);
    double* o = (double*)malloc(sizeof(double) * (size_t)c);
    if (!keys || !l || !qh || !o) {
#pragma omp atomic write
      fail = 1;
    } else {
      int64_t nk = 0;
      for (int64_t j = 0; j < nsel; ++j) {
        int64_t s = dense ? j : (int64_t)idx[qi * k + j];
        if (s < 0) continue;
        keys[nk++] = E + ((int64_t)b * ldE + s) * c;
      }
      for (int64_t j = w0; j <= p && n_win > 0; ++j) {
        int64_t row = win_ring ? (j % n_win) : j;
        keys[nk++] = win + ((int64_t)b * ldW + row) * c;
      }
      if (nkeys_out) nkeys_out[qi] = (int32_t)nk;
      for (int h = 0; h < Hq; ++h) {
        orc_rmsnorm(q + (qi * Hq + h) * c, c, q_gain, eps, qh);
        orc_rope(qh, c, r, base, (double)p);
        double M = sink[h];
        for (int64_t j = 0; j < nk; ++j) {
          double dot = 0.0;
          for (int i = 0; i < c; ++i) dot += qh[i] * keys[j][i];
          l[j] = dot * scale;
          if (l[j] > M) M = l[j];
        }
        double den = exp(sink[h] - M);
        for (int i = 0; i < c; ++i) o[i] = 0.0;
        for (int64_t j = 0; j < nk; ++j) {
          double e = exp(l[j] - M);
          den += e;
          for (int i = 0; i < c; ++i) o[i] += e * keys[j][i];
        }
        for (int i = 0; i < c; ++i) o[i] /= den;
        orc_rope(o, c, r, base, -(double)p);
        memcpy(O + (qi * Hq + h) * c, o, sizeof(double) * (size_t)c);
      }
    }
    free(keys);
    free(l);
    free(qh);
    free(o);
  }
  return fail ? ORC_ERR : ORC_OK;
}

/* ---------------------------------------------------------------------
 * FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; largest finite 448) for the mixed entry
 * storage of [EL] Sec 2.3.4 / [SY] 06.
 * ------------------------------------------------------------------- */

/* Exact value of an E4M3 code. */
double orc_e4m3_decode(uint8_t code) {
  int sgn = code >> 7, e = (code >> 3) & 15, f = code & 7;
  if (e == 15 && f == 7) return NAN;
  double v = (e == 0) ? ldexp((double)f, -9) : ldexp(8.0 + f, e - 10);
  return sgn ? -v : v;
}

/* Nearest E4M3 code to x, ties to the even code, magnitudes above 448
 * clamped to 448 (saturating). Scans the 127 non-negative finite codes,
 * whose values increase with the code. */
uint8_t orc_e4m3_encode(double x) {
  uint8_t sgn = (x < 0) ? 0x80 : 0;
  double a = fabs(x);
  if (a >= 448.0) return sgn | 0x7E;
  uint8_t best = 0;
  for (int cde = 1; cde <= 0x7E; ++cde) {
    double v = orc_e4m3_decode((uint8_t)cde);
    double vb = orc_e4m3_decode(best);
    double dv = fabs(v - a), db = fabs(vb - a);
    if (dv < db || (dv == db && (cde & 1) == 0)) best = (uint8_t)cde;
  }
  return sgn | best;
}

/* Mixed row (592 bytes) from 512 FP32 values: scale = max|x[0:448]| / 448
 * and codes RNE(x / scale), both divisions in FP32 so that the quantised
 * codes follow the same rounding decisions as any FP32 writer; 64 trailing
 * values rounded to BF16 (nearest, ties to even). */
void orc_pack_mixed_row(const float* x, uint8_t* out) {
  float amax = 0.0f;
  for (int i = 0; i < 448; ++i) {
    float a = fabsf(x[i]);
    if (a > amax) amax = a;
  }
  volatile float scale = amax / 448.0f;
  memset(out, 0, 592);
  for (int i = 0; i < 448; ++i) {
    volatile float qv = (scale > 0.0f) ? x[i] / scale : 0.0f;
    out[i] = orc_e4m3_encode((double)qv);
  }
  for (int i = 0; i < 64; ++i) {
    uint32_t u;
    memcpy(&u, &x[448 + i], 4);
    uint32_t lsb = (u >> 16) & 1u;
    uint16_t bf = (uint16_t)((u + 0x7FFFu + lsb) >> 16);
    memcpy(out + 448 + 2 * i, &bf, 2);
  }
  float s = scale;
  memcpy(out + 576, &s, 4);
}

/* Exact FP64 values of a mixed row. */
void orc_unpack_mixed_row(const uint8_t* in, double* x) {
  float s;
  memcpy(&s, in + 576, 4);
  for (int i = 0; i < 448; ++i) x[i] = orc_e4m3_decode(in[i]) * (double)s;
  for (int i = 0; i < 64; ++i) {
    uint16_t bf;
    memcpy(&bf, in + 448 + 2 * i, 2);
    uint32_t u = (uint32_t)bf << 16;
    float f;
    memcpy(&f, &u, 4);
    x[448 + i] = (double)f;
  }
}
