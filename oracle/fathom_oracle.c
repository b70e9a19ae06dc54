/*
 * Fathom key-scan ORACLE -- test infrastructure, not the product.
 *
 * A plain, slow, single-threaded CPU statement of what the Fathom scan
 * computes, in fp64, written from the method as the pages describe it:
 *   "Fathom Makes KV-Cache Scans Query-Adaptive for Long-Context Decoding"
 *     (cctest.ai), method paragraphs 2-3;
 *   "Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded KV
 *     Caches" (arXiv 2609.17652), abstract.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg load
 * this file.  It shares no code, header or table with the CUDA library.
 *
 * Readings taken where the pages are silent (each is listed with its reason
 * in the design notes):
 *   - plane j = 0 is the most significant bit of the 4-bit code, so the first
 *     t planes give the code's top t bits; token 32*w + b sits in bit b of
 *     word w of a plane row; a row holds ceil(n / 128) * 4 words (16-byte
 *     multiple) and every bit past the last token is 0;
 *   - a t-plane prefix v reconstructs at the centre of its t-bit cell:
 *     deq_t(v) = m + s * (2^(4-t) * v + (2^(4-t) - 1) / 2); t = 0 gives the
 *     constant m + 7.5 s;
 *   - the integer allocation is the greedy over the 4d "slots" (c, tau)
 *     with keys w_c * 4^-tau, ordered by key descending, then c ascending,
 *     then tau ascending; the first B slots are taken and t_c counts the
 *     slots of channel c.  This is the exact integer optimum of
 *     sum_c w_c 4^-t_c subject to sum_c t_c = B, 0 <= t_c <= 4, whose
 *     continuous relaxation is the closed form b_c = clip(log2(w_c/theta)/2,
 *     0, 4) (the abstract's reverse water-filling);
 *   - scores are the raw dot product (no 1/sqrt(d)); top-k is ordered by
 *     score descending, then index ascending; k > n pads with index -1.
 *
 * Parity pins: every function here is checked in tests/test_oracle_pins.py
 * against closed forms, invariants, brute force and a library matmul.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Words in one plane row: the row is padded to a multiple of 128 tokens. */
int64_t oracle_plane_words(int64_t n) { return ((n + 127) / 128) * 4; }

static unsigned code_at(const uint8_t *codes_g, int d, int64_t i, int c) {
  uint8_t byte = codes_g[i * (d / 2) + c / 2];
  return (c & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 15u);
}

/* Channel-major bit planes (method paragraph 2: the 4-bit K cache is kept as
 * bit planes, channel by channel).  codes: [h_kv][n][d/2] nibbles,
 * planes: [h_kv][d][4][W]. */
void oracle_pack_planes(const uint8_t *codes, int64_t n, int d, int h_kv, uint32_t *planes) {
  int64_t W = oracle_plane_words(n);
  memset(planes, 0, (size_t)h_kv * d * 4 * W * sizeof(uint32_t));
  for (int g = 0; g < h_kv; ++g) {
    const uint8_t *codes_g = codes + (int64_t)g * n * (d / 2);
    for (int c = 0; c < d; ++c) {
      for (int j = 0; j < 4; ++j) {
        uint32_t *row = planes + (((int64_t)g * d + c) * 4 + j) * W;
        for (int64_t i = 0; i < n; ++i) {
          unsigned u = code_at(codes_g, d, i, c);
          if ((u >> (3 - j)) & 1u) row[i / 32] |= 1u << (i % 32);
        }
      }
    }
  }
}

/* The value of the first t planes of every (token, channel): v[g][i][c] =
 * sum_{j<t} bit_j * 2^(t-1-j).  This is what reading a t-plane prefix gives. */
void oracle_prefix_values(const uint32_t *planes, int64_t n, int d, int h_kv, int t, uint8_t *v) {
  int64_t W = oracle_plane_words(n);
  for (int g = 0; g < h_kv; ++g)
    for (int64_t i = 0; i < n; ++i)
      for (int c = 0; c < d; ++c) {
        unsigned val = 0;
        for (int j = 0; j < t; ++j) {
          const uint32_t *row = planes + (((int64_t)g * d + c) * 4 + j) * W;
          unsigned bit = (row[i / 32] >> (i % 32)) & 1u;
          val += bit << (t - 1 - j);
        }
        v[((int64_t)g * n + i) * d + c] = (uint8_t)val;
      }
}

/* ---- per-query allocation: reverse water-filling, integer form ---------- */

typedef struct {
  double key; /* w_c * 4^-tau */
  int c;
  int tau;
} slot_t;

static int slot_order(const void *pa, const void *pb) {
  const slot_t *a = (const slot_t *)pa, *b = (const slot_t *)pb;
  if (a->key > b->key) return -1;
  if (a->key < b->key) return 1;
  if (a->c != b->c) return a->c < b->c ? -1 : 1;
  if (a->tau != b->tau) return a->tau < b->tau ? -1 : 1;
  return 0;
}

/* Importance w_c = q_c^2 * sigma_c^2 (abstract: the channels' importance
 * weighted by their variance), one rounding after two exact squares. */
double oracle_importance(double q, double sigma) { return (q * q) * (sigma * sigma); }

/* One query head: t[c] in 0..4 with sum t = budget (0 <= budget <= 4d). */
void oracle_allocate(const double *q, const double *sigma, int d, int budget, uint8_t *t) {
  slot_t *slots = (slot_t *)malloc(sizeof(slot_t) * 4 * (size_t)d);
  for (int c = 0; c < d; ++c) {
    double w = oracle_importance(q[c], sigma[c]);
    for (int tau = 0; tau < 4; ++tau) {
      slots[c * 4 + tau].key = ldexp(w, -2 * tau);
      slots[c * 4 + tau].c = c;
      slots[c * 4 + tau].tau = tau;
    }
  }
  qsort(slots, 4 * (size_t)d, sizeof(slot_t), slot_order);
  for (int c = 0; c < d; ++c) t[c] = 0;
  for (int s = 0; s < budget && s < 4 * d; ++s) t[slots[s].c] += 1;
  free(slots);
}

/* ---- scores -------------------------------------------------------------- */

/* Cell-centre reconstruction of a t-bit prefix value v of a channel with
 * offset m and step s (method paragraph 2: a channel's first t planes
 * give that channel's t-bit quantised value). */
double oracle_dequant_prefix(double m, double s, int t, unsigned v) {
  double cell = ldexp(1.0, 4 - t); /* 2^(4-t) */
  return m + s * (cell * (double)v + (cell - 1.0) / 2.0);
}

/* Scores of one query head over its KV head, from the 4-bit codes:
 * s(i) = sum_c q_c * deq_{t_c}(u_{i,c} >> (4 - t_c)). */
void oracle_scores_from_codes(const uint8_t *codes_g, int64_t n, int d, const float *qmin_g,
                              const float *qscale_g, const double *q, const uint8_t *t,
                              double *out) {
  for (int64_t i = 0; i < n; ++i) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c) {
      unsigned u = code_at(codes_g, d, i, c);
      unsigned v = u >> (4 - t[c]);
      acc += q[c] * oracle_dequant_prefix((double)qmin_g[c], (double)qscale_g[c], t[c], v);
    }
    out[i] = acc;
  }
}

/* The same scores at selected token indices only. */
void oracle_scores_at(const uint8_t *codes_g, int64_t n, int d, const float *qmin_g,
                      const float *qscale_g, const double *q, const uint8_t *t,
                      const int64_t *idx, int64_t m, double *out) {
  (void)n;
  for (int64_t r = 0; r < m; ++r) {
    int64_t i = idx[r];
    double acc = 0.0;
    for (int c = 0; c < d; ++c) {
      unsigned u = code_at(codes_g, d, i, c);
      unsigned v = u >> (4 - t[c]);
      acc += q[c] * oracle_dequant_prefix((double)qmin_g[c], (double)qscale_g[c], t[c], v);
    }
    out[r] = acc;
  }
}

/* Second formulation, from the bit planes: a per-query constant plus one
 * weight per set bit of every allocated plane,
 *   s(i) = C + sum_c sum_{j < t_c} q_c s_c 2^(3-j) bit_{c,j}(i),
 *   C    = sum_c q_c (m_c + s_c (2^(4-t_c) - 1) / 2). */
void oracle_scores_from_planes(const uint32_t *planes_g, int64_t n, int d, const float *qmin_g,
                               const float *qscale_g, const double *q, const uint8_t *t,
                               double *out) {
  int64_t W = oracle_plane_words(n);
  double C = 0.0;
  for (int c = 0; c < d; ++c)
    C += q[c] * ((double)qmin_g[c] + (double)qscale_g[c] * (ldexp(1.0, 4 - t[c]) - 1.0) / 2.0);
  for (int64_t i = 0; i < n; ++i) out[i] = C;
  for (int c = 0; c < d; ++c)
    for (int j = 0; j < t[c]; ++j) {
      double wgt = q[c] * (double)qscale_g[c] * ldexp(1.0, 3 - j);
      const uint32_t *row = planes_g + ((int64_t)c * 4 + j) * W;
      for (int64_t i = 0; i < n; ++i)
        if ((row[i / 32] >> (i % 32)) & 1u) out[i] += wgt;
    }
}

/* ---- top-k ---------------------------------------------------------------- */

typedef struct {
  double s;
  int64_t i;
} scored_t;

static int scored_order(const void *pa, const void *pb) {
  const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return a->i < b->i ? -1 : (a->i > b->i ? 1 : 0);
}

/* Brute force: sort all n by (score desc, index asc), keep the first k
 * (abstract: the scan ranks every one of the n keys for the top-k step). */
void oracle_topk(const double *scores, int64_t n, int k, int32_t *idx, double *val) {
  scored_t *all = (scored_t *)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
  for (int64_t i = 0; i < n; ++i) {
    all[i].s = scores[i];
    all[i].i = i;
  }
  qsort(all, (size_t)n, sizeof(scored_t), scored_order);
  for (int r = 0; r < k; ++r) {
    if (r < n) {
      idx[r] = (int32_t)all[r].i;
      val[r] = all[r].s;
    } else {
      idx[r] = -1;
      val[r] = -INFINITY;
    }
  }
  free(all);
}
