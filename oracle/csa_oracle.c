/*
 * CSA / HCA attention-layer core: float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the parity reference for the CUDA
 * library and the timed CPU baseline.  Only the test suite, the smoke check of
 * the package entry module and the CPU-baseline leg of the benchmark may load
 * it.  It shares no code, header, table or helper with the CUDA path.
 *
 * Everything here is a literal, slow restatement of the method in double
 * precision, one query row at a time (OpenMP spreads rows over host cores).
 * Sources, by page title and section:
 *   [P1] "DeepSeek-V4：迈向高效百万 Token 上下文智能" (summary/translation of
 *        the DeepSeek-V4 report), §3.3 "CSA 与 HCA 混合注意力" -- compression,
 *        lightning indexer, top-k, shared-KV MQA, HCA, RMSNorm, partial RoPE
 *        with the output rotated again at position -i, sliding window;
 *        §3.5 "通用基础设施" -- classical KV blocks and the tail of an
 *        unfinished block.
 *   [P2] "DeepSeek V4 完整技术报告", section "混合注意力：CSA + HCA" -- window of
 *        128 tokens, top-k 512/1024, RoPE on the last 64 dims, learnable sink
 *        logits that let total attention weight fall below one.
 *
 * Readings taken where the pages are silent (each is repeated at its use):
 *   R1 overlap: entry s pools group a over its own block [m s, m s + m) and
 *      group b over the previous block [m(s-1), m s); entry 0 has no b slots.
 *   R2 compression logits are per channel (z_cols == c) or one per token
 *      (z_cols == 1, broadcast over channels); softmax per channel.
 *   R4 N = floor(T / m); tail tokens make no entry.
 *   R5 RMSNorm has unit gain and eps (1e-6 by default), over all c dims;
 *      it is applied to the query, to compressed entries and to window rows.
 *   R6 RoPE rotates interleaved pairs (c-r+2i, c-r+2i+1) of the last r dims by
 *      angle p * base^(-2i/r); an entry sits at position pos0 + m s, window
 *      row j at pos0 + j, a query at its own position; the output is rotated
 *      by -pos.
 *   R7 logit scale 1/sqrt(c) unless given.
 *   R8 the sink is a per-head logit in the softmax denominator with a zero
 *      value; absent sink == -inf.
 *   R9 the window holds the n_win positions pos-n_win+1 .. pos (own token
 *      included), taken from the per-token rows (group a for CSA).
 *   R10 one joint softmax over sink, selected entries and window rows.
 *   R12 top-k order: larger score first, ties to the lower entry index; the
 *      selected set is emitted in ascending index order, padded with -1.
 *   R13 entry s is visible to a query at position pos iff its last token
 *      m(s+1)-1 <= pos, i.e. s < floor((pos+1)/m).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_NO_NORM 1u
#define ORC_NO_ROPE 2u

typedef struct {
  int32_t c;          /* entry / head dim */
  int32_t rope_dims;  /* r: RoPE acts on the last r dims (even) */
  double rope_base;   /* theta base (10000) */
  double norm_eps;    /* RMSNorm epsilon */
  uint32_t flags;     /* ORC_NO_NORM | ORC_NO_ROPE (used only by tests) */
} orc_fmt;

/* ---- the two per-vector transforms of [P1 §3.3, last paragraph] ---------- */

/* RMSNorm with unit gain (R5): y = x / sqrt(mean(x^2) + eps). */
static void orc_rmsnorm_inplace(double* x, int c, double eps) {
  double ss = 0.0;
  for (int i = 0; i < c; ++i) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss / (double)c + eps);
  for (int i = 0; i < c; ++i) x[i] *= inv;
}

/* Partial RoPE on the last r dims at position p (R6). */
static void orc_rope_inplace(double* x, int c, int r, double base, double p) {
  int d0 = c - r;
  for (int i = 0; i < r / 2; ++i) {
    double theta = pow(base, -2.0 * (double)i / (double)r);
    double a = p * theta;
    double cs = cos(a), sn = sin(a);
    double x0 = x[d0 + 2 * i], x1 = x[d0 + 2 * i + 1];
    x[d0 + 2 * i] = x0 * cs - x1 * sn;
    x[d0 + 2 * i + 1] = x0 * sn + x1 * cs;
  }
}

/* The transform a stored KV entry (or a query) receives before attention. */
static void orc_norm_rope(double* x, const orc_fmt* f, double pos) {
  if (!(f->flags & ORC_NO_NORM)) orc_rmsnorm_inplace(x, f->c, f->norm_eps);
  if (!(f->flags & ORC_NO_ROPE)) orc_rope_inplace(x, f->c, f->rope_dims, f->rope_base, pos);
}

/* Exported single-vector forms, so tests can pin each transform by itself. */
void orc_rmsnorm(int32_t c, double eps, const double* x, double* y) {
  memcpy(y, x, sizeof(double) * (size_t)c);
  orc_rmsnorm_inplace(y, c, eps);
}

void orc_rope(int32_t c, int32_t r, double base, double pos, const double* x, double* y) {
  memcpy(y, x, sizeof(double) * (size_t)c);
  orc_rope_inplace(y, c, r, base, pos);
}

/* R13: number of compressed entries (rate 1/m) visible at query position pos. */
int64_t orc_visible(int64_t pos, int32_t m, int64_t n_entries) {
  if (pos < 0) return 0;
  int64_t v = (pos + 1) / m;
  return v < n_entries ? v : n_entries;
}

/* ---- (1) softmax-gated compression [P1 §3.3, CSA and HCA paragraphs] ----- */

/*
 * Pools one entry: softmax over the listed token slots of the per-channel
 * compression logits, then the weighted sum of the token rows.
 * rows/logits: n_slots pointers to a [c] value row and a [z_cols] logit row.
 * weights_out (optional): [n_slots][c] softmax weights.
 */
static void orc_pool(int c, int n_slots, const double* const* rows, const double* const* logits,
                     int z_cols, double* out, double* weights_out) {
  for (int ch = 0; ch < c; ++ch) {
    int zc = (z_cols == 1) ? 0 : ch;
    double mx = -INFINITY;
    for (int j = 0; j < n_slots; ++j)
      if (logits[j][zc] > mx) mx = logits[j][zc];
    double den = 0.0;
    for (int j = 0; j < n_slots; ++j) den += exp(logits[j][zc] - mx);
    double acc = 0.0;
    for (int j = 0; j < n_slots; ++j) {
      double wgt = exp(logits[j][zc] - mx) / den;
      acc += wgt * rows[j][ch];
      if (weights_out) weights_out[(size_t)j * c + ch] = wgt;
    }
    out[ch] = acc;
  }
}

/*
 * CSA compression, rate exactly 1/m with overlapping groups (R1, R2, R4).
 * ca, cb, za, zb: [T][c] (logits [T][z_cols]); entries: [T/m][c], stored
 * RMSNorm'd and rotated at position pos0 + m*s.
 * weights (optional): [T/m][2m][c]; slot order a_0..a_{m-1}, b_0..b_{m-1};
 * missing b slots of entry 0 get weight 0.
 */
void orc_csa_compress(int64_t T, int32_t m, const orc_fmt* f, const double* ca, const double* cb,
                      const double* za, const double* zb, int32_t z_cols, int64_t pos0,
                      double* entries, double* weights) {
  int c = f->c;
  int64_t n = T / m;
#pragma omp parallel for schedule(static)
  for (int64_t s = 0; s < n; ++s) {
    const double* rows[512];
    const double* lg[512];
    int ns = 0;
    for (int j = 0; j < m; ++j) {
      int64_t tok = m * s + j;
      rows[ns] = ca + tok * c;
      lg[ns] = za + tok * z_cols;
      ++ns;
    }
    if (s >= 1) {
      for (int j = 0; j < m; ++j) {
        int64_t tok = m * (s - 1) + j;
        rows[ns] = cb + tok * c;
        lg[ns] = zb + tok * z_cols;
        ++ns;
      }
    }
    double* e = entries + s * c;
    double* wts = weights ? weights + (size_t)s * 2 * m * c : NULL;
    if (wts) memset(wts, 0, sizeof(double) * (size_t)2 * m * c);
    orc_pool(c, ns, rows, lg, z_cols, e, wts);
    orc_norm_rope(e, f, (double)(pos0 + m * s));
  }
}

/*
 * HCA compression: one group, rate 1/m', no overlap [P1 §3.3, HCA paragraph].
 * kv, z: [T][c] ([T][z_cols]); entries [T/m'][c] at position pos0 + m' s.
 * weights (optional): [T/m'][m'][c].
 */
void orc_hca_compress(int64_t T, int32_t mp, const orc_fmt* f, const double* kv, const double* z,
                      int32_t z_cols, int64_t pos0, double* entries, double* weights) {
  int c = f->c;
  int64_t n = T / mp;
#pragma omp parallel for schedule(static)
  for (int64_t s = 0; s < n; ++s) {
    const double** rows = (const double**)malloc(sizeof(double*) * (size_t)mp);
    const double** lg = (const double**)malloc(sizeof(double*) * (size_t)mp);
    for (int j = 0; j < mp; ++j) {
      rows[j] = kv + (mp * s + j) * c;
      lg[j] = z + (mp * s + j) * z_cols;
    }
    double* e = entries + s * c;
    orc_pool(c, mp, rows, lg, z_cols, e, weights ? weights + (size_t)s * mp * c : NULL);
    orc_norm_rope(e, f, (double)(pos0 + mp * s));
    free(rows);
    free(lg);
  }
}

/* Window rows: win[j] = RoPE_{pos0+j}(RMSNorm(kv[j])) (R5, R6, R9). */
void orc_window_rows(int64_t T, const orc_fmt* f, const double* kv, int64_t pos0, double* win) {
  int c = f->c;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < T; ++j) {
    memcpy(win + j * c, kv + j * c, sizeof(double) * (size_t)c);
    orc_norm_rope(win + j * c, f, (double)(pos0 + j));
  }
}

/* ---- (2) lightning indexer and top-k [P1 §3.3, CSA paragraph] ----------- */

/*
 * I[t,s] = sum_h w[t,h] * ReLU(q_I[t,h] . K_I[s]) for every visible s (R13);
 * invisible entries get -inf.
 * q_I: [Tq][H_I][d_I]; w: [Tq][H_I]; k_I: [N][d_I]; q_pos: [Tq];
 * scores: [Tq][N].
 */
void orc_indexer_scores(int64_t Tq, int32_t HI, int32_t dI, int64_t N, const double* qI,
                        const double* w, const double* kI, const int64_t* q_pos, int32_t m,
                        double* scores) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < Tq; ++t) {
    int64_t vis = orc_visible(q_pos[t], m, N);
    double* row = scores + t * N;
    for (int64_t s = 0; s < N; ++s) {
      if (s >= vis) {
        row[s] = -INFINITY;
        continue;
      }
      double acc = 0.0;
      for (int h = 0; h < HI; ++h) {
        const double* q = qI + (t * HI + h) * dI;
        const double* k = kI + s * dI;
        double dot = 0.0;
        for (int d = 0; d < dI; ++d) dot += q[d] * k[d];
        acc += w[t * HI + h] * (dot > 0.0 ? dot : 0.0);
      }
      row[s] = acc;
    }
  }
}

typedef struct {
  double score;
  int64_t s;
} orc_cand;

/* R12: descending score, ties to the lower index -- a strict total order. */
static int orc_cand_cmp(const void* pa, const void* pb) {
  const orc_cand* a = (const orc_cand*)pa;
  const orc_cand* b = (const orc_cand*)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->s < b->s) ? -1 : (a->s > b->s) ? 1 : 0;
}

static int orc_i32_cmp(const void* pa, const void* pb) {
  int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
  return (a > b) - (a < b);
}

/*
 * Causal per-query top-k over the visible entries; idx: [Tq][k], ascending,
 * padded with -1 when fewer than k entries are visible.
 */
void orc_topk(int64_t Tq, int64_t N, const double* scores, const int64_t* q_pos, int32_t m,
              int32_t k, int32_t* idx) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < Tq; ++t) {
    int64_t vis = orc_visible(q_pos[t], m, N);
    orc_cand* cand = (orc_cand*)malloc(sizeof(orc_cand) * (size_t)(vis > 0 ? vis : 1));
    for (int64_t s = 0; s < vis; ++s) {
      cand[s].score = scores[t * N + s];
      cand[s].s = s;
    }
    qsort(cand, (size_t)vis, sizeof(orc_cand), orc_cand_cmp);
    int64_t keff = vis < k ? vis : k;
    int32_t* out = idx + t * k;
    for (int64_t i = 0; i < keff; ++i) out[i] = (int32_t)cand[i].s;
    qsort(out, (size_t)keff, sizeof(int32_t), orc_i32_cmp);
    for (int64_t i = keff; i < k; ++i) out[i] = -1;
    free(cand);
  }
}

/* ---- (3) shared-KV MQA with window and sink [P1 §3.3; P2] ---------------- */

/*
 * One attention layer output for Tq query rows.
 *   q: [Tq][H][c] raw queries; q_pos: [Tq] absolute positions.
 *   entries: [N][c] stored (transformed) compressed entries.
 *   idx: [Tq][k] selected entries (CSA) or NULL for dense HCA, where every
 *        visible entry s < floor((pos+1)/m_dense) is used.
 *   win: [Tw][c] stored window rows, row j at position win_pos0 + j.
 *   sink: [H] logits or NULL (== -inf).
 *   out: [Tq][H][c]; lse (optional): [Tq][H] natural log of the softmax
 *        denominator (sink term included).
 * One joint softmax over {sink} U selected entries U window rows (R8-R10),
 * logits scale * q^ . key with q^ = RoPE_pos(RMSNorm(q)), then the weighted
 * sum of the same rows (K = V), then the output rotated by -pos.
 */
void orc_attention(int64_t Tq, int32_t H, const orc_fmt* f, const double* q, const int64_t* q_pos,
                   const double* entries, int64_t N, const int32_t* idx, int32_t k, int32_t m_dense,
                   const double* win, int64_t Tw, int64_t win_pos0, int32_t n_win,
                   const double* sink, double scale, double* out, double* lse) {
  int c = f->c;
  if (!(scale > 0.0)) scale = 1.0 / sqrt((double)c);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < Tq; ++t) {
    int64_t pos = q_pos[t];
    /* key list for this query row */
    int64_t cap = (idx ? k : (N > 0 ? N : 0)) + n_win + 1;
    const double** keys = (const double**)malloc(sizeof(double*) * (size_t)cap);
    int64_t nk = 0;
    if (idx) {
      for (int i = 0; i < k; ++i) {
        int32_t s = idx[t * k + i];
        if (s >= 0 && s < N) keys[nk++] = entries + (int64_t)s * c;
      }
    } else {
      int64_t vis = orc_visible(pos, m_dense, N);
      for (int64_t s = 0; s < vis; ++s) keys[nk++] = entries + s * c;
    }
    int64_t jlo = pos - n_win + 1;
    if (jlo < win_pos0) jlo = win_pos0;
    int64_t jhi = pos;
    if (jhi > win_pos0 + Tw - 1) jhi = win_pos0 + Tw - 1;
    for (int64_t j = jlo; j <= jhi; ++j) keys[nk++] = win + (j - win_pos0) * c;

    double* qh = (double*)malloc(sizeof(double) * (size_t)c);
    double* lg = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    for (int h = 0; h < H; ++h) {
      memcpy(qh, q + (t * H + h) * c, sizeof(double) * (size_t)c);
      orc_norm_rope(qh, f, (double)pos);
      double zs = sink ? sink[h] : -INFINITY;
      double mx = zs;
      for (int64_t i = 0; i < nk; ++i) {
        double d = 0.0;
        for (int e = 0; e < c; ++e) d += qh[e] * keys[i][e];
        lg[i] = scale * d;
        if (lg[i] > mx) mx = lg[i];
      }
      double den = isinf(zs) && zs < 0 ? 0.0 : exp(zs - mx);
      double* o = out + (t * H + h) * c;
      for (int e = 0; e < c; ++e) o[e] = 0.0;
      for (int64_t i = 0; i < nk; ++i) {
        double p = exp(lg[i] - mx);
        den += p;
        for (int e = 0; e < c; ++e) o[e] += p * keys[i][e];
      }
      for (int e = 0; e < c; ++e) o[e] = (den > 0.0) ? o[e] / den : 0.0;
      if (!(f->flags & ORC_NO_ROPE)) orc_rope_inplace(o, c, f->rope_dims, f->rope_base, -(double)pos);
      if (lse) lse[t * H + h] = log(den) + mx;
    }
    free(qh);
    free(lg);
    free(keys);
  }
}

/* ---- (next) block-scaled FP8 indexer inputs ------------------------------ */
/*
 * The pages run the indexer's QK product in low precision ([P1] §3.3, last
 * paragraph: an FP4 lightning indexer that keeps almost all of the bf16
 * top-k).  These functions restate the OCP Microscaling (MX) format for that
 * path with FP8 E4M3 elements (the FN variant: no infinities; 0x7f and 0xff
 * are NaN; largest finite 448): blocks of 32 consecutive elements share one
 * power-of-two scale X = 2^(floor(log2(amax)) - 8), 8 being E4M3's largest
 * exponent; each element is the E4M3 value nearest to v / X (ties to the code
 * with an even mantissa), saturated to +-448.
 */

/* Value of an E4M3 code. */
double orc_e4m3_value(uint8_t code) {
  int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -mag : mag;
}

/* Nearest E4M3 code to x by search over every finite magnitude code; ties go
 * to the even code; |x| beyond 448 saturates; NaN maps to 0x7f. */
uint8_t orc_e4m3_encode(double x) {
  if (isnan(x)) return 0x7f;
  double a = fabs(x);
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c < 0x7f; ++c) {   /* 0x00 .. 0x7e: every finite magnitude */
    double err = fabs(orc_e4m3_value((uint8_t)c) - a);
    if (err < best_err || (err == best_err && (c & 1) == 0)) {
      best = c;
      best_err = err;
    }
  }
  /* the sign is kept, zero included: a negative value that rounds to zero is -0 */
  return (uint8_t)(signbit(x) ? (best | 0x80) : best);
}

/* MX quantization of n elements (n a multiple of 32): codes[n], exps[n/32]
 * (the scale exponent; an all-zero block gets -127). */
void orc_mxfp8_quantize(int64_t n, const double* x, uint8_t* codes, int32_t* exps) {
  for (int64_t b = 0; b < n / 32; ++b) {
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) {
      double a = fabs(x[b * 32 + i]);
      if (a > amax) amax = a;
    }
    int e = -127;
    if (amax > 0.0) {
      e = (int)floor(log2(amax)) - 8;
      if (e < -127) e = -127;
      if (e > 127) e = 127;
    }
    exps[b] = e;
    for (int i = 0; i < 32; ++i) codes[b * 32 + i] = orc_e4m3_encode(ldexp(x[b * 32 + i], -e));
  }
}

void orc_mxfp8_dequantize(int64_t n, const uint8_t* codes, const int32_t* exps, double* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = ldexp(orc_e4m3_value(codes[i]), exps[i / 32]);
}

/*
 * The same MX scheme with FP4 E2M1 elements (the pages' indexer precision):
 * 4-bit codes, sign bit 3, a 2-bit exponent with bias 1 and one mantissa bit,
 * so the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6; blocks of 32 share the
 * scale 2^(floor(log2(amax)) - 2), 2 being E2M1's largest exponent.
 */
double orc_e2m1_value(uint8_t code) {
  int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
  return sign ? -mag : mag;
}

/* Nearest E2M1 code (ties to the even code), saturating at +-6. */
uint8_t orc_e2m1_encode(double x) {
  double a = fabs(x);
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c < 8; ++c) {
    double err = fabs(orc_e2m1_value((uint8_t)c) - a);
    if (err < best_err || (err == best_err && (c & 1) == 0)) {
      best = c;
      best_err = err;
    }
  }
  return (uint8_t)(signbit(x) ? (best | 8) : best);   /* sign kept, -0 included */
}

void orc_mxfp4_quantize(int64_t n, const double* x, uint8_t* codes, int32_t* exps) {
  for (int64_t b = 0; b < n / 32; ++b) {
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) {
      double a = fabs(x[b * 32 + i]);
      if (a > amax) amax = a;
    }
    int e = -127;
    if (amax > 0.0) {
      e = (int)floor(log2(amax)) - 2;
      if (e < -127) e = -127;
      if (e > 127) e = 127;
    }
    exps[b] = e;
    for (int i = 0; i < 32; ++i) codes[b * 32 + i] = orc_e2m1_encode(ldexp(x[b * 32 + i], -e));
  }
}

void orc_mxfp4_dequantize(int64_t n, const uint8_t* codes, const int32_t* exps, double* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = ldexp(orc_e2m1_value(codes[i]), exps[i / 32]);
}

/* ---- (next) streaming compression for decode ----------------------------- */
/*
 * Decode appends one token at a time ([P1] §3.5: the KV of an unfinished
 * block waits in a tail buffer until the block completes).  The state of one
 * sequence, caller-owned, for rate m and overlap (CSA) or not (HCA):
 *   state[0]                 tokens appended so far (as a double)
 *   rows:  cur_a[m][c], cur_b[m][c], prev_b[m][c]   (values)
 *   logit: cur_za[m][zc], cur_zb[m][zc], prev_zb[m][zc]
 * orc_stream_state_len() gives its length in doubles.  Each append writes the
 * token's window row; when the token completes block s it writes entry s
 * (pooled over the block's a rows and, for CSA with s >= 1, the previous
 * block's b rows, then RMSNorm and RoPE at pos0 + m s) and returns 1.
 */
int64_t orc_stream_state_len(int32_t m, int32_t c, int32_t z_cols) {
  return 1 + 3 * (int64_t)m * c + 3 * (int64_t)m * z_cols;
}

int32_t orc_stream_append(int32_t m, int32_t overlap, const orc_fmt* f, int64_t pos0,
                          const double* kv_a, const double* kv_b, const double* z_a,
                          const double* z_b, int32_t z_cols, double* state, double* win_row,
                          double* entry) {
  int c = f->c;
  int64_t t = (int64_t)state[0];
  double* cur_a = state + 1;
  double* cur_b = cur_a + (size_t)m * c;
  double* prev_b = cur_b + (size_t)m * c;
  double* cur_za = prev_b + (size_t)m * c;
  double* cur_zb = cur_za + (size_t)m * z_cols;
  double* prev_zb = cur_zb + (size_t)m * z_cols;
  int j = (int)(t % m);
  memcpy(cur_a + (size_t)j * c, kv_a, sizeof(double) * (size_t)c);
  memcpy(cur_za + (size_t)j * z_cols, z_a, sizeof(double) * (size_t)z_cols);
  if (overlap) {
    memcpy(cur_b + (size_t)j * c, kv_b, sizeof(double) * (size_t)c);
    memcpy(cur_zb + (size_t)j * z_cols, z_b, sizeof(double) * (size_t)z_cols);
  }
  memcpy(win_row, kv_a, sizeof(double) * (size_t)c);
  orc_norm_rope(win_row, f, (double)(pos0 + t));
  state[0] = (double)(t + 1);
  if (j != m - 1) return 0;
  int64_t s = t / m;
  const double** rows = (const double**)malloc(sizeof(double*) * (size_t)(2 * m));
  const double** lg = (const double**)malloc(sizeof(double*) * (size_t)(2 * m));
  int ns = 0;
  for (int i = 0; i < m; ++i, ++ns) {
    rows[ns] = cur_a + (size_t)i * c;
    lg[ns] = cur_za + (size_t)i * z_cols;
  }
  if (overlap && s >= 1) {
    for (int i = 0; i < m; ++i, ++ns) {
      rows[ns] = prev_b + (size_t)i * c;
      lg[ns] = prev_zb + (size_t)i * z_cols;
    }
  }
  orc_pool(c, ns, rows, lg, z_cols, entry, NULL);
  free(rows);
  free(lg);
  orc_norm_rope(entry, f, (double)(pos0 + m * s));
  if (overlap) {   /* this block's b rows serve the next entry */
    memcpy(prev_b, cur_b, sizeof(double) * (size_t)m * c);
    memcpy(prev_zb, cur_zb, sizeof(double) * (size_t)m * z_cols);
  }
  return 1;
}

/* ---- (next) mixed BF16 / FP8 storage of KV entries ----------------------- */
/*
 * The pages store KV entries in mixed precision ([P1] §3.3, last paragraph:
 * the RoPE dims in BF16, the rest in FP8).  Reading taken: the last r dims
 * (RoPE) are rounded to BF16; the first c - r dims are MX-FP8 (E4M3, blocks
 * of 32 along the entry, as orc_mxfp8_quantize).
 */

/* Nearest BF16 value to x (8 significant bits, ties to even, the exponent
 * range of float32 with its subnormals; beyond the largest finite: inf). */
double orc_bf16_round(double x) {
  if (x == 0.0 || isnan(x) || isinf(x)) return x;
  int e = (int)floor(log2(fabs(x)));
  if (e < -126) e = -126;                 /* subnormal spacing 2^-133 */
  double q = ldexp(1.0, e - 7);
  double y = rint(x / q) * q;             /* rint: round half to even */
  if (fabs(y) > ldexp(2.0 - ldexp(1.0, -7), 127)) return x > 0 ? INFINITY : -INFINITY;
  return y;
}

/* Stores n entries of c dims (c - r a multiple of 32): codes[n][c-r],
 * exps[n][(c-r)/32], rope[n][r] (BF16 values held as doubles); loads them
 * back into out[n][c]. */
void orc_mixed_store(int64_t n, int32_t c, int32_t r, const double* x, uint8_t* codes,
                     int32_t* exps, double* rope) {
  int cq = c - r;
  for (int64_t i = 0; i < n; ++i) {
    orc_mxfp8_quantize(cq, x + i * c, codes + i * cq, exps + i * (cq / 32));
    for (int d = 0; d < r; ++d) rope[i * r + d] = orc_bf16_round(x[i * c + cq + d]);
  }
}

void orc_mixed_load(int64_t n, int32_t c, int32_t r, const uint8_t* codes, const int32_t* exps,
                    const double* rope, double* out) {
  int cq = c - r;
  for (int64_t i = 0; i < n; ++i) {
    orc_mxfp8_dequantize(cq, codes + i * cq, exps + i * (cq / 32), out + i * c);
    for (int d = 0; d < r; ++d) out[i * c + cq + d] = rope[i * r + d];
  }
}

/*
 * FP4 with finer scales (the NVFP4 layout): blocks of 16 elements, each with
 * an E4M3 scale, under one float scale per tensor g = amax / (448 * 6).  A
 * block's scale is the E4M3 value nearest to amax_block / (6 g); its elements
 * are the E2M1 codes nearest to v / (scale g) (an all-zero scale leaves the
 * block at zero).
 */
void orc_nvfp4_quantize(int64_t n, const double* x, uint8_t* codes, uint8_t* scales,
                        double* gscale) {
  double amax = 0.0;
  for (int64_t i = 0; i < n; ++i)
    if (fabs(x[i]) > amax) amax = fabs(x[i]);
  double g = amax > 0.0 ? amax / (448.0 * 6.0) : 1.0;
  *gscale = g;
  for (int64_t b = 0; b < n / 16; ++b) {
    double bmax = 0.0;
    for (int i = 0; i < 16; ++i)
      if (fabs(x[b * 16 + i]) > bmax) bmax = fabs(x[b * 16 + i]);
    uint8_t sc = orc_e4m3_encode(bmax / (6.0 * g));
    scales[b] = sc;
    double s = orc_e4m3_value(sc) * g;
    for (int i = 0; i < 16; ++i) codes[b * 16 + i] = s > 0.0 ? orc_e2m1_encode(x[b * 16 + i] / s) : 0;
  }
}

void orc_nvfp4_dequantize(int64_t n, const uint8_t* codes, const uint8_t* scales, double gscale,
                          double* y) {
  for (int64_t i = 0; i < n; ++i)
    y[i] = orc_e2m1_value(codes[i]) * orc_e4m3_value(scales[i / 16]) * gscale;
}
