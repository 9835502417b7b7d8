/*
 * oracle.c -- plain fp64 CPU oracle for DuoAttention's hybrid-head attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference leg may load this library.  It shares no code with the
 * CUDA library (no headers, helpers or tables) and is deliberately slow: no
 * blocking, no fusion, no reordering beyond what the definitions state.
 *
 * Sources (DuoAttention: Efficient Long-Context LLM Inference with Retrieval and
 * Streaming Heads, arXiv 2410.10819, as explained on the paper-graph-ui page):
 *   - "The Full and Streaming Attention Masks": full_attn = softmax(QK^T (.) M_causal) V,
 *     streaming_attn = softmax(QK^T (.) M_streaming) V; M_causal admits key q <= query p;
 *     M_streaming is the Lambda mask: the first S sink tokens plus the recent tokens,
 *     every other logit set to -inf before the softmax.
 *   - "Deployment Architecture / Decoding Procedure", steps 1-5: retrieval heads attend
 *     over the full cache, streaming heads over sinks + recent tokens; the streaming
 *     cache evicts the oldest token that is neither a sink nor recent.
 *   - "Chunked Pre-filling", Figure 5 (right): after every chunk the streaming cache is
 *     pruned to sinks + recent tokens.
 *   - KV memory (H_r L + H_s (S+R)) d ("Decoding Procedure") and the full-attention
 *     KV size 2 D H L d ("The Core Problem").
 *   - OpenReview rebuttal, "RazorAttention and Echo Heads": the KV budget ratio.
 *
 * Readings where the pages leave a step open (each also listed in the design notes):
 *   R1 the recent window W counts the query's own token: key j is recent for
 *      query i iff i - j < W (so the streaming cache holds exactly S + W tokens);
 *   R2 every query row of a chunk uses the Lambda mask of its own position;
 *   R3 logits are scaled by 1/sqrt(d) unless a scale is given; the mask is an
 *      additive -inf before the softmax;
 *   R6 decode appends the new token first, then attends (the token sees itself);
 *   R7 ring slot of position p is p (p < S) or S + (p mod W);
 *   R8 query head h uses KV head h / (Hq / Hkv);
 *   R9 INT4: one group = one token's row of a head; fp32 min/max; scale =
 *      fp16((max-min)/15), zero = fp16(min); code = clamp(rint((x-zero)/scale),0,15);
 *      element 2t in the low nibble of byte t; dequant = code*scale + zero.
 *   R14 FP8: one group = one token's row of a head; amax = fp32 max |x|; scale =
 *      amax / 448 in IEEE fp32 (kept as fp32); code = the OCP E4M3 value nearest to
 *      x / scale (fp32 division), ties to even mantissa, magnitudes past 448 held at
 *      448; amax = 0 gives scale 0 and zero codes; dequant = value(code) * scale.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* element types accepted for inputs; every conversion to double is exact */
enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

static double load_elem(const void *base, int dtype, int64_t idx) {
  if (dtype == ORC_F64) return ((const double *)base)[idx];
  if (dtype == ORC_F32) return (double)((const float *)base)[idx];
  /* bf16: the upper 16 bits of an IEEE single */
  uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Mutations used only by the tests that show the pins can fail (0 = none). */
enum {
  MUT_NONE = 0,
  MUT_WINDOW_INCLUSIVE = 1, /* i - j <= W instead of i - j < W            */
  MUT_SINK_OFF_BY_ONE = 2,  /* j <= S instead of j < S                     */
  MUT_NO_SCALE = 3,         /* drop the 1/sqrt(d) logit scale              */
  MUT_NON_CAUSAL = 4,       /* retrieval heads see future keys             */
  MUT_WRONG_GROUP = 5,      /* query head h uses KV head h % Hkv           */
  MUT_LSE_NO_MAX = 6,       /* lse drops the max term                      */
  MUT_V_FROM_K = 7          /* output mixes K rows instead of V rows       */
};

/* Key j is visible to query position i (masks of "The Full and Streaming
 * Attention Masks", readings R1-R2). */
static int visible_mut(int64_t i, int64_t j, int is_retrieval, int64_t S, int64_t W, int mut) {
  if (mut == MUT_NON_CAUSAL && is_retrieval) return 1;
  if (j > i) return 0; /* M_causal: the query sees itself and earlier keys */
  if (is_retrieval) return 1;
  if (mut == MUT_SINK_OFF_BY_ONE ? (j <= S) : (j < S)) return 1; /* attention sinks */
  if (mut == MUT_WINDOW_INCLUSIVE) return i - j <= W;
  return i - j < W; /* recent window, current token included (R1) */
}

int oracle_visible(int64_t i, int64_t j, int is_retrieval, int64_t S, int64_t W) {
  return visible_mut(i, j, is_retrieval, S, W, MUT_NONE);
}

/*
 * Masked softmax attention, written out from its definition.
 *
 *   q   [B][nq][Hq][d]  query row r sits at absolute position pos0 + r
 *   k,v [B][Lk][Hkv][d] the dense key/value history, positions 0..Lk-1
 *                       (nothing evicted: the mask alone decides visibility)
 *   retr[Hkv]           1 = retrieval head (causal mask), 0 = streaming (Lambda)
 *   scale               logit scale; <= 0 means 1/sqrt(d)
 *   rows, nrows         optional list of flattened (b, r, h) rows to evaluate
 *                       (row id = (b*nq + r)*Hq + h); NULL = every row
 *   out                 [nrows or B*nq*Hq][d] fp64
 *   lse                 [nrows or B*nq*Hq] natural-log sum of exp of the scaled
 *                       visible logits (nullable)
 * Returns 0, or -1 if a query position has no key history (pos0 + nq > Lk).
 */
int oracle_attend(int B, int64_t nq, int Hq, int Hkv, int d, const void *q, int q_dtype, int64_t pos0,
                  const void *k, const void *v, int kv_dtype, int64_t Lk, const uint8_t *retr, int64_t S,
                  int64_t W, double scale, const int64_t *rows, int64_t nrows, double *out, double *lse,
                  int mut) {
  if (pos0 + nq > Lk) return -1;
  if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
  if (mut == MUT_NO_SCALE) scale = 1.0;
  const int G = Hq / Hkv;
  const int64_t total = rows ? nrows : (int64_t)B * nq * Hq;
  int bad = 0;

#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    if (!s || !o) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < total; ++t) {
      if (!s || !o) continue;
      const int64_t id = rows ? rows[t] : t;
      const int h = (int)(id % Hq);
      const int64_t r = (id / Hq) % nq;
      const int64_t b = id / ((int64_t)Hq * nq);
      const int g = (mut == MUT_WRONG_GROUP) ? (h % Hkv) : (h / G);
      const int64_t i = pos0 + r;
      const int is_r = retr[g] ? 1 : 0;
      const int64_t qoff = ((b * nq + r) * Hq + h) * (int64_t)d;
      const int64_t jmax = (mut == MUT_NON_CAUSAL && is_r) ? Lk - 1 : i;

      /* pass 1: scaled logits of the visible keys and their maximum */
      double m = -INFINITY;
      for (int64_t j = 0; j <= jmax; ++j) {
        if (!visible_mut(i, j, is_r, S, W, mut)) continue;
        const int64_t koff = ((b * Lk + j) * Hkv + g) * (int64_t)d;
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += load_elem(q, q_dtype, qoff + e) * load_elem(k, kv_dtype, koff + e);
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
      }
      /* pass 2: softmax normaliser Z and the weighted sum of value rows */
      double Z = 0.0;
      for (int e = 0; e < d; ++e) o[e] = 0.0;
      for (int64_t j = 0; j <= jmax; ++j) {
        if (!visible_mut(i, j, is_r, S, W, mut)) continue;
        const double w = exp(s[j] - m);
        Z += w;
        const int64_t voff = ((b * Lk + j) * Hkv + g) * (int64_t)d;
        const void *src = (mut == MUT_V_FROM_K) ? k : v;
        for (int e = 0; e < d; ++e) o[e] += w * load_elem(src, kv_dtype, voff + e);
      }
      for (int e = 0; e < d; ++e) out[t * d + e] = o[e] / Z;
      if (lse) lse[t] = (mut == MUT_LSE_NO_MAX) ? log(Z) : m + log(Z);
    }
    free(s);
    free(o);
  }
  return bad ? -2 : 0;
}

/*
 * Gated mixed attention of the identification phase ("Gate Parameterization"): for
 * KV head g with gate alpha[g] in [0, 1], the output of each of its query heads is
 *   alpha[g] * full_attn + (1 - alpha[g]) * streaming_attn
 * with full_attn under the causal mask and streaming_attn under the Lambda mask ("The
 * Full and Streaming Attention Masks"), both over the same scaled logits.
 *
 *   q [B][L][Hq][d], k, v [B][L][Hkv][d]: one sequence per batch entry, positions 0..L-1
 *   alpha [Hkv] fp64; rows / nrows / out as in oracle_attend (row id = (b*L + i)*Hq + h)
 */
int oracle_gated(int B, int64_t L, int Hq, int Hkv, int d, const void *q, int q_dtype, const void *k,
                 const void *v, int kv_dtype, const double *alpha, int64_t S, int64_t W, double scale,
                 const int64_t *rows, int64_t nrows, double *out) {
  if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
  const int G = Hq / Hkv;
  const int64_t total = rows ? nrows : (int64_t)B * L * Hq;
  int bad = 0;

#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *of = (double *)malloc(sizeof(double) * (size_t)d);
    double *os = (double *)malloc(sizeof(double) * (size_t)d);
    if (!s || !of || !os) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < total; ++t) {
      if (!s || !of || !os) continue;
      const int64_t id = rows ? rows[t] : t;
      const int h = (int)(id % Hq);
      const int64_t i = (id / Hq) % L;
      const int64_t b = id / ((int64_t)Hq * L);
      const int g = h / G;
      const int64_t qoff = ((b * L + i) * Hq + h) * (int64_t)d;

      /* the scaled logits of every key the causal mask admits, and both maxima */
      double mf = -INFINITY, ms = -INFINITY;
      for (int64_t j = 0; j <= i; ++j) {
        const int64_t koff = ((b * L + j) * Hkv + g) * (int64_t)d;
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += load_elem(q, q_dtype, qoff + e) * load_elem(k, kv_dtype, koff + e);
        s[j] = scale * dot;
        if (s[j] > mf) mf = s[j];
        if (oracle_visible(i, j, 0, S, W) && s[j] > ms) ms = s[j];
      }
      /* two softmax normalisers and two weighted sums of the value rows */
      double Zf = 0.0, Zs = 0.0;
      for (int e = 0; e < d; ++e) of[e] = os[e] = 0.0;
      for (int64_t j = 0; j <= i; ++j) {
        const int64_t voff = ((b * L + j) * Hkv + g) * (int64_t)d;
        const double wf = exp(s[j] - mf);
        Zf += wf;
        for (int e = 0; e < d; ++e) of[e] += wf * load_elem(v, kv_dtype, voff + e);
        if (oracle_visible(i, j, 0, S, W)) {
          const double ws = exp(s[j] - ms);
          Zs += ws;
          for (int e = 0; e < d; ++e) os[e] += ws * load_elem(v, kv_dtype, voff + e);
        }
      }
      const double a = alpha[g];
      for (int e = 0; e < d; ++e) out[t * d + e] = a * (of[e] / Zf) + (1.0 - a) * (os[e] / Zs);
    }
    free(s);
    free(of);
    free(os);
  }
  return bad ? -2 : 0;
}

/*
 * Retained set of a streaming head after `len` tokens, in closed form:
 * the sinks {p < min(S, len)} and the recent tokens {max(S, len-W) <= p < len}
 * ("Decoding Procedure" step 3 and Figure 5, reading R1).
 */
void oracle_retained(int64_t len, int64_t S, int64_t W, uint8_t *mask) {
  for (int64_t p = 0; p < len; ++p) {
    const int sink = p < S;
    const int recent = (p >= S) && (p >= len - W);
    mask[p] = (uint8_t)(sink || recent);
  }
}

/*
 * Replays appends into one streaming head's cache of S sink slots and W ring
 * slots, one position at a time, in the order the tokens arrive (reading R7:
 * slot(p) = p for p < S, else S + (p mod W); writing a ring slot evicts the
 * position it held).  chunk_lens[c] tokens arrive in chunk c; after each chunk
 * the position held by every slot is written to slots_out[c][S+W] (-1 = empty).
 */
void oracle_ring_replay(int64_t S, int64_t W, int nchunks, const int64_t *chunk_lens, int64_t *slots_out) {
  const int64_t nslots = S + W;
  int64_t *slot = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nslots > 0 ? nslots : 1));
  for (int64_t s = 0; s < nslots; ++s) slot[s] = -1;
  int64_t p = 0;
  for (int c = 0; c < nchunks; ++c) {
    for (int64_t t = 0; t < chunk_lens[c]; ++t, ++p) {
      if (p < S) slot[p] = p;
      else slot[S + (p % W)] = p;
    }
    memcpy(slots_out + (int64_t)c * nslots, slot, sizeof(int64_t) * (size_t)nslots);
  }
  free(slot);
}

/* ---- INT4 asymmetric quantisation, reading R9 (fp32 arithmetic, IEEE rounding) ---- */

static float fp16_round(float x, uint16_t *bits) {
  _Float16 h = (_Float16)x; /* IEEE binary16, round to nearest even */
  memcpy(bits, &h, 2);
  return (float)h;
}

static float fp16_value(uint16_t bits) {
  _Float16 h;
  memcpy(&h, &bits, 2);
  return (float)h;
}

static float load_f32(const void *base, int dtype, int64_t idx) {
  return (float)load_elem(base, dtype, idx); /* bf16 / f32 inputs are exact in f32 */
}

/*
 * x [nrows][gs] (bf16 or f32) -> codes [nrows][gs/2], scale/zero as fp16 bit patterns [nrows].
 */
void oracle_int4_quantize(int64_t nrows, int gs, const void *x, int dtype, uint8_t *codes, uint16_t *scale_bits,
                          uint16_t *zero_bits) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t base = r * gs;
    float mn = load_f32(x, dtype, base), mx = mn;
    for (int e = 1; e < gs; ++e) {
      const float f = load_f32(x, dtype, base + e);
      if (f < mn) mn = f;
      if (f > mx) mx = f;
    }
    volatile float range = mx - mn; /* volatile: keep every step a separate fp32 rounding */
    volatile float step = range / 15.0f;
    const float scale = fp16_round(step, &scale_bits[r]);
    const float zero = fp16_round(mn, &zero_bits[r]);
    for (int e = 0; e < gs; e += 2) {
      int c[2];
      for (int u = 0; u < 2; ++u) {
        int code = 0;
        if (scale != 0.0f) {
          volatile float diff = load_f32(x, dtype, base + e + u) - zero;
          volatile float ratio = diff / scale;
          float rq = rintf(ratio); /* round half to even */
          if (rq < 0.0f) rq = 0.0f;
          if (rq > 15.0f) rq = 15.0f;
          code = (int)rq;
        }
        c[u] = code;
      }
      codes[r * (gs / 2) + e / 2] = (uint8_t)(c[0] | (c[1] << 4));
    }
  }
}

/* codes [nrows][gs/2], scale/zero fp16 bits -> out [nrows][gs] fp64, value = code*scale + zero */
void oracle_int4_dequantize(int64_t nrows, int gs, const uint8_t *codes, const uint16_t *scale_bits,
                            const uint16_t *zero_bits, double *out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    const double sc = (double)fp16_value(scale_bits[r]);
    const double z = (double)fp16_value(zero_bits[r]);
    for (int e = 0; e < gs; ++e) {
      const uint8_t byte = codes[r * (gs / 2) + e / 2];
      const int code = (e & 1) ? (byte >> 4) : (byte & 15);
      out[r * gs + e] = (double)code * sc + z;
    }
  }
}

/* ---- FP8 (E4M3) quantisation with a per-row scale, reading R14 ---- */

/* OCP 8-bit floating point E4M3 ("OFP8" specification): 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; no
 * infinities, and S.1111.111 is NaN, so the largest finite magnitude is 1.75 * 2^8 =
 * 448 (S.1111.110).  This encodes a finite float by round to nearest, ties to the
 * even mantissa, holding magnitudes >= 448 at 448. */
static uint8_t e4m3_encode(float y) {
  const uint8_t sign = signbit(y) ? 0x80 : 0x00;
  const double a = fabs((double)y);
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2); /* a = f 2^e2 with f in [0.5, 1): a lies in [2^(e2-1), 2^e2) */
  int E = e2 - 1;
  if (E < -6) E = -6;                   /* subnormal range shares the step of binade -6 */
  const double step = ldexp(1.0, E - 3); /* 3 mantissa bits: 8 steps per binade */
  const double r = rint(a / step);       /* a / step is exact; rint rounds half to even */
  const double v = r * step;             /* may carry into the next binade: still <= 448 */
  if (v == 0.0) return sign;
  int ev;
  frexp(v, &ev);
  const int Ev = ev - 1;
  if (Ev < -6) return sign | (uint8_t)(v / ldexp(1.0, -9)); /* subnormal: m * 2^-9, m in 1..7 */
  const int mant = (int)(v / ldexp(1.0, Ev - 3)) - 8;       /* 1.mmm -> mmm */
  return sign | (uint8_t)((Ev + 7) << 3) | (uint8_t)mant;
}

/* value of an E4M3 code (exact in fp64); NaN codes are never produced here */
static double e4m3_value(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

double oracle_e4m3_value(uint8_t c) { return e4m3_value(c); }
uint8_t oracle_e4m3_encode(float y) { return e4m3_encode(y); }

/* x [nrows][gs] (bf16 or f32) -> codes [nrows][gs] E4M3, scales [nrows] fp32 */
void oracle_fp8_quantize(int64_t nrows, int gs, const void *x, int dtype, uint8_t *codes, float *scales) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t base = r * gs;
    float amax = 0.0f;
    for (int e = 0; e < gs; ++e) {
      const float f = fabsf(load_f32(x, dtype, base + e));
      if (f > amax) amax = f;
    }
    volatile float scale = amax / 448.0f; /* volatile: one IEEE fp32 division */
    scales[r] = scale;
    for (int e = 0; e < gs; ++e) {
      uint8_t c = 0;
      if (scale != 0.0f) {
        volatile float y = load_f32(x, dtype, base + e) / scale;
        c = e4m3_encode(y);
      }
      codes[base + e] = c;
    }
  }
}

/* codes [nrows][gs] E4M3 + scales [nrows] fp32 -> out [nrows][gs] fp64, value(code) * scale */
void oracle_fp8_dequantize(int64_t nrows, int gs, const uint8_t *codes, const float *scales, double *out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r)
    for (int e = 0; e < gs; ++e) out[r * gs + e] = e4m3_value(codes[r * gs + e]) * (double)scales[r];
}

/* ---- memory closed forms ---- */

/* Elements of K (or of V) one layer keeps: (H_r L + H_s (S+W)) d, with the
 * streaming term capped at L while the sequence is shorter than S+W. */
double oracle_layer_kv_elems(int64_t Hr, int64_t Hs, int64_t L, int64_t S, int64_t W, int64_t d) {
  const int64_t keep = (S + W < L) ? (S + W) : L;
  return (double)((Hr * L + Hs * keep) * d);
}

/* KV budget ratio: (L r + (S+W)(1-r)) / L, r = retrieval-head fraction. */
double oracle_budget_ratio(double L, double r, double SW) { return (L * r + SW * (1.0 - r)) / L; }

/* Full-attention KV bytes: 2 (K and V) x layers x heads x L x d x bytes per element. */
double oracle_full_kv_bytes(int64_t layers, int64_t heads, int64_t d, int64_t L, int64_t elem_bytes) {
  return 2.0 * (double)layers * (double)heads * (double)L * (double)d * (double)elem_bytes;
}
