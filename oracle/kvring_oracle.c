/*
 * kvring_oracle.c -- plain, slow, fp64 CPU oracle for the ring KV-cache attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
 * baseline leg may load this library.  It shares no code with the CUDA path and the
 * product never calls it.
 *
 * What it follows (page titles and sections; none of the pages prints code for this):
 *  - "Runway Characters: Serving a 57B Video Diffusion Transformer for Real-Time
 *    Conversation", abstract: a ring KV cache; RoPE and FP8 quantisation applied once
 *    per write; a delta rotation of the cache when positions reset; 240 attention calls
 *    per chunk, each reading a 5,788-slot cache of which 757 tokens are new.
 *  - "KREA Real-Time 14B / video-conductor", section "Plastic Windows": lowering the cache
 *    attention bias during transitions (read here as an additive logit on history slots).
 *  - "Why Live Video Generation Still Struggles With Timing": attention is bidirectional
 *    inside the current chunk and backward-only across chunks; a sliding window of
 *    recent history, with the first chunk kept beside it as a persistent anchor.
 *  - "Stream LTX", section "Training": block structure (1 s blocks of video + audio
 *    latents) and a causal mask on every attention path.
 *
 * Precision.  The write and the rotation are defined as a fixed sequence of IEEE binary32
 * round-to-nearest-even operations.  Each one is emulated here as the binary64 operation
 * followed by one rounding to binary32.  For +, -, *, / this equals the correctly rounded
 * binary32 result because 53 >= 2*24 + 2 (double rounding is innocuous; S. Figueroa,
 * "When is double rounding innocuous?", SIGNUM 1995).  Compile WITHOUT floating-point
 * contraction (-ffp-contract=off) and without fast-math.  Attention is evaluated in
 * binary64, directly (two passes: row maximum, then sums), not in the online form.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - FP8 is OCP e4m3fn (bias 7, max 448, subnormals down to 2^-9, no infinities,
 *    S.1111.111 is NaN), round-to-nearest-even, saturating to +-448.
 *  - One fp32 scale per (token, head) row: scale = amax/448, codes = e4m3(y * (448/amax)).
 *    All-zero rows: scale 0, codes 0.  Rows with amax < 448/FLT_MAX (448/amax overflows):
 *    scale 0, codes 0.  Rows with a non-finite element: scale NaN (0x7FC00000), every
 *    code 0x7F.
 *  - RoPE: 1-D positions, interleaved pairs (x[2i], x[2i+1]), theta_i = base^(-2i/D)
 *    evaluated as pow(base, -(2i)/D) in binary64, angle = p * theta_i in binary64,
 *    c = fl32(cos(angle)), s = fl32(sin(angle)) from the C library.
 *      y0 = fl32(fl32(x0*c) - fl32(x1*s)),  y1 = fl32(fl32(x0*s) + fl32(x1*c)).
 *  - Queries are rotated at q_pos0 + i with the same op sequence, then rounded to bf16.
 *  - Attention score: softmax_scale * (q . k) + (history ? cache_bias : 0).
 *  - Block id of current-chunk token t: t < first ? 0 : 1 + (t - first) / block_len,
 *    separately for queries and keys; a current key is visible iff its block id <= the
 *    query's.  History keys are always visible.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

/* ---------------------------------------------------------------- binary32 emulation */

static inline float fl32(double x) { return (float)x; } /* one RNE rounding to binary32 */
static inline float mul32(float a, float b) { return fl32((double)a * (double)b); }
static inline float add32(float a, float b) { return fl32((double)a + (double)b); }
static inline float sub32(float a, float b) { return fl32((double)a - (double)b); }
static inline float div32(float a, float b) { return fl32((double)a / (double)b); }

static float nan32(void) {
  uint32_t bits = 0x7FC00000u;
  float f;
  memcpy(&f, &bits, 4);
  return f;
}

/* ---------------------------------------------------------------- e4m3 (OCP FP8) */

/* Value of an e4m3fn code, from the OCP 8-bit floating point definition. */
ORC_API double orc_e4m3_decode(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 0xF, m = code & 7;
  double mag;
  if (e == 0xF && m == 7) return NAN;
  if (e == 0) mag = ldexp((double)m, -9);                  /* subnormal: m * 2^-9 */
  else mag = ldexp(1.0 + (double)m / 8.0, e - 7);          /* normal: 1.m * 2^(e-7) */
  return s ? -mag : mag;
}

/* Nearest e4m3fn code (ties to even), saturating to +-448; NaN -> 0x7F. */
ORC_API uint8_t orc_e4m3_encode(float v) {
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs((double)v);
  if (a > 448.0) return sign | 0x7E;
  double quantum;
  if (a >= 0x1p-6) {
    int e;
    frexp(a, &e);                                          /* a in [2^(e-1), 2^e) */
    quantum = ldexp(1.0, (e - 1) - 3);                     /* 3 mantissa bits */
  } else {
    quantum = 0x1p-9;                                      /* subnormal spacing */
  }
  double r = nearbyint(a / quantum) * quantum;             /* a/quantum is exact */
  if (r == 0.0) return sign;
  if (r < 0x1p-6) return sign | (uint8_t)(r / 0x1p-9);
  int e;
  double f = frexp(r, &e);                                 /* r = f * 2^e, f in [0.5,1) */
  int biased = (e - 1) + 7;
  int mant = (int)((2.0 * f - 1.0) * 8.0);
  return sign | (uint8_t)(biased << 3) | (uint8_t)mant;
}

/* Round a binary32 value to the nearest bfloat16 (ties to even); returned widened. */
ORC_API float orc_bf16_round(float v) {
  if (isnan(v) || isinf(v) || v == 0.0f) return v;
  double a = fabs((double)v);
  int e;
  frexp(a, &e);
  int ex = e - 1;                                          /* a in [2^ex, 2^(ex+1)) */
  if (ex < -126) ex = -126;                                /* bf16 subnormal spacing 2^-133 */
  double quantum = ldexp(1.0, ex - 7);                     /* 8 significant bits */
  double r = nearbyint(a / quantum) * quantum;
  if (r > 0x1.FEp127) r = INFINITY;                        /* above the largest bf16 */
  return (float)(signbit(v) ? -r : r);
}

/* ---------------------------------------------------------------- RoPE */

/* cos/sin of p*theta_i for every pair i of a D-wide row, rounded to binary32. */
ORC_API void orc_rope_cs(int64_t p, int D, double base, float* c, float* s) {
  for (int i = 0; i < D / 2; ++i) {
    double theta_i = pow(base, -(2.0 * (double)i) / (double)D);
    double angle = (double)p * theta_i;
    c[i] = (float)cos(angle);
    s[i] = (float)sin(angle);
  }
}

/* Rotate one row by the given cos/sin, as the binary32 op sequence above. */
ORC_API void orc_rope_apply(const float* x, int D, const float* c, const float* s, float* y) {
  for (int i = 0; i < D / 2; ++i) {
    float x0 = x[2 * i], x1 = x[2 * i + 1];
    y[2 * i] = sub32(mul32(x0, c[i]), mul32(x1, s[i]));
    y[2 * i + 1] = add32(mul32(x0, s[i]), mul32(x1, c[i]));
  }
}

/* The same rotation in binary64 (exact-arithmetic reference for invariants). */
ORC_API void orc_rope_apply_f64(const double* x, int D, int64_t p, double base, double* y) {
  for (int i = 0; i < D / 2; ++i) {
    double theta_i = pow(base, -(2.0 * (double)i) / (double)D);
    double angle = (double)p * theta_i, c = cos(angle), s = sin(angle);
    double x0 = x[2 * i], x1 = x[2 * i + 1];
    y[2 * i] = x0 * c - x1 * s;
    y[2 * i + 1] = x0 * s + x1 * c;
  }
}

/* ---------------------------------------------------------------- per-row FP8 quantisation */

ORC_API void orc_quant_row(const float* y, int D, uint8_t* code, float* scale) {
  double amax = 0.0;
  int nonfinite = 0;
  for (int i = 0; i < D; ++i) {
    if (!isfinite(y[i])) nonfinite = 1;
    double a = fabs((double)y[i]);
    if (a > amax) amax = a;
  }
  if (nonfinite) {
    *scale = nan32();
    memset(code, 0x7F, (size_t)D);
    return;
  }
  float inv = (amax > 0.0) ? div32(448.0f, (float)amax) : 0.0f;
  if (amax == 0.0 || !isfinite(inv)) {
    *scale = 0.0f;
    memset(code, 0x00, (size_t)D);
    return;
  }
  *scale = div32((float)amax, 448.0f);
  for (int i = 0; i < D; ++i) code[i] = orc_e4m3_encode(mul32(y[i], inv));
}

/* ---------------------------------------------------------------- ring state */

typedef struct {
  int32_t C, H, D, _pad;
  double base;
  /* 3-D RoPE (all zero: 1-D): pairs of the t, h, w runs of the head dimension and the
   * frame grid (tokens per frame = grid_h * grid_w, raster order) */
  int32_t pairs_t, pairs_h, pairs_w, grid_h, grid_w, _pad2;
  int64_t write_slot, live, pending, next_pos;
  uint8_t* kc;      /* [H][C][D] */
  uint8_t* vc;      /* [H][C][D] */
  float* ks;        /* [H][C] */
  float* vs;        /* [H][C] */
  int32_t* slot_pos; /* [C] */
} orc_ring;

/* Angles of token position p under the ring's RoPE rule, rounded to binary32.
 *  1-D (pairs all zero): pair i turns by p * base^(-2i/D) (orc_rope_cs).
 *  3-D: the video-DiT form of RoPE, read from "Why Live Video Generation Still Struggles
 *  With Timing", Transcript (positions of long streams calibrated and reset along time):
 *  the D/2 pairs form three consecutive runs for time, height and width (pairs_t,
 *  pairs_h, pairs_w of them); token position p is frame f = floor(p / (gh*gw)), row
 *  y = floor(p / gw) mod gh and column x = p mod gw of a raster-ordered frame grid
 *  gh x gw; pair k of a run of n pairs turns by (its coordinate) * base^(-2k/(2n)).
 *  With pairs (D/2, 0, 0) and a 1 x 1 grid this is the 1-D rule, bit for bit. */
ORC_API void orc_rope_cs_ring(const orc_ring* r, int64_t p, float* c, float* s) {
  if (r->pairs_t == 0 && r->pairs_h == 0 && r->pairs_w == 0) {
    orc_rope_cs(p, r->D, r->base, c, s);
    return;
  }
  const int64_t gh = r->grid_h, gw = r->grid_w, hw = gh * gw;
  int64_t f = p / hw;
  if (p % hw != 0 && p < 0) f -= 1;                        /* floor division */
  const int64_t rem = p - f * hw;                          /* 0 <= rem < hw */
  const int64_t coord[3] = {f, rem / gw, rem % gw};
  const int n[3] = {r->pairs_t, r->pairs_h, r->pairs_w};
  int at = 0;
  for (int a = 0; a < 3; ++a) {
    for (int k = 0; k < n[a]; ++k, ++at) {
      double theta = pow(r->base, -(2.0 * (double)k) / (double)(2 * n[a]));
      double angle = (double)coord[a] * theta;
      c[at] = (float)cos(angle);
      s[at] = (float)sin(angle);
    }
  }
}

static int64_t mod_c(int64_t a, int64_t C) {
  int64_t r = a % C;
  return r < 0 ? r + C : r;
}

/* Number of valid slots: committed history plus the pending chunk, capped at C. */
static int64_t valid_slots(const orc_ring* r) {
  int64_t v = r->live + r->pending;
  return v > r->C ? r->C : v;
}

/* Slot holding the age-th newest valid token (age 0 = newest). */
ORC_API int64_t orc_slot_of_age(const orc_ring* r, int64_t age) {
  return mod_c(r->write_slot + r->pending - 1 - age, r->C);
}

ORC_API void orc_ring_commit(orc_ring* r) {
  r->write_slot = mod_c(r->write_slot + r->pending, r->C);
  r->live = r->live + r->pending > r->C ? r->C : r->live + r->pending;
  r->next_pos += r->pending;
  r->pending = 0;
}

/* Write n tokens of K and V ([n][H][D] binary32 values) as the pending chunk at
 * write_slot, positions next_pos + t; commit if asked. */
ORC_API void orc_ring_write(orc_ring* r, const float* k, const float* v, int n, int commit) {
  const int C = r->C, H = r->H, D = r->D;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < n; ++t) {
    float c[256], s[256], y[512];
    int64_t slot = mod_c(r->write_slot + t, C);
    int64_t pos = r->next_pos + t;
    orc_rope_cs_ring(r, pos, c, s);
    r->slot_pos[slot] = (int32_t)pos;
    for (int h = 0; h < H; ++h) {
      const float* kr = k + ((size_t)t * H + h) * D;
      const float* vr = v + ((size_t)t * H + h) * D;
      size_t at = ((size_t)h * C + slot) * D;
      orc_rope_apply(kr, D, c, s, y);
      orc_quant_row(y, D, r->kc + at, r->ks + (size_t)h * C + slot);
      orc_quant_row(vr, D, r->vc + at, r->vs + (size_t)h * C + slot);
    }
  }
  r->pending = n;
  if (commit) orc_ring_commit(r);
}

/* Position reset: re-rotate every valid cached key by delta (dequantise, rotate,
 * requantise); V is untouched; slot positions and next_pos shift by delta.  Under 3-D
 * RoPE a reset moves time only: delta must be a whole number of frames (a multiple of
 * grid_h * grid_w), whose angles are zero on the h and w runs; otherwise nothing changes
 * and -1 is returned. */
ORC_API int orc_ring_delta_rotate(orc_ring* r, int64_t delta) {
  const int C = r->C, H = r->H, D = r->D;
  float c[256], s[256];
  if ((r->pairs_t | r->pairs_h | r->pairs_w) != 0 &&
      delta % ((int64_t)r->grid_h * r->grid_w) != 0)
    return -1;
  orc_rope_cs_ring(r, delta, c, s);
  int64_t nv = valid_slots(r);
#pragma omp parallel for schedule(static)
  for (int64_t age = 0; age < nv; ++age) {
    float x[512], y[512];
    int64_t slot = orc_slot_of_age(r, age);
    r->slot_pos[slot] = (int32_t)(r->slot_pos[slot] + delta);
    for (int h = 0; h < H; ++h) {
      size_t at = ((size_t)h * C + slot) * D;
      float sc = r->ks[(size_t)h * C + slot];
      for (int i = 0; i < D; ++i) x[i] = mul32((float)orc_e4m3_decode(r->kc[at + i]), sc);
      orc_rope_apply(x, D, c, s, y);
      orc_quant_row(y, D, r->kc + at, r->ks + (size_t)h * C + slot);
    }
  }
  r->next_pos += delta;
  return 0;
}

/* ---------------------------------------------------------------- chunk attention */

static int64_t block_id(int64_t t, int64_t first, int64_t len) {
  return t < first ? 0 : 1 + (t - first) / len;
}

/* Attention of query rows rows[0..n_rows) (all n_q rows if rows is NULL) over the valid
 * slots of rings[0..n_rings).  rings[0] is the stream's main ring: its newest n_current
 * slots are the current chunk (block mask, no bias) and the rest is history.  Every valid
 * slot of rings[1..] is history too: always visible, cache_bias added.  That is how a
 * persistent anchor ("Why Live Video Generation Still Struggles With Timing", Transcript:
 * the first chunk kept beside a sliding window of recent history) joins the attention.
 * All rings share H, D and the RoPE base.  q is [n_q][H][D] binary32 (the exact values of
 * the caller's inputs).  out: [n_rows][H][D] binary64; lse: [H][n_rows] binary64 (natural
 * log), may be NULL.  flags bit 0 (mode B): the rotated bf16 query is also quantised to
 * e4m3 per row by the write rule and dequantised before the dot products. */
ORC_API void orc_chunk_attention_multi(const orc_ring* const* rings, int n_rings,
                                       const float* q, int n_q, int64_t q_pos0, int n_current,
                                       int q_first, int q_block, int k_first, int k_block,
                                       float cache_bias, float softmax_scale, int flags,
                                       const int32_t* rows, int n_rows, double* out,
                                       double* lse) {
  const orc_ring* r0 = rings[0];
  const int H = r0->H, D = r0->D;
  int64_t nv = 0;
  for (int g = 0; g < n_rings; ++g) nv += valid_slots(rings[g]);
  if (!rows) n_rows = n_q;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int ri = 0; ri < n_rows; ++ri) {
    for (int h = 0; h < H; ++h) {
      const int i = rows ? rows[ri] : ri;
      float c[256], s[256], y[512];
      double qt[512];
      orc_rope_cs_ring(r0, q_pos0 + i, c, s);
      orc_rope_apply(q + ((size_t)i * H + h) * D, D, c, s, y);
      for (int d = 0; d < D; ++d) y[d] = orc_bf16_round(y[d]);
      if (flags & 1) {
        uint8_t qc[512];
        float qs;
        orc_quant_row(y, D, qc, &qs);
        for (int d = 0; d < D; ++d) qt[d] = orc_e4m3_decode(qc[d]) * (double)qs;
      } else {
        for (int d = 0; d < D; ++d) qt[d] = (double)y[d];
      }
      const int64_t qb = block_id(i, q_first, q_block);
      double* sc = (double*)malloc(sizeof(double) * (size_t)(nv > 0 ? nv : 1));
      int64_t* sl = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nv > 0 ? nv : 1));
      int* sg = (int*)malloc(sizeof(int) * (size_t)(nv > 0 ? nv : 1));
      int64_t nvis = 0;
      double m = -INFINITY;
      for (int g = 0; g < n_rings; ++g) {
        const orc_ring* r = rings[g];
        const int C = r->C;
        const int64_t nv_g = valid_slots(r);
        for (int64_t age = 0; age < nv_g; ++age) {
          int history = g > 0 || age >= n_current;
          if (!history) {
            int64_t t = n_current - 1 - age;          /* token index inside the chunk */
            if (block_id(t, k_first, k_block) > qb) continue;
          }
          int64_t slot = orc_slot_of_age(r, age);
          const uint8_t* kr = r->kc + ((size_t)h * C + slot) * D;
          double ksc = (double)r->ks[(size_t)h * C + slot], dot = 0.0;
          for (int d = 0; d < D; ++d) dot += qt[d] * (orc_e4m3_decode(kr[d]) * ksc);
          double sv = (double)softmax_scale * dot + (history ? (double)cache_bias : 0.0);
          sc[nvis] = sv;
          sl[nvis] = slot;
          sg[nvis] = g;
          ++nvis;
          if (sv > m) m = sv;
        }
      }
      if (m == -INFINITY) nvis = 0;  /* every visible score is -inf: nothing attended */
      double* o = out + ((size_t)ri * H + h) * D;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      double l = 0.0;
      for (int64_t j = 0; j < nvis; ++j) {
        const orc_ring* r = rings[sg[j]];
        double p = exp(sc[j] - m);
        l += p;
        const uint8_t* vr = r->vc + ((size_t)h * r->C + sl[j]) * D;
        double vsc = (double)r->vs[(size_t)h * r->C + sl[j]];
        for (int d = 0; d < D; ++d) o[d] += p * (orc_e4m3_decode(vr[d]) * vsc);
      }
      if (nvis > 0) {
        for (int d = 0; d < D; ++d) o[d] /= l;
      }
      if (lse) lse[(size_t)h * n_rows + ri] = nvis > 0 ? m + log(l) : -INFINITY;
      free(sc);
      free(sl);
      free(sg);
    }
  }
}

/* The one-ring case: the stream's ring alone. */
ORC_API void orc_chunk_attention(const orc_ring* r, const float* q, int n_q, int64_t q_pos0,
                                 int n_current, int q_first, int q_block, int k_first,
                                 int k_block, float cache_bias, float softmax_scale, int flags,
                                 const int32_t* rows, int n_rows, double* out, double* lse) {
  const orc_ring* rings[1] = {r};
  orc_chunk_attention_multi(rings, 1, q, n_q, q_pos0, n_current, q_first, q_block, k_first,
                            k_block, cache_bias, softmax_scale, flags, rows, n_rows, out, lse);
}

/* ---------------------------------------------------------------- content memory */

/* Attention mass that history slots of rings[ri] receive in one attention call over
 * rings[0..n_rings) (same arguments as orc_chunk_attention_multi): for candidate c (the
 * slot of age ages[c] in rings[ri], a history slot), mass[c] = sum over heads h and query
 * rows i of exp(s_ihc - lse_ih), the softmax probability row i of head h gives the slot,
 * with lse the call's own log-sum-exp over every visible key of every ring.  This is the
 * "attention quality" of "Stream LTX", Inference (each layer scores its own keys), read
 * as the probability mass the keys received from the newest chunk's queries. */
ORC_API void orc_key_mass(const orc_ring* const* rings, int n_rings, const float* q, int n_q,
                          int64_t q_pos0, int n_current, int q_first, int q_block,
                          int k_first, int k_block, float cache_bias, float softmax_scale,
                          int ri, const int64_t* ages, int n_cand, double* mass) {
  const orc_ring* r0 = rings[0];
  const orc_ring* rk = rings[ri];
  const int H = r0->H, D = r0->D;
  double* out = (double*)malloc(sizeof(double) * (size_t)n_q * H * D);
  double* lse = (double*)malloc(sizeof(double) * (size_t)H * n_q);
  orc_chunk_attention_multi(rings, n_rings, q, n_q, q_pos0, n_current, q_first, q_block,
                            k_first, k_block, cache_bias, softmax_scale, 0, NULL, n_q, out, lse);
  for (int c = 0; c < n_cand; ++c) mass[c] = 0.0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int c = 0; c < n_cand; ++c) {
    const int64_t slot = orc_slot_of_age(rk, ages[c]);
    double acc = 0.0;
    for (int h = 0; h < H; ++h) {
      const uint8_t* kr = rk->kc + ((size_t)h * rk->C + slot) * D;
      const double ksc = (double)rk->ks[(size_t)h * rk->C + slot];
      for (int i = 0; i < n_q; ++i) {
        if (!isfinite(lse[(size_t)h * n_q + i])) continue;
        float cc[256], ss[256], y[512];
        orc_rope_cs_ring(r0, q_pos0 + i, cc, ss);
        orc_rope_apply(q + ((size_t)i * H + h) * D, D, cc, ss, y);
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
          dot += (double)orc_bf16_round(y[d]) * (orc_e4m3_decode(kr[d]) * ksc);
        const double sv = (double)softmax_scale * dot + (double)cache_bias;
        acc += exp(sv - lse[(size_t)h * n_q + i]);
      }
    }
    mass[c] = acc;
  }
  free(out);
  free(lse);
}

/* Top-M selection with temporal diversity ("Stream LTX", Inference: keys scored on
 * attention quality and temporal diversity, evicted down to a top-M budget).  Read as a
 * greedy choice in which every key already kept from a frame multiplies the remaining
 * keys of that frame by gamma: equivalently, the k-th best key of its frame (by quality,
 * k = 0, 1, ...) scores quality * gamma^k, and the M best scores are kept.  Ties break
 * toward the lower position, then the lower candidate index, so the choice is unique.
 * Writes the kept candidate indices in ascending order and returns how many (min(n, M)). */
typedef struct { double key; int64_t pos; int idx; int64_t frame; } orc_cand;

static int cmp_frame_then_quality(const void* a, const void* b) {
  const orc_cand *x = (const orc_cand*)a, *y = (const orc_cand*)b;
  if (x->frame != y->frame) return x->frame < y->frame ? -1 : 1;
  if (x->key != y->key) return x->key > y->key ? -1 : 1;
  if (x->pos != y->pos) return x->pos < y->pos ? -1 : 1;
  return x->idx < y->idx ? -1 : (x->idx > y->idx);
}

static int cmp_score(const void* a, const void* b) {
  const orc_cand *x = (const orc_cand*)a, *y = (const orc_cand*)b;
  if (x->key != y->key) return x->key > y->key ? -1 : 1;
  if (x->pos != y->pos) return x->pos < y->pos ? -1 : 1;
  return x->idx < y->idx ? -1 : (x->idx > y->idx);
}

static int cmp_int(const void* a, const void* b) {
  const int x = *(const int*)a, y = *(const int*)b;
  return x < y ? -1 : (x > y);
}

ORC_API int orc_memory_select(const double* quality, const int64_t* frame, const int64_t* pos,
                              int n, int M, double gamma, int32_t* kept) {
  orc_cand* c = (orc_cand*)malloc(sizeof(orc_cand) * (size_t)(n > 0 ? n : 1));
  for (int i = 0; i < n; ++i) {
    c[i].key = quality[i];
    c[i].pos = pos[i];
    c[i].idx = i;
    c[i].frame = frame[i];
  }
  qsort(c, (size_t)n, sizeof(orc_cand), cmp_frame_then_quality);
  double scale = 1.0;
  for (int i = 0; i < n; ++i) {
    scale = (i > 0 && c[i].frame == c[i - 1].frame) ? scale * gamma : 1.0;
    c[i].key = c[i].key * scale;                     /* quality * gamma^(rank in frame) */
  }
  qsort(c, (size_t)n, sizeof(orc_cand), cmp_score);
  const int m = n < M ? n : M;
  int* ids = (int*)malloc(sizeof(int) * (size_t)(m > 0 ? m : 1));
  for (int i = 0; i < m; ++i) ids[i] = c[i].idx;
  qsort(ids, (size_t)m, sizeof(int), cmp_int);
  for (int i = 0; i < m; ++i) kept[i] = ids[i];
  free(ids);
  free(c);
  return m;
}

/* ---------------------------------------------------------------- array helpers for tests */

ORC_API void orc_e4m3_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}
ORC_API void orc_e4m3_decode_n(const uint8_t* c, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(c[i]);
}
ORC_API void orc_bf16_round_n(const float* v, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_round(v[i]);
}
ORC_API void orc_quant_rows(const float* y, int64_t rows, int D, uint8_t* code, float* scale) {
  for (int64_t r = 0; r < rows; ++r) orc_quant_row(y + r * D, D, code + r * D, scale + r);
}
ORC_API int orc_struct_size(void) { return (int)sizeof(orc_ring); }
