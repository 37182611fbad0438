/*
 * sq_oracle.c -- plain, slow CPU oracle of the quantized-state decode step.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load this library. The product path (the
 * CUDA library under quantized_linear_attention_sq_b200/csrc) never calls
 * it, and the two share no code, headers, tables or helpers.
 *
 * What it computes (one decode step of a gated delta-rule state, kept in a
 * low-bit, two-axis-scaled format):
 *
 *   - gated delta rule, per (request, value head) state S (d x d):
 *       S <- diag(g) S ;  u = beta (v - S^T k) ;  S <- S + k u^T ;  o = S^T q
 *     GDN has one gate per head, KDA one gate per key channel
 *     ["STEPQuant review (e-cogni)", section "Contexto"; "STEPQuant talk
 *     announcement (qingkeai)", opening section].
 *   - the state is stored as S_ij ~= r_i * c_j * q_ij: a row scale per key
 *     row, a column scale per value column, and low-bit integer codes
 *     ["STEPQuant review (e-cogni)", "O que os autores propõem",
 *     Key-Row-Aware Dual-Axis Fitting; talk announcement, section
 *     "STEPQuant 核心设计"].
 *   - bit widths are set per unit (a head for GDN, a key row for KDA) and a
 *     few units stay in FP16 as pivots ["STEPQuant: estados recurrentes a
 *     6 bit" (gpt-diffusion), "Las dos ideas: cuándo y dónde importa el
 *     error"].
 *   - after every update the state is requantized; the row scale comes from
 *     the row's current magnitude times its calibrated row-impact factor
 *     (same sections), so errors feed back step after step
 *     ["STEPQuant review (e-cogni)", "Contexto"].
 *
 * The pages fix the method but not its arithmetic; the canonical
 * elementwise arithmetic below is this project's reading, chosen so that
 * two implementations agree bit for bit on the integer codes. The only sums
 * are the column dot products (S^T k and S^T q); each is the exact value of
 * the sum of exact products, rounded once to fp32 (round to nearest, ties to
 * even; an exact zero gives +0). Here that is computed literally: every
 * product is an integer times a power of two, and the products are added
 * without rounding in a wide fixed-point accumulator (xacc below) that is
 * rounded once at the end. S^T k is the one sum that feeds back into the
 * state, so it is the one whose rounding decides reproducibility over a
 * long rollout; because it is exact, the result does not depend on any
 * summation order.
 *
 * Column-normalised form. With S = T diag(c), the whole step is carried out
 * on T (the row-scale x code part), and c enters only where S^T k and S^T q
 * are formed and where u is mapped back to T units. A row is stored as
 * values V_ij with a per-row multiplier M_i, the gated T being V_ij M_i:
 *   1. quantized rows: V = integer code q_ij, M_i = a_i = fp32(r_i * g_i)
 *      pivot rows:     V = stored fp16 value h_ij of T, M_i = g_i
 *   2. P_j   = sum_i V_ij M_i k_i  (the exact value, rounded once to fp32)
 *   3. p_j = fp32(c_j P_j); u_j = fp32(beta fp32(v_j - p_j));
 *      w_j = fp32(u_j * ic_j) with ic_j = fp32(1 / c_j)
 *   4. T'_ij = fmaf(V_ij, M_i, fp32(k_i * w_j))   (gate, decay and update,
 *      one rounding of the exact gated value plus the rounded update)
 *   5. O_j   = sum_i T'_ij q_i (exact, rounded once); o_j = fp32(c_j O_j)
 *   6. m_i   = max_j |T'_ij| (a NaN makes m_i NaN)
 *   7. s_i   = fp32(fp32(min(phi_i, 1) m_i) / qmax_i); r'_i = fp16 of s_i rounded
 *      toward +inf (saturating at 65504); ir_i = 0 if r'_i == 0 else
 *      fp32(1 / r'_i)
 *   8. q'_ij = min(max(RNE(T'_ij * ir_i), -qmax), qmax), the product taken
 *      exactly (no fp32 rounding before the rounding to an integer)
 *   9. pivot rows: h'_ij = fp16 round-to-nearest-even of T'_ij, saturating
 *      at +-65504; a NaN stores 0.
 *  A row whose m_i is NaN stores r' = 0 and all codes 0 (status bit 0).
 *
 * Storage format (this project's reading; the pages give only the bit
 * accounting): a request's state is one contiguous slot; inside it the
 * value heads follow each other; a head's record is
 *   [d row scales, fp16 little-endian][row 0][row 1]...[row d-1][zero pad to 16 B]
 * A pivot row holds d fp16 values (its scale slot holds fp16 1.0). A
 * quantized row of width b holds d codes in a little-endian bit stream:
 * code j occupies stream bits [b*j, b*j + b), stream bit n is bit n%8 of
 * byte n/8, and the stored field is the code plus 2^(b-1) (offset binary),
 * so a code q in [-qmax, qmax] is stored as q + 2^(b-1) in [1, 2^b - 1].
 * A row takes ceil(d*b/8) bytes (exactly d*b/8 for the d = 32, 64, 128 the
 * CUDA path supports; tiny tiles used by the brute-force pins round up).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math (oracle/build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ST_NAN 1u       /* a NaN reached the state or the output */
#define ST_SATURATED 2u /* an fp16 value or row scale saturated at 65504 */
#define ST_BAD_SLOT 4u  /* a slot id outside [0, n_slots) was skipped */

typedef struct {
  int32_t n_slots;
  int32_t h_v;
  int32_t h_k;
  int32_t d;
  int32_t gate_kind;         /* 0: one gate per head (GDN); 1: per key channel (KDA) */
  const int8_t *unit_bits;   /* GDN [h_v], KDA [h_v*d]; 2, 4, 6 or 8 */
  const uint8_t *pivot;      /* same shape; nonzero = FP16 pivot unit */
  const float *col_scale;    /* [h_v*d] c_j */
  const float *row_impact;   /* [h_v*d] phi_i */
} sqo_desc;

/* ------------------------------------------------------------------ fp16 */
/* Written from the IEEE-754 binary16 definition: 1 sign bit, 5 exponent bits
 * (bias 15), 10 fraction bits; subnormals have quantum 2^-24. */

float sqo_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(m | 0x400), e - 25);
  return (float)(sign ? -v : v);
}

/* Encode |value| = n * 2^qexp (n integer, 0 <= n <= 2048) as fp16 bits. */
static uint16_t f16_encode(int sign, double n, int qexp) {
  uint16_t s = sign ? 0x8000 : 0;
  if (n == 0.0) return s;
  if (n >= 2048.0) { n = 1024.0; qexp += 1; }
  if (n < 1024.0) return (uint16_t)(s | (uint16_t)n); /* subnormal, qexp == -24 */
  int ef = qexp + 25;
  if (ef >= 31) return (uint16_t)(s | 0x7c00);
  return (uint16_t)(s | (ef << 10) | ((int)n - 1024));
}

/* The quantum (spacing) of fp16 numbers around a finite a >= 0, as 2^qexp. */
static int f16_quantum_exp(double a) {
  if (a < ldexp(1.0, -14)) return -24;
  int e;
  frexp(a, &e); /* a = f 2^e, f in [0.5, 1) */
  return e - 11;
}

/* round to nearest, ties to even */
uint16_t sqo_f16_rne(float x) {
  if (isnan(x)) return 0x7e00;
  int sign = signbit(x) ? 1 : 0;
  double a = fabs((double)x);
  if (isinf(x) || a >= 65520.0) return (uint16_t)(sign ? 0xfc00 : 0x7c00);
  int qe = f16_quantum_exp(a);
  double n = nearbyint(ldexp(a, -qe)); /* default rounding mode: nearest-even */
  return f16_encode(sign, n, qe);
}

/* round toward +infinity */
uint16_t sqo_f16_ru(float x) {
  if (isnan(x)) return 0x7e00;
  int sign = signbit(x) ? 1 : 0;
  double a = fabs((double)x);
  if (isinf(x)) return (uint16_t)(sign ? 0xfbff : 0x7c00);
  if (!sign && a > 65504.0) return 0x7c00;
  if (sign && a > 65504.0) return 0xfbff;
  int qe = f16_quantum_exp(a);
  double t = ldexp(a, -qe);
  double n = sign ? floor(t) : ceil(t); /* toward +inf: down in magnitude for negatives */
  return f16_encode(sign, n, qe);
}

/* --------------------------------------------------------- exact sums */
/* A sum of products of floats, held exactly. Every finite float is an
 * integer significand (below 2^24) times a power of two (2^-149 at the
 * least), so a product of up to three floats is an integer below 2^72 times
 * 2^e with e >= -447. The accumulator is a two's complement fixed-point
 * number of XA_LIMBS 32-bit limbs whose bit 0 has weight 2^XA_LSB; that
 * covers every product of three finite floats (weights from 2^-447 to below
 * 2^(3 128)) with room for the carries of any number of terms this file
 * adds. Each limb is kept in an int64 and
 * normalised only at the end, so adding a term never loses a bit. */
#define XA_LIMBS 32
#define XA_LSB (-544)

typedef struct {
  int64_t limb[XA_LIMBS];
} xacc;

static void xacc_init(xacc *a) { memset(a, 0, sizeof *a); }

/* significand and exponent of a finite float: |x| = m 2^e exactly, read
 * from its IEEE-754 binary32 fields (subnormals: exponent field 0, no
 * implicit bit) */
static void split_f32(float x, uint64_t *m, int *e) {
  uint32_t b;
  memcpy(&b, &x, 4);
  uint32_t ef = (b >> 23) & 0xffu, fr = b & 0x7fffffu;
  if (ef) { *m = fr | 0x800000u; *e = (int)ef - 150; }
  else { *m = fr; *e = -149; }
}

/* a += x * y * z for finite x, y, z */
static void xacc_add3(xacc *a, float x, float y, float z) {
  if (x == 0.0f || y == 0.0f || z == 0.0f) return;
  uint64_t mx, my, mz;
  int ex, ey, ez;
  split_f32(x, &mx, &ex);
  split_f32(y, &my, &ey);
  split_f32(z, &mz, &ez);
  unsigned __int128 v = (unsigned __int128)(mx * my) * mz; /* < 2^72 */
  int pos = ex + ey + ez - XA_LSB;                           /* bit index of v's bit 0, >= 544 - 447 */
  int neg = signbit(x) ^ signbit(y) ^ signbit(z);
  int li = pos / 32, sh = pos % 32;
  v <<= sh; /* < 2^103 */
  for (int t = 0; t < 4 && li + t < XA_LIMBS; t++) {
    int64_t piece = (int64_t)(uint32_t)(v >> (32 * t));
    a->limb[li + t] += neg ? -piece : piece;
  }
}

/* carries into limbs 0 .. XA_LIMBS-2 in [0, 2^32); the top limb keeps the sign */
static void xacc_normalise(int64_t *l) {
  for (int i = 0; i + 1 < XA_LIMBS; i++) {
    int64_t c = l[i] >> 32; /* floor division by 2^32 (arithmetic shift) */
    l[i] -= c * ((int64_t)1 << 32);
    l[i + 1] += c;
  }
}

static int limb_bit(const int64_t *l, int n) { return (int)((l[n / 32] >> (n % 32)) & 1); }

/* The exact sum rounded once to fp32: to nearest, ties to even, with the
 * subnormal quantum 2^-149 at the bottom and inf above the largest float;
 * an exact zero gives +0. */
static float xacc_round_f32(const xacc *a) {
  int64_t l[XA_LIMBS];
  memcpy(l, a->limb, sizeof l);
  xacc_normalise(l);
  int neg = l[XA_LIMBS - 1] < 0;
  if (neg) {
    for (int i = 0; i < XA_LIMBS; i++) l[i] = -l[i];
    xacc_normalise(l);
  }
  int top = -1; /* index of the most significant set bit */
  for (int i = XA_LIMBS - 1; i >= 0 && top < 0; i--)
    if (l[i]) {
      int b = 31;
      while (!((l[i] >> b) & 1)) b--;
      top = 32 * i + b;
    }
  if (top < 0) return 0.0f;
  int qexp = top + XA_LSB - 23; /* exponent of the unit in the last place */
  if (qexp < -149) qexp = -149;
  int q0 = qexp - XA_LSB; /* bit index of that unit */
  uint64_t n = 0;
  for (int b = top; b >= q0 && b >= 0; b--) n = (n << 1) | (uint64_t)limb_bit(l, b);
  int half = q0 - 1 >= 0 ? limb_bit(l, q0 - 1) : 0;
  int sticky = 0; /* any set bit below the half bit */
  int below = q0 - 1; /* bits 0 .. below-1 */
  if (below > 0) {
    int full = below / 32; /* limbs wholly below */
    for (int i = 0; i < full && !sticky; i++) sticky = l[i] != 0;
    int rem = below % 32;
    if (!sticky && rem) sticky = (l[full] & (((int64_t)1 << rem) - 1)) != 0;
  }
  if (half && (sticky || (n & 1))) n++;
  float r = (float)ldexp((double)n, qexp); /* exact, or inf beyond the largest float */
  return neg ? -r : r;
}

/* sum_i x[i*xs] y[i] z[i] of n terms (z NULL: all ones), exact and rounded
 * once to fp32. A term with an inf or NaN factor makes the result the IEEE
 * sum of the terms instead (inf, -inf or NaN, whatever the order). */
static float exact_dot(const float *x, size_t xs, const float *y, const float *z, int n) {
  for (int i = 0; i < n; i++)
    if (!isfinite(x[i * xs]) || !isfinite(y[i]) || (z && !isfinite(z[i]))) {
      long double s = 0.0L;
      for (int t = 0; t < n; t++)
        s += (long double)x[t * xs] * (long double)y[t] * (long double)(z ? z[t] : 1.0f);
      return (float)s;
    }
  xacc a;
  xacc_init(&a);
  for (int i = 0; i < n; i++) xacc_add3(&a, x[i * xs], y[i], z ? z[i] : 1.0f);
  return xacc_round_f32(&a);
}

/* sum_i x[i] y[i] z[i] exactly (z may be NULL: all ones), rounded once; an
 * entry point of its own so that the pins can check the exact sum directly */
float sqo_exact_dot3(const float *x, const float *y, const float *z, int n) {
  return exact_dot(x, 1, y, z, n);
}

/* -------------------------------------------------------------- layout */

static int unit_index(const sqo_desc *D, int h, int i) {
  return D->gate_kind == 0 ? h : h * D->d + i;
}
static int row_is_pivot(const sqo_desc *D, int h, int i) {
  return D->pivot[unit_index(D, h, i)] != 0;
}
static int row_width(const sqo_desc *D, int h, int i) {
  return D->unit_bits[unit_index(D, h, i)];
}
static size_t row_bytes(const sqo_desc *D, int h, int i) {
  if (row_is_pivot(D, h, i)) return (size_t)2 * D->d;
  return ((size_t)D->d * (size_t)row_width(D, h, i) + 7) / 8;
}
size_t sqo_record_bytes(const sqo_desc *D, int h) {
  size_t n = (size_t)2 * D->d;
  for (int i = 0; i < D->d; i++) n += row_bytes(D, h, i);
  return (n + 15) / 16 * 16;
}
size_t sqo_slot_bytes(const sqo_desc *D) {
  size_t n = 0;
  for (int h = 0; h < D->h_v; h++) n += sqo_record_bytes(D, h);
  return n;
}
size_t sqo_head_offset(const sqo_desc *D, int h) {
  size_t n = 0;
  for (int hh = 0; hh < h; hh++) n += sqo_record_bytes(D, hh);
  return n;
}
size_t sqo_pool_bytes(const sqo_desc *D) { return sqo_slot_bytes(D) * (size_t)D->n_slots; }

static size_t row_offset(const sqo_desc *D, int h, int i) {
  size_t n = (size_t)2 * D->d;
  for (int ii = 0; ii < i; ii++) n += row_bytes(D, h, ii);
  return n;
}

/* ------------------------------------------------------- bit streams */

static void put_bit(uint8_t *p, long n, unsigned bit) {
  uint8_t mask = (uint8_t)(1u << (n % 8));
  if (bit) p[n / 8] |= mask; else p[n / 8] &= (uint8_t)~mask;
}
static unsigned get_bit(const uint8_t *p, long n) { return (p[n / 8] >> (n % 8)) & 1u; }

/* store code q (in [-qmax, qmax]) as field q + 2^(b-1) at position j */
void sqo_put_code(uint8_t *row, int b, int j, int q) {
  unsigned field = (unsigned)(q + (1 << (b - 1)));
  for (int t = 0; t < b; t++) put_bit(row, (long)b * j + t, (field >> t) & 1u);
}
int sqo_get_code(const uint8_t *row, int b, int j) {
  unsigned field = 0;
  for (int t = 0; t < b; t++) field |= get_bit(row, (long)b * j + t) << t;
  return (int)field - (1 << (b - 1));
}

static uint16_t rd16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static void wr16(uint8_t *p, uint16_t v) { p[0] = (uint8_t)(v & 0xff); p[1] = (uint8_t)(v >> 8); }

static int qmax_of(int b) { return (1 << (b - 1)) - 1; }

/* ------------------------------------------------ per-tile primitives */

/* Read a head record as stored values V (d x d) and a per-row multiplier M,
 * so that the gated, column-normalised state is exactly V_ij * M_i:
 * quantized rows V = integer code, M = a_i = fp32(r_i * g_i); pivot rows
 * V = the fp16 value, M = g_i. With gate == NULL the multiplier is r_i
 * (quantized) and 1 (pivots). Nothing is rounded here. */
static void load_VM(const sqo_desc *D, int h, const uint8_t *rec, const float *gate, float *V, float *M) {
  int d = D->d;
  for (int i = 0; i < d; i++) {
    const uint8_t *row = rec + row_offset(D, h, i);
    if (row_is_pivot(D, h, i)) {
      M[i] = gate ? gate[i] : 1.0f;
      for (int j = 0; j < d; j++) V[i * d + j] = sqo_f16_to_f32(rd16(row + 2 * j));
    } else {
      int b = row_width(D, h, i);
      float r = sqo_f16_to_f32(rd16(rec + 2 * i));
      M[i] = gate ? r * gate[i] : r;
      for (int j = 0; j < d; j++) V[i * d + j] = (float)sqo_get_code(row, b, j);
    }
  }
}

/* Steps 6-9: requantize column-normalised T' into the record. */
static uint32_t store_T(const sqo_desc *D, int h, uint8_t *rec, const float *T) {
  int d = D->d;
  uint32_t st = 0;
  const float *phi = D->row_impact + (size_t)h * d;
  memset(rec, 0, sqo_record_bytes(D, h));
  for (int i = 0; i < d; i++) {
    uint8_t *row = rec + row_offset(D, h, i);
    const float *t = T + (size_t)i * d;
    if (row_is_pivot(D, h, i)) {
      wr16(rec + 2 * i, 0x3c00);
      for (int j = 0; j < d; j++) {
        float x = t[j];
        uint16_t hv;
        if (isnan(x)) { hv = 0; st |= ST_NAN; }
        else if (fabsf(x) > 65504.0f) { hv = signbit(x) ? 0xfbff : 0x7bff; st |= ST_SATURATED; }
        else hv = sqo_f16_rne(x);
        wr16(row + 2 * j, hv);
      }
      continue;
    }
    int b = row_width(D, h, i);
    int qm = qmax_of(b);
    /* 7. row magnitude */
    float m = 0.0f;
    int has_nan = 0;
    for (int j = 0; j < d; j++) {
      if (isnan(t[j])) has_nan = 1;
      else if (fabsf(t[j]) > m) m = fabsf(t[j]);
    }
    if (has_nan) {
      st |= ST_NAN;
      wr16(rec + 2 * i, 0);
      for (int j = 0; j < d; j++) sqo_put_code(row, b, j, 0);
      continue;
    }
    /* 8. row scale from magnitude x row impact, rounded up to fp16; the
     * impact factor only ever shrinks the scale (a clip ratio, min(phi, 1)) */
    float clip = phi[i] < 1.0f ? phi[i] : 1.0f;
    float s = (clip * m) / (float)qm;
    uint16_t rb;
    if (s > 65504.0f) { rb = 0x7bff; st |= ST_SATURATED; }
    else rb = sqo_f16_ru(s);
    wr16(rec + 2 * i, rb);
    float r = sqo_f16_to_f32(rb);
    float ir = (r == 0.0f) ? 0.0f : 1.0f / r;
    /* 8. codes: the integer nearest to the exact product T' * ir (ties to
     * even; the product of two floats is exact in double), clamped to the
     * symmetric range */
    for (int j = 0; j < d; j++) {
      double y = nearbyint((double)t[j] * (double)ir);
      if (y > (double)qm) y = (double)qm;
      if (y < -(double)qm) y = -(double)qm;
      sqo_put_code(row, b, j, (int)y);
    }
  }
  return st;
}

static const float *gate_vector(const sqo_desc *D, const float *g, int b, int h, float *buf) {
  int d = D->d;
  if (D->gate_kind == 0) {
    for (int i = 0; i < d; i++) buf[i] = g[(size_t)b * D->h_v + h];
    return buf;
  }
  return g + ((size_t)b * D->h_v + h) * d;
}

static int slot_of(const sqo_desc *D, const int32_t *slots, int b, uint32_t *st) {
  int s = slots ? slots[b] : b;
  if (s < 0 || s >= D->n_slots) { *st |= ST_BAD_SLOT; return -1; }
  return s;
}

/* One quantized-format decode step for one (request b, value head h) tile. */
static uint32_t step_tile(const sqo_desc *D, uint8_t *rec, int b, int h,
                          const float *q_all, const float *k_all, const float *v_all,
                          const float *beta_all, const float *g_all, float *o_all,
                          float *T, float *M, float *gbuf, float *w) {
  int d = D->d;
  int hk = h / (D->h_v / D->h_k);
  const float *q = q_all + ((size_t)b * D->h_k + hk) * d;
  const float *k = k_all + ((size_t)b * D->h_k + hk) * d;
  const float *v = v_all + ((size_t)b * D->h_v + h) * d;
  float beta = beta_all[(size_t)b * D->h_v + h];
  float *o = o_all + ((size_t)b * D->h_v + h) * d;
  const float *c = D->col_scale + (size_t)h * d;
  const float *gate = gate_vector(D, g_all, b, h, gbuf);
  uint32_t st = 0;

  load_VM(D, h, rec, gate, T, M);                      /* step 1 */
  for (int j = 0; j < d; j++) {                        /* steps 2-3 */
    float P = exact_dot(T + j, (size_t)d, M, k, d);
    float p = c[j] * P;
    float u = beta * (v[j] - p);
    float ic = 1.0f / c[j];
    w[j] = u * ic;
  }
  for (int i = 0; i < d; i++)                          /* step 4 */
    for (int j = 0; j < d; j++) {
      float kw = k[i] * w[j];
      T[i * d + j] = fmaf(T[i * d + j], M[i], kw);
    }
  for (int j = 0; j < d; j++) {                        /* step 5 */
    float O = exact_dot(T + j, (size_t)d, q, NULL, d);
    o[j] = c[j] * O;
    if (isnan(o[j])) st |= ST_NAN;
  }
  st |= store_T(D, h, rec, T);                         /* steps 6-9 */
  return st;
}

/* ------------------------------------------------------ public entry */

/* One decode step for the tiles t in [t0, t1) (tile t = request t / h_v,
 * value head t % h_v) of a batch of B requests in a quantized pool. Inputs:
 * q, k [B, h_k, d]; v [B, h_v, d]; beta [B, h_v]; g [B, h_v] (GDN) or
 * [B, h_v, d] (KDA); o [B, h_v, d]; slots [B] or NULL (identity). Returns
 * the status bits. Tiles of a skipped slot write o = 0. */
uint32_t sqo_step_tiles(const sqo_desc *D, uint8_t *pool, const float *q, const float *k,
                        const float *v, const float *beta, const float *g, float *o,
                        const int32_t *slots, int t0, int t1) {
  int d = D->d;
  float *T = malloc(sizeof(float) * d * d);
  float *M = malloc(sizeof(float) * d);
  float *gbuf = malloc(sizeof(float) * d);
  float *w = malloc(sizeof(float) * d);
  uint32_t st = 0;
  size_t slot_bytes = sqo_slot_bytes(D);
  for (int t = t0; t < t1; t++) {
    int b = t / D->h_v, h = t % D->h_v;
    int s = slot_of(D, slots, b, &st);
    if (s < 0) {
      memset(o + ((size_t)b * D->h_v + h) * d, 0, sizeof(float) * d);
      continue;
    }
    uint8_t *rec = pool + (size_t)s * slot_bytes + sqo_head_offset(D, h);
    st |= step_tile(D, rec, b, h, q, k, v, beta, g, o, T, M, gbuf, w);
  }
  free(T); free(M); free(gbuf); free(w);
  return st;
}

uint32_t sqo_step(const sqo_desc *D, uint8_t *pool, const float *q, const float *k,
                  const float *v, const float *beta, const float *g, float *o,
                  const int32_t *slots, int B) {
  return sqo_step_tiles(D, pool, q, k, v, beta, g, o, slots, 0, B * D->h_v);
}

/* Quantize fp32 states S [B, h_v, d, d] (S-space) into the pool slots:
 * T_ij = fp32(S_ij * ic_j), then steps 6-9. */
uint32_t sqo_quantize(const sqo_desc *D, uint8_t *pool, const float *S, const int32_t *slots, int B) {
  int d = D->d;
  float *T = malloc(sizeof(float) * d * d);
  uint32_t st = 0;
  size_t slot_bytes = sqo_slot_bytes(D);
  for (int b = 0; b < B; b++) {
    int s = slot_of(D, slots, b, &st);
    if (s < 0) continue;
    for (int h = 0; h < D->h_v; h++) {
      const float *Sh = S + ((size_t)b * D->h_v + h) * d * d;
      const float *c = D->col_scale + (size_t)h * d;
      for (int i = 0; i < d; i++)
        for (int j = 0; j < d; j++) {
          float ic = 1.0f / c[j];
          T[i * d + j] = Sh[i * d + j] * ic;
        }
      st |= store_T(D, h, pool + (size_t)s * slot_bytes + sqo_head_offset(D, h), T);
    }
  }
  free(T);
  return st;
}

/* Dequantize pool slots into S [B, h_v, d, d]: S_ij = fp32(fp32(q r) c_j)
 * for quantized rows and fp32(h c_j) for pivot rows. Skipped slots give 0. */
uint32_t sqo_dequantize(const sqo_desc *D, const uint8_t *pool, float *S, const int32_t *slots, int B) {
  int d = D->d;
  float *V = malloc(sizeof(float) * d * d);
  float *M = malloc(sizeof(float) * d);
  uint32_t st = 0;
  size_t slot_bytes = sqo_slot_bytes(D);
  for (int b = 0; b < B; b++) {
    int s = slot_of(D, slots, b, &st);
    for (int h = 0; h < D->h_v; h++) {
      float *Sh = S + ((size_t)b * D->h_v + h) * d * d;
      if (s < 0) { memset(Sh, 0, sizeof(float) * d * d); continue; }
      const float *c = D->col_scale + (size_t)h * d;
      load_VM(D, h, pool + (size_t)s * slot_bytes + sqo_head_offset(D, h), NULL, V, M);
      for (int i = 0; i < d; i++)
        for (int j = 0; j < d; j++) {
          float t = V[i * d + j] * M[i]; /* exact: at most 19 significant bits */
          Sh[i * d + j] = t * c[j];
        }
    }
  }
  free(V); free(M);
  return st;
}

/* Unquantized FP32 state step (S-space) for tiles [t0, t1), S pool
 * [n_slots, h_v, d, d]:
 *   G = g_i S_ij ; P_j = sum_i G_ij k_i ; u_j = beta (v_j - P_j) ;
 *   S'_ij = fmaf(k_i, u_j, G_ij) ; o_j = sum_i S'_ij q_i,
 * both sums exact and rounded once, as in the quantized step. */
uint32_t sqo_step_fp32_tiles(const sqo_desc *D, float *Spool, const float *q_all, const float *k_all,
                             const float *v_all, const float *beta_all, const float *g_all, float *o_all,
                             const int32_t *slots, int t0, int t1) {
  int d = D->d;
  float *gbuf = malloc(sizeof(float) * d);
  float *u = malloc(sizeof(float) * d);
  uint32_t st = 0;
  for (int t = t0; t < t1; t++) {
    int b = t / D->h_v, h = t % D->h_v;
    int s = slot_of(D, slots, b, &st);
    float *o = o_all + ((size_t)b * D->h_v + h) * d;
    if (s < 0) { memset(o, 0, sizeof(float) * d); continue; }
    int hk = h / (D->h_v / D->h_k);
    const float *q = q_all + ((size_t)b * D->h_k + hk) * d;
    const float *k = k_all + ((size_t)b * D->h_k + hk) * d;
    const float *v = v_all + ((size_t)b * D->h_v + h) * d;
    float beta = beta_all[(size_t)b * D->h_v + h];
    const float *gate = gate_vector(D, g_all, b, h, gbuf);
    float *S = Spool + ((size_t)s * D->h_v + h) * d * d;
    for (int i = 0; i < d; i++)
      for (int j = 0; j < d; j++) S[i * d + j] = gate[i] * S[i * d + j];
    for (int j = 0; j < d; j++) {
      float P = exact_dot(S + j, (size_t)d, k, NULL, d);
      u[j] = beta * (v[j] - P);
    }
    for (int i = 0; i < d; i++)
      for (int j = 0; j < d; j++) S[i * d + j] = fmaf(k[i], u[j], S[i * d + j]);
    for (int j = 0; j < d; j++) {
      o[j] = exact_dot(S + j, (size_t)d, q, NULL, d);
      if (isnan(o[j])) st |= ST_NAN;
    }
  }
  free(gbuf); free(u);
  return st;
}

uint32_t sqo_step_fp32(const sqo_desc *D, float *Spool, const float *q, const float *k, const float *v,
                       const float *beta, const float *g, float *o, const int32_t *slots, int B) {
  return sqo_step_fp32_tiles(D, Spool, q, k, v, beta, g, o, slots, 0, B * D->h_v);
}

/* ------------------------------------------------ per-window variant */
/* Per-window quantization ("线性注意力每生成一个token都要搬状态，LeapQuant
 * 把它压到8位还不掉点" (wink.run), the first of the three techniques): the
 * packed state is not requantized after every token; it stays frozen for a
 * window of W tokens, the tokens' updates are kept at high precision in a
 * buffer, the outputs come from the frozen state and the buffer together,
 * and at the end of the window the state is requantized once.
 *
 * Window buffer (this project's layout): per (slot, value head) a record of
 * sqo_window_record_bytes() bytes: [int32 count, 12 pad bytes]
 * [k: W x d fp32][u: W x d fp32][gates: W x gd fp32, padded to 16 B], gd = d
 * for one gate per key channel, 1 for one per head. count tokens are
 * buffered (0 <= count < W); token tau's key k_tau, its u_tau and its gate
 * G_tau are stored at row tau.
 *
 * One token for a tile with n buffered tokens (current token = n), in fp64
 * (every product and sum below in double; only u and o are rounded to
 * fp32, u because the buffer stores it in fp32):
 *   S0_ij = V_ij M_i c_j, the frozen state (V, M as in load_VM without gate)
 *   D_tau,i = prod_{sigma = tau+1 .. n} G_sigma,i (tau = -1 .. n-1; D_-1
 *            decays S0 through token n)
 *   Sg_ij = D_-1,i S0_ij + sum_{tau<n} D_tau,i k_tau,i u_tau,j
 *           (the state after the buffered tokens, gated by G_n)
 *   p_j = sum_i Sg_ij k_n,i ; u_n,j = fp32(beta (v_j - p_j))
 *   S_ij = Sg_ij + k_n,i u_n,j ; o_j = fp32(sum_i S_ij q_n,i)
 * then token n is appended (count n + 1), and when count reaches W the
 * state is requantized once by the step's requantization (store_T) from
 * its column-normalised form, summed in fp32 like the step's T' (below),
 * and count returns to 0.
 * A slot id out of range skips the tile (o = 0, status bit). */
static size_t window_gate_floats(const sqo_desc *D, int W) {
  size_t n = (size_t)W * (D->gate_kind == 0 ? 1 : (size_t)D->d);
  return (n + 3) / 4 * 4;
}
size_t sqo_window_record_bytes(const sqo_desc *D, int W) {
  return 16 + 4 * (2 * (size_t)W * D->d + window_gate_floats(D, W));
}

static uint32_t window_tile(const sqo_desc *D, uint8_t *rec, uint8_t *wrec, int W, int b, int h,
                            const float *q_all, const float *k_all, const float *v_all,
                            const float *beta_all, const float *g_all, float *o_all) {
  int d = D->d;
  int hk = h / (D->h_v / D->h_k);
  const float *q = q_all + ((size_t)b * D->h_k + hk) * d;
  const float *k = k_all + ((size_t)b * D->h_k + hk) * d;
  const float *v = v_all + ((size_t)b * D->h_v + h) * d;
  double beta = beta_all[(size_t)b * D->h_v + h];
  float *o = o_all + ((size_t)b * D->h_v + h) * d;
  const float *c = D->col_scale + (size_t)h * d;
  int gd = D->gate_kind == 0 ? 1 : d;
  int32_t n;
  memcpy(&n, wrec, 4);
  float *kb = (float *)(wrec + 16);
  float *ub = kb + (size_t)W * d;
  float *gb = ub + (size_t)W * d;
  uint32_t st = 0;
  float *V = malloc(sizeof(float) * d * d);
  float *M = malloc(sizeof(float) * d);
  double *S = malloc(sizeof(double) * d * d);
  double *Dg = malloc(sizeof(double) * (W + 1) * d); /* Dg[(tau+1) d + i] = D_tau,i */
  float *T = malloc(sizeof(float) * d * d);
  load_VM(D, h, rec, NULL, V, M);
  /* the current token's gate */
  float *gcur = gb + (size_t)n * gd;
  for (int x = 0; x < gd; x++) gcur[x] = D->gate_kind == 0 ? g_all[(size_t)b * D->h_v + h]
                                                           : g_all[((size_t)b * D->h_v + h) * d + x];
  for (int i = 0; i < d; i++) {
    double acc = 1.0;
    for (int tau = n - 1; tau >= -1; tau--) {
      acc *= (double)gb[(size_t)(tau + 1) * gd + (gd == 1 ? 0 : i)];
      Dg[(size_t)(tau + 1) * d + i] = acc;
    }
  }
  for (int i = 0; i < d; i++)
    for (int j = 0; j < d; j++) {
      double s = Dg[i] * ((double)V[i * d + j] * (double)M[i] * (double)c[j]);
      for (int tau = 0; tau < n; tau++)
        s += Dg[(size_t)(tau + 1) * d + i] * (double)kb[(size_t)tau * d + i] * (double)ub[(size_t)tau * d + j];
      S[i * d + j] = s;
    }
  float *un = ub + (size_t)n * d;
  for (int j = 0; j < d; j++) {
    double p = 0.0;
    for (int i = 0; i < d; i++) p += S[i * d + j] * (double)k[i];
    un[j] = (float)(beta * ((double)v[j] - p));
  }
  for (int i = 0; i < d; i++) kb[(size_t)n * d + i] = k[i];
  for (int i = 0; i < d; i++)
    for (int j = 0; j < d; j++) S[i * d + j] += (double)k[i] * (double)un[j];
  for (int j = 0; j < d; j++) {
    double acc = 0.0;
    for (int i = 0; i < d; i++) acc += S[i * d + j] * (double)q[i];
    o[j] = (float)acc;
    if (isnan(o[j])) st |= ST_NAN;
  }
  n += 1;
  if (n == W) {
    /* The window's W tokens are all in the buffer (the current one last,
     * with no gate after it). In the column-normalised units of the
     * record, the state is the frozen term plus W rank-one terms:
     *   T_ij = V_ij a_i + sum_tau e_tau,i w_tau,j
     *   a_i = fp32(D_-1,i M_i), e_tau,i = fp32(D_tau,i k_tau,i) (D = 1 for the
     *   current token), w_tau,j = fp32(u_tau,j ic_j), as the step's w = u / c;
     * summed in fp32 the way the step forms T': t = fmaf(e, w, t) over the
     * tokens in order from t = 0, then T = fmaf(V, a, t). */
    for (int i = 0; i < d; i++) {
      const float a = (float)(Dg[i] * (double)M[i]);
      for (int j = 0; j < d; j++) {
        const float ic = 1.0f / c[j];
        float t = 0.0f;
        for (int tau = 0; tau < W; tau++) {
          const double Dt = tau < W - 1 ? Dg[(size_t)(tau + 1) * d + i] : 1.0;
          const float e = (float)(Dt * (double)kb[(size_t)tau * d + i]);
          const float w = ub[(size_t)tau * d + j] * ic;
          t = fmaf(e, w, t);
        }
        T[i * d + j] = fmaf(V[i * d + j], a, t);
      }
    }
    st |= store_T(D, h, rec, T);
    n = 0;
  }
  memcpy(wrec, &n, 4);
  free(V); free(M); free(S); free(Dg); free(T);
  return st;
}

/* One token of the per-window variant for tiles [t0, t1) of a batch of B
 * requests (inputs as in sqo_step_tiles); wbuf is [n_slots][h_v] window
 * records. Returns the status bits. */
uint32_t sqo_window_step_tiles(const sqo_desc *D, uint8_t *pool, uint8_t *wbuf, int W, const float *q,
                               const float *k, const float *v, const float *beta, const float *g, float *o,
                               const int32_t *slots, int t0, int t1) {
  int d = D->d;
  uint32_t st = 0;
  size_t slot_bytes = sqo_slot_bytes(D);
  size_t wrb = sqo_window_record_bytes(D, W);
  for (int t = t0; t < t1; t++) {
    int b = t / D->h_v, h = t % D->h_v;
    int s = slot_of(D, slots, b, &st);
    if (s < 0) {
      memset(o + ((size_t)b * D->h_v + h) * d, 0, sizeof(float) * d);
      continue;
    }
    uint8_t *rec = pool + (size_t)s * slot_bytes + sqo_head_offset(D, h);
    uint8_t *wrec = wbuf + ((size_t)s * D->h_v + h) * wrb;
    st |= window_tile(D, rec, wrec, W, b, h, q, k, v, beta, g, o);
  }
  return st;
}
