/*
 * fp8q oracle: plain, slow, obviously correct CPU definitions of the
 * block-scaled FP8 linear-layer path.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load or call this file. It shares no code,
 * header, table or constant generator with the CUDA library, and the CUDA
 * library never calls it.
 *
 * The method: "Resumen Técnico: Jet-RL" (gist.science, paper 2601.14243),
 * section "Esquema de Cuantización":
 *   - activations are quantized per 1x128 group,
 *   - weights per 128x128 block,
 *   - activations saved for backward are stored in FP8, produced inside the
 *     preceding operator,
 *   - gradients between operators stay BF16,
 *   - DGrad and WGrad run in FP8, WGrad with 1x128 and 128x1 grouping.
 * Section "Implementación" names fused activation/RMSNorm and transposition
 * kernels next to the quantizers.
 *
 * Where the page is silent, each function states the reading it takes:
 *   - FP8 is OCP E4M3 "fn": bias 7, no infinities, max finite 448;
 *   - a group's scale is s = fl32(amax / 448); an all-zero group has s = 1;
 *   - t = fl32(x / s) (IEEE division), code = nearest E4M3 value to t,
 *     ties to even mantissa, |t| >= 448 saturates to +-448, sign kept (-0 -> 0x80);
 *   - RMSNorm rounds to BF16 before quantizing; SwiGLU likewise.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math -fopenmp
 * (no FMA contraction, IEEE single-precision division, no flush-to-zero).
 * OpenMP only splits independent rows/blocks; no sum changes order.
 */
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>

#if defined(__FAST_MATH__)
#error "the oracle must be built without -ffast-math"
#endif

typedef int64_t i64;

/* ------------------------------------------------------------------ */
/* E4M3 "fn" decode/encode, from the format definition (OCP 8-bit FP   */
/* specification v1.0, E4M3: 1 sign, 4 exponent bits with bias 7,      */
/* 3 mantissa bits; exponent 0 is subnormal; S.1111.111 is NaN; no inf) */
/* ------------------------------------------------------------------ */

/* Value of an E4M3 code as a double (exact). NaN code returns NAN. */
double oracle_e4m3_decode(uint8_t c) {
  int sign = (c >> 7) & 1;
  int e = (c >> 3) & 0xF;
  int m = c & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);            /* m/8 * 2^(1-7) */
  else v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* Magnitudes of the 127 non-negative finite codes 0x00..0x7E, which the
 * definition above makes strictly increasing in the code. Filled once. */
static double g_mag[127];
static int g_mag_ready = 0;

static void init_mag(void) {
  if (g_mag_ready) return;
  for (int c = 0; c < 127; ++c) g_mag[c] = oracle_e4m3_decode((uint8_t)c);
  g_mag_ready = 1;
}

/* Nearest E4M3 value to the fp32 number t (round to nearest, ties to the
 * code whose mantissa LSB is 0), saturating to +-448, sign preserved.
 * NaN input is outside the contract (returns the NaN code 0x7F). */
uint8_t oracle_e4m3_encode(float t) {
  init_mag();
  if (isnan(t)) return 0x7F;
  uint8_t sign = signbit(t) ? 0x80 : 0x00;
  double a = fabs((double)t);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  /* largest code lo with mag(lo) <= a (binary search over the sorted table) */
  int lo = 0, hi = 126;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if (g_mag[mid] <= a) lo = mid; else hi = mid - 1;
  }
  if (g_mag[lo] == a) return (uint8_t)(sign | lo);
  int up = lo + 1; /* exists: a < 448 = mag(126) */
  double dlo = a - g_mag[lo], dup = g_mag[up] - a; /* exact in double */
  int pick;
  if (dlo < dup) pick = lo;
  else if (dup < dlo) pick = up;
  else pick = (lo & 1) ? up : lo; /* tie: even mantissa (code LSB = mantissa LSB) */
  return (uint8_t)(sign | pick);
}

/* ------------------------------------------------------------------ */
/* BF16 <-> fp32                                                        */
/* ------------------------------------------------------------------ */

float oracle_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round an fp32 value to the nearest BF16 (ties to even), by comparing the two
 * BF16 neighbours of x exactly in double. Overflow rounds to infinity. */
uint16_t oracle_f32_to_bf16(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000);
  uint32_t mag = u & 0x7FFFFFFFu;
  uint16_t lo = (uint16_t)(mag >> 16);            /* truncation toward zero */
  if ((mag & 0xFFFFu) == 0) return (uint16_t)(sign | lo);
  uint16_t up = (uint16_t)(lo + 1);               /* next BF16 magnitude    */
  double a = fabs((double)x);
  double vlo = (double)oracle_bf16_to_f32(lo);
  double vup = (up >= 0x7F80) ? INFINITY : (double)oracle_bf16_to_f32(up);
  uint16_t pick;
  if (isinf(vup)) {
    /* the midpoint between the largest finite BF16 and 2^128 decides */
    double vmax = vlo, mid = vmax + ldexp(1.0, 127 - 8);
    pick = (a < mid) ? lo : ((a > mid) ? 0x7F80 : ((lo & 1) ? 0x7F80 : lo));
    return (uint16_t)(sign | pick);
  }
  double dlo = a - vlo, dup = vup - a;
  if (dlo < dup) pick = lo;
  else if (dup < dlo) pick = up;
  else pick = (lo & 1) ? up : lo;
  return (uint16_t)(sign | pick);
}

/* ------------------------------------------------------------------ */
/* One quantization group (1x128, 128x1 or 128x128).                    */
/* s = fl32(amax / 448); zero group -> s = 1; q_i = enc(fl32(x_i / s)).  */
/* ------------------------------------------------------------------ */

static float group_scale(float amax) {
  if (amax == 0.0f) return 1.0f;
  volatile float s = amax / 448.0f; /* IEEE single division */
  return s;
}

static uint8_t quant_one(float x, float s) {
  volatile float t = x / s; /* IEEE single division, correctly rounded */
  return oracle_e4m3_encode(t);
}

/* Groups along a dimension of n elements, and the width of group g: every group
 * has 128 elements except, when n is not a multiple of 128, the last one, which has
 * the n % 128 remaining elements. Reading (the page fixes only the 1x128 / 128x128
 * grouping): a partial group is the full group with zeros in the missing places;
 * zeros raise no maximum, so its scale comes from its valid elements alone, and the
 * codes of the missing places, which would all be 0, are not stored. */
static i64 ngroups(i64 n) { return (n + 127) / 128; }
static int gwidth(i64 n, i64 g) { return n - g * 128 < 128 ? (int)(n - g * 128) : 128; }

/* ------------------------------------------------------------------ */
/* a1: activation quantization per 1x128 group.                         */
/* x [M][K] BF16 (row stride ldx) -> q [M][K] (row stride K),            */
/* s [K/128][lds] fp32 (scale of row m, group g at s[g*lds + m]).        */
/* Jet-RL summary, "Esquema de Cuantización", activations bullet.        */
/* ------------------------------------------------------------------ */
void oracle_quant_act_1x128(const uint16_t* x, i64 M, i64 K, i64 ldx,
                            uint8_t* q, float* s, i64 lds) {
  init_mag();
  i64 G = ngroups(K);
#pragma omp parallel for schedule(static)
  for (i64 m = 0; m < M; ++m) {
    for (i64 g = 0; g < G; ++g) {
      int w = gwidth(K, g);
      float amax = 0.0f;
      for (int i = 0; i < w; ++i) {
        float v = fabsf(oracle_bf16_to_f32(x[m * ldx + g * 128 + i]));
        if (v > amax) amax = v;
      }
      float sc = group_scale(amax);
      s[g * lds + m] = sc;
      for (int i = 0; i < w; ++i)
        q[m * K + g * 128 + i] = quant_one(oracle_bf16_to_f32(x[m * ldx + g * 128 + i]), sc);
    }
  }
}

/* ------------------------------------------------------------------ */
/* a2: weight quantization per 128x128 block.                           */
/* w [N][K] BF16 (row stride ldw) -> q [N][K], s [N/128][K/128],         */
/* and, when qT is not NULL, the same codes transposed: qT [K][N].       */
/* Jet-RL summary, "Esquema de Cuantización", weights bullet.            */
/* ------------------------------------------------------------------ */
void oracle_quant_weight_128x128(const uint16_t* w, i64 N, i64 K, i64 ldw,
                                 uint8_t* q, float* s, uint8_t* qT) {
  init_mag();
  i64 NB = ngroups(N), KB = ngroups(K);
#pragma omp parallel for schedule(static)
  for (i64 blk = 0; blk < NB * KB; ++blk) {
    i64 nb = blk / KB, kb = blk % KB;
    int hr = gwidth(N, nb), wc = gwidth(K, kb);
    float amax = 0.0f;
    for (i64 r = 0; r < hr; ++r)
      for (i64 c = 0; c < wc; ++c) {
        float v = fabsf(oracle_bf16_to_f32(w[(nb * 128 + r) * ldw + kb * 128 + c]));
        if (v > amax) amax = v;
      }
    float sc = group_scale(amax);
    s[nb * KB + kb] = sc;
    for (i64 r = 0; r < hr; ++r)
      for (i64 c = 0; c < wc; ++c) {
        i64 n = nb * 128 + r, k = kb * 128 + c;
        uint8_t code = quant_one(oracle_bf16_to_f32(w[n * ldw + k]), sc);
        q[n * K + k] = code;
        if (qT) qT[k * N + n] = code;
      }
  }
}

/* ------------------------------------------------------------------ */
/* a3: RMSNorm fused with 1x128 quantization (the FP8 saved activation). */
/* Jet-RL summary, "Esquema de Cuantización" (saved activations in FP8,  */
/* fused with the previous operator) and "Implementación" (fused RMSNorm */
/* kernels). Reading: the fused kernel equals an unfused BF16 RMSNorm    */
/* followed by the 1x128 quantizer:                                      */
/*   ss = sum_i x_i^2 in fp64 (each term exact)                          */
/*   r  = (float)(1 / sqrt(ss/H + eps)) in fp64                          */
/*   y_i = bf16( fl32( fl32(x_i * r) * gamma_i ) )                       */
/* y (if not NULL) receives the BF16 normalised row [M][H].              */
/* ------------------------------------------------------------------ */
float oracle_rmsnorm_rstd(const uint16_t* xrow, i64 H, float eps) {
  double ss = 0.0;
  for (i64 i = 0; i < H; ++i) {
    double v = (double)oracle_bf16_to_f32(xrow[i]);
    ss += v * v;
  }
  double ms = ss / (double)H;
  double r = 1.0 / sqrt(ms + (double)eps);
  return (float)r;
}

void oracle_rmsnorm_quant(const uint16_t* x, const uint16_t* gamma, i64 M, i64 H,
                          i64 ldx, float eps, uint8_t* q, float* s, i64 lds,
                          uint16_t* y) {
  init_mag();
  i64 G = ngroups(H);
#pragma omp parallel for schedule(static)
  for (i64 m = 0; m < M; ++m) {
    const uint16_t* xr = x + m * ldx;
    float r = oracle_rmsnorm_rstd(xr, H, eps);
    for (i64 g = 0; g < G; ++g) {
      int w = gwidth(H, g);
      float yv[128];
      float amax = 0.0f;
      for (int i = 0; i < w; ++i) {
        i64 c = g * 128 + i;
        volatile float t1 = oracle_bf16_to_f32(xr[c]) * r;
        volatile float t2 = t1 * oracle_bf16_to_f32(gamma[c]);
        uint16_t yb = oracle_f32_to_bf16(t2);
        if (y) y[m * H + c] = yb;
        yv[i] = oracle_bf16_to_f32(yb);
        float a = fabsf(yv[i]);
        if (a > amax) amax = a;
      }
      float sc = group_scale(amax);
      s[g * lds + m] = sc;
      for (int i = 0; i < w; ++i) q[m * H + g * 128 + i] = quant_one(yv[i], sc);
    }
  }
}

/* ------------------------------------------------------------------ */
/* a4: SwiGLU fused with 1x128 quantization.                            */
/* Jet-RL summary, "Implementación" (fused activation kernels) and      */
/* "Esquema de Cuantización" (saved activations in FP8).                 */
/* Reading: gu [M][2I] holds gate in columns 0..I-1 and up in I..2I-1;  */
/*   e = E(-g); silu = fl32(g / fl32(1 + e)); h = bf16(fl32(silu * u)). */
/* E is the method's fixed fp32 exponential, defined here as Cody-Waite  */
/* range reduction (W. J. Cody and W. Waite, "Software Manual for the    */
/* Elementary Functions", 1980) followed by the degree-7 Taylor          */
/* polynomial of e^r in Horner form, on x clamped to [-80, 88]:          */
/*   n = rint(fl32(x * log2e)); r = fma(-n, LN2_HI, x); r = fma(-n, LN2_LO, r)
 *   p = Horner(1/7!, ..., 1/2!, 1, 1)(r) with fma; E = p * 2^n (exact).
 * LN2_HI = ln2 rounded to 12 significant bits (n*LN2_HI is exact for    */
/* |n| < 2^12); LN2_LO = fl32(ln2 - LN2_HI); the Taylor coefficients are */
/* fl32(1/k!). Clamping at -80 changes nothing downstream: 1 + e == 1    */
/* in fp32 for any e < 2^-24.                                            */
/* ------------------------------------------------------------------ */
float oracle_exp_cw(float x) {
  const float LOG2E = 0x1.715476p+0f;   /* fl32(1/ln2)          */
  const float LN2_HI = 0x1.62ep-1f;     /* 2839 / 4096          */
  const float LN2_LO = 0x1.0bfbe8p-15f; /* fl32(ln2 - LN2_HI)   */
  const float C7 = 0x1.a01a02p-13f;     /* fl32(1/5040)         */
  const float C6 = 0x1.6c16c2p-10f;     /* fl32(1/720)          */
  const float C5 = 0x1.111112p-7f;      /* fl32(1/120)          */
  const float C4 = 0x1.555556p-5f;      /* fl32(1/24)           */
  const float C3 = 0x1.555556p-3f;      /* fl32(1/6)            */
  const float C2 = 0x1p-1f;
  const float C1 = 1.0f, C0 = 1.0f;
  if (x < -80.0f) x = -80.0f;
  if (x > 88.0f) x = 88.0f;
  volatile float xl = x * LOG2E;
  float n = rintf(xl); /* round half to even in the default mode */
  float r = fmaf(-n, LN2_HI, x);
  r = fmaf(-n, LN2_LO, r);
  float p = C7;
  p = fmaf(p, r, C6);
  p = fmaf(p, r, C5);
  p = fmaf(p, r, C4);
  p = fmaf(p, r, C3);
  p = fmaf(p, r, C2);
  p = fmaf(p, r, C1);
  p = fmaf(p, r, C0);
  return ldexpf(p, (int)n); /* exact: the result is a normal float */
}

uint16_t oracle_swiglu_one(uint16_t gate, uint16_t up) {
  float g = oracle_bf16_to_f32(gate), u = oracle_bf16_to_f32(up);
  float e = oracle_exp_cw(-g);
  volatile float d = 1.0f + e;
  volatile float silu = g / d;
  volatile float h = silu * u;
  return oracle_f32_to_bf16(h);
}

void oracle_swiglu_quant(const uint16_t* gu, i64 M, i64 I, i64 ldgu,
                         uint8_t* q, float* s, i64 lds, uint16_t* h) {
  init_mag();
  i64 G = ngroups(I);
#pragma omp parallel for schedule(static)
  for (i64 m = 0; m < M; ++m) {
    for (i64 g = 0; g < G; ++g) {
      int w = gwidth(I, g);
      float hv[128];
      float amax = 0.0f;
      for (int i = 0; i < w; ++i) {
        i64 c = g * 128 + i;
        uint16_t hb = oracle_swiglu_one(gu[m * ldgu + c], gu[m * ldgu + I + c]);
        if (h) h[m * I + c] = hb;
        hv[i] = oracle_bf16_to_f32(hb);
        float a = fabsf(hv[i]);
        if (a > amax) amax = a;
      }
      float sc = group_scale(amax);
      s[g * lds + m] = sc;
      for (int i = 0; i < w; ++i) q[m * I + g * 128 + i] = quant_one(hv[i], sc);
    }
  }
}

/* ------------------------------------------------------------------ */
/* Backward of the SwiGLU producer, in BF16 (Jet-RL summary, "Esquema de */
/* Cuantización": gradients between operators stay BF16). The page       */
/* gives no formula; this is the derivative of h = silu(g) * u with      */
/* silu(g) = g * sigma(g), sigma(g) = 1 / (1 + e^-g):                    */
/*   dL/du = dh * silu(g),  dL/dg = dh * u * sigma(g) * (1 + g*(1 - sigma(g))). */
/* Reading (every step one IEEE fp32 operation, no contraction; the      */
/* exponential and silu exactly as in the forward producer):             */
/*   e = E(-g); d = fl32(1 + e); silu = fl32(g / d); sig = fl32(1 / d);   */
/*   du = bf16(fl32(dh * silu));                                         */
/*   ds = fl32(sig * fl32(1 + fl32(g * fl32(1 - sig))));                  */
/*   dg = bf16(fl32(fl32(dh * u) * ds)).                                 */
/* Layout: gu and dgu [M][2I] with gate / d_gate in columns 0..I-1 and   */
/* up / d_up in I..2I-1; dh [M][I].                                      */
/* ------------------------------------------------------------------ */
void oracle_swiglu_bwd_one(uint16_t gate, uint16_t up, uint16_t dhb, uint16_t* dgate,
                           uint16_t* dup) {
  float g = oracle_bf16_to_f32(gate), u = oracle_bf16_to_f32(up);
  float dh = oracle_bf16_to_f32(dhb);
  float e = oracle_exp_cw(-g);
  volatile float d = 1.0f + e;
  volatile float silu = g / d;
  volatile float sig = 1.0f / d;
  volatile float du = dh * silu;
  volatile float t1 = 1.0f - sig;
  volatile float t2 = g * t1;
  volatile float t3 = 1.0f + t2;
  volatile float ds = sig * t3;
  volatile float dhu = dh * u;
  volatile float dg = dhu * ds;
  *dgate = oracle_f32_to_bf16(dg);
  *dup = oracle_f32_to_bf16(du);
}

void oracle_swiglu_bwd(const uint16_t* gu, const uint16_t* dh, i64 M, i64 I,
                       uint16_t* dgu) {
#pragma omp parallel for schedule(static)
  for (i64 m = 0; m < M; ++m)
    for (i64 c = 0; c < I; ++c)
      oracle_swiglu_bwd_one(gu[m * 2 * I + c], gu[m * 2 * I + I + c], dh[m * I + c],
                            &dgu[m * 2 * I + c], &dgu[m * 2 * I + I + c]);
}

/* ------------------------------------------------------------------ */
/* Exact sum of fp32 numbers, rounded once (the reductions of the         */
/* RMSNorm backward). Every finite fp32 value is an integer multiple of   */
/* 2^-149 (the smallest subnormal), so a sum of them is that integer      */
/* times 2^-149. The integer is kept in two's complement over ten         */
/* little-endian 32-bit words (320 bits: room for 2^42 terms of the       */
/* largest magnitude), every addition carried through all the words (a    */
/* Kulisch accumulator). No term is ever rounded, so the result does not  */
/* depend on the order of the additions.                                  */
/* ------------------------------------------------------------------ */
#define XACC_WORDS 10
typedef struct { uint32_t w[XACC_WORDS]; } xacc;

static void xacc_zero(xacc* a) { memset(a, 0, sizeof(*a)); }

static void xacc_add_f32(xacc* a, float t) {
  uint32_t u;
  memcpy(&u, &t, 4);
  uint32_t E = (u >> 23) & 0xFFu, f = u & 0x7FFFFFu;
  /* |t| = m * 2^(sh - 149): normal numbers carry the implicit bit */
  uint64_t m = E ? (uint64_t)(f | 0x800000u) : (uint64_t)f;
  int sh = E ? (int)E - 1 : 0;
  uint32_t term[XACC_WORDS];
  memset(term, 0, sizeof(term));
  uint64_t x = m << (sh % 32); /* < 2^55: two words */
  term[sh / 32] = (uint32_t)x;
  term[sh / 32 + 1] = (uint32_t)(x >> 32);
  if (u >> 31) { /* negative: two's complement of the term */
    uint64_t c = 1;
    for (int i = 0; i < XACC_WORDS; ++i) {
      uint64_t v = (uint64_t)(uint32_t)~term[i] + c;
      term[i] = (uint32_t)v;
      c = v >> 32;
    }
  }
  uint64_t c = 0;
  for (int i = 0; i < XACC_WORDS; ++i) {
    uint64_t v = (uint64_t)a->w[i] + term[i] + c;
    a->w[i] = (uint32_t)v;
    c = v >> 32;
  }
}

static int xacc_bit(const uint32_t* w, int i) { return i >= 0 ? (int)((w[i / 32] >> (i % 32)) & 1u) : 0; }

/* The accumulated value rounded to a double: to nearest, ties to even; or,
 * with odd != 0, to odd (the last mantissa bit forced to 1 when any lower
 * bit is dropped). A double rounded to odd and then rounded to fp32 (to
 * nearest even) is the fp32 nearest to the exact value, since 53 >= 24 + 2
 * (S. Boldo, G. Melquiond, "Emulation of FMA and correctly rounded sums:
 * proved algorithms using rounding to odd", IEEE Trans. Computers 2008).
 * An exact zero gives +0. */
static double xacc_round(const xacc* a, int odd) {
  uint32_t mag[XACC_WORDS];
  memcpy(mag, a->w, sizeof(mag));
  int neg = (int)(mag[XACC_WORDS - 1] >> 31);
  if (neg) {
    uint64_t c = 1;
    for (int i = 0; i < XACC_WORDS; ++i) {
      uint64_t v = (uint64_t)(uint32_t)~mag[i] + c;
      mag[i] = (uint32_t)v;
      c = v >> 32;
    }
  }
  int p = -1; /* highest set bit of the magnitude */
  for (int i = XACC_WORDS * 32 - 1; i >= 0; --i)
    if (xacc_bit(mag, i)) { p = i; break; }
  if (p < 0) return 0.0;
  uint64_t mant = 0; /* bits p .. p-52 */
  for (int i = p; i > p - 53; --i) mant = (mant << 1) | (uint64_t)xacc_bit(mag, i);
  int round = xacc_bit(mag, p - 53), sticky = 0;
  for (int i = p - 54; i >= 0; --i) sticky |= xacc_bit(mag, i);
  if (odd) {
    if (round || sticky) mant |= 1u;
  } else if (round && (sticky || (mant & 1u))) {
    mant += 1u; /* may reach 2^53, still exact as a double */
  }
  double v = ldexp((double)mant, p - 52 - 149);
  return neg ? -v : v;
}

/* The accumulated value rounded once to the nearest fp32 (ties to even). */
static float xacc_round_f32(const xacc* a) { return (float)xacc_round(a, 1); }

/* Exported for the tests: the exact sum of t[0..n) rounded once, to the
 * nearest double (to_f32 == 0) or to the nearest fp32 (to_f32 != 0, returned
 * as a double). */
double oracle_exact_sum_f32(const float* t, i64 n, int to_f32) {
  xacc a;
  xacc_zero(&a);
  for (i64 i = 0; i < n; ++i) xacc_add_f32(&a, t[i]);
  if (to_f32) return (double)xacc_round_f32(&a);
  return xacc_round(&a, 0);
}

/* ------------------------------------------------------------------ */
/* Backward of the RMSNorm producer, in BF16, with the residual          */
/* gradient added (the gradient that flows on along the residual        */
/* stream). Forward: y_j = x_j * r * gamma_j, r = (mean(x^2) + eps)^-1/2. */
/* Derivative: dx_j = r * gamma_j * dy_j - x_j * r^3 * c / H with        */
/* c = sum_j gamma_j * dy_j * x_j; dgamma_j = sum_m dy_mj * x_mj * r_m.  */
/* Reading (the page gives no formula; rounding as an unfused BF16       */
/* RMSNorm backward followed by a BF16 residual add; the two reductions  */
/* are exact sums rounded once, so no summation order enters them):      */
/*   r as in the forward producer (oracle_rmsnorm_rstd);                 */
/*   c = the exact sum over j of fl32(fl32(gamma_j * dy_j) * x_j),        */
/*       rounded to the nearest double;                                   */
/*   k = (float)((((c * r) * r) * r) / H) in fp64;                        */
/*   dx_j = bf16(fl32(fl32(r * fl32(gamma_j * dy_j)) - fl32(k * x_j)));   */
/*   out_j = bf16(fl32(dx_j + dres_j))  (dres NULL: out_j = dx_j);        */
/*   dgamma_j = the exact sum over m of fl32(dy_mj * fl32(x_mj * r_m)),   */
/*       rounded to the nearest fp32.                                     */
/* r_out (if not NULL) receives r per row, k_out (if not NULL) k.        */
/* ------------------------------------------------------------------ */
void oracle_rmsnorm_bwd(const uint16_t* x, const uint16_t* gamma, const uint16_t* dy,
                        const uint16_t* dres, i64 M, i64 H, float eps, uint16_t* out,
                        float* dgamma, float* r_out, float* k_out) {
  float* rr = (float*)malloc(sizeof(float) * (size_t)M);
#pragma omp parallel for schedule(static)
  for (i64 m = 0; m < M; ++m) {
    const uint16_t* xr = x + m * H;
    const uint16_t* dyr = dy + m * H;
    float r = oracle_rmsnorm_rstd(xr, H, eps);
    xacc cs;
    xacc_zero(&cs);
    for (i64 j = 0; j < H; ++j) {
      volatile float gd = oracle_bf16_to_f32(gamma[j]) * oracle_bf16_to_f32(dyr[j]);
      volatile float t = gd * oracle_bf16_to_f32(xr[j]);
      xacc_add_f32(&cs, t);
    }
    double c = xacc_round(&cs, 0);
    double kd = c * (double)r;
    kd = kd * (double)r;
    kd = kd * (double)r;
    kd = kd / (double)H;
    float k = (float)kd;
    rr[m] = r;
    if (r_out) r_out[m] = r;
    if (k_out) k_out[m] = k;
    for (i64 j = 0; j < H; ++j) {
      float xv = oracle_bf16_to_f32(xr[j]);
      volatile float gd = oracle_bf16_to_f32(gamma[j]) * oracle_bf16_to_f32(dyr[j]);
      volatile float a = r * gd;
      volatile float b = k * xv;
      volatile float dx = a - b;
      uint16_t dxb = oracle_f32_to_bf16(dx);
      if (dres) {
        volatile float o = oracle_bf16_to_f32(dxb) + oracle_bf16_to_f32(dres[m * H + j]);
        out[m * H + j] = oracle_f32_to_bf16(o);
      } else {
        out[m * H + j] = dxb;
      }
    }
  }
  if (dgamma) {
#pragma omp parallel for schedule(static)
    for (i64 j = 0; j < H; ++j) {
      xacc acc;
      xacc_zero(&acc);
      for (i64 m = 0; m < M; ++m) {
        volatile float xr = oracle_bf16_to_f32(x[m * H + j]) * rr[m];
        volatile float t = oracle_bf16_to_f32(dy[m * H + j]) * xr;
        xacc_add_f32(&acc, t);
      }
      dgamma[j] = xacc_round_f32(&acc);
    }
  }
  free(rr);
}

/* ------------------------------------------------------------------ */
/* a6: the BF16 gradient dY [M][N] quantized twice:                     */
/*  row-wise 1x128 (groups along N) for DGrad: q_row [M][N],            */
/*    s_row [N/128][lds_row] (as a1);                                   */
/*  column-wise 128x1 (groups of 128 rows along M) for WGrad, stored     */
/*    transposed: q_colT [N][M], s_col [M/128][N].                      */
/* Jet-RL summary, "Esquema de Cuantización" (BF16 gradients, FP8        */
/* DGrad/WGrad, 1x128 and 128x1 for WGrad) and "Implementación"          */
/* (transposition kernels). q_row/s_row may be NULL.                     */
/* ------------------------------------------------------------------ */
void oracle_transpose_quant_bf16(const uint16_t* dy, i64 M, i64 N, i64 lddy,
                                 uint8_t* q_row, float* s_row, i64 lds_row,
                                 uint8_t* q_colT, float* s_col) {
  init_mag();
  if (q_row && s_row) oracle_quant_act_1x128(dy, M, N, lddy, q_row, s_row, lds_row);
  i64 MB = ngroups(M);
#pragma omp parallel for schedule(static)
  for (i64 n = 0; n < N; ++n) {
    for (i64 mb = 0; mb < MB; ++mb) {
      int w = gwidth(M, mb);
      float amax = 0.0f;
      for (int i = 0; i < w; ++i) {
        float v = fabsf(oracle_bf16_to_f32(dy[(mb * 128 + i) * lddy + n]));
        if (v > amax) amax = v;
      }
      float sc = group_scale(amax);
      s_col[mb * N + n] = sc;
      for (int i = 0; i < w; ++i) {
        i64 m = mb * 128 + i;
        q_colT[n * M + m] = quant_one(oracle_bf16_to_f32(dy[m * lddy + n]), sc);
      }
    }
  }
}

/* ------------------------------------------------------------------ */
/* a8: the saved FP8 activation (1x128 groups) re-grouped 128x1 for      */
/* WGrad. Reading: dequantize each code to fp32, xhat = fl32(s * dec(q)), */
/* then quantize columns in groups of 128 rows and store transposed:     */
/*   q [M][K], s [K/128][lds]  ->  qT [K][M], sT [M/128][K].             */
/* Jet-RL summary, "Esquema de Cuantización" (saved activations in FP8;  */
/* 128x1 grouping for WGrad) and "Implementación" (transposition).       */
/* ------------------------------------------------------------------ */
void oracle_transpose_quant_fp8(const uint8_t* q, const float* s, i64 M, i64 K,
                                i64 lds, uint8_t* qT, float* sT) {
  init_mag();
  i64 MB = ngroups(M);
#pragma omp parallel for schedule(static)
  for (i64 k = 0; k < K; ++k) {
    for (i64 mb = 0; mb < MB; ++mb) {
      int w = gwidth(M, mb);
      float xh[128];
      float amax = 0.0f;
      for (int i = 0; i < w; ++i) {
        i64 m = mb * 128 + i;
        float dec = (float)oracle_e4m3_decode(q[m * K + k]); /* exact */
        volatile float v = s[(k / 128) * lds + m] * dec;
        xh[i] = v;
        float a = fabsf(xh[i]);
        if (a > amax) amax = a;
      }
      float sc = group_scale(amax);
      sT[mb * K + k] = sc;
      for (int i = 0; i < w; ++i) qT[k * M + mb * 128 + i] = quant_one(xh[i], sc);
    }
  }
}

/* ------------------------------------------------------------------ */
/* Dequantization to fp64 (exact: a 4-bit significand times a 24-bit    */
/* scale fits in 53 bits). Used by the GEMM oracle, which takes the dot  */
/* products in fp64 over these values.                                   */
/*   rows-scaled operand:  out[i][k] = s[(k/128)*lds + i] * dec(q[i][k]) */
/*   block-scaled weight:  out[n][k] = s[(n/128)*(K/128) + k/128] * dec  */
/*   column-scaled (128x1, transposed storage qT [C][R], sT [R/128][C]): */
/*                         out[c][r] = sT[(r/128)*C + c] * dec(qT[c][r]) */
/* ------------------------------------------------------------------ */
void oracle_dequant_rows(const uint8_t* q, const float* s, i64 R, i64 K, i64 lds,
                         i64 r0, i64 nr, double* out) {
  init_mag();
#pragma omp parallel for schedule(static)
  for (i64 i = 0; i < nr; ++i)
    for (i64 k = 0; k < K; ++k)
      out[i * K + k] = (double)s[(k / 128) * lds + (r0 + i)] *
                       oracle_e4m3_decode(q[(r0 + i) * K + k]);
  (void)R;
}

void oracle_dequant_block(const uint8_t* q, const float* s, i64 N, i64 K,
                          i64 r0, i64 nr, double* out) {
  init_mag();
  i64 KB = ngroups(K);
#pragma omp parallel for schedule(static)
  for (i64 i = 0; i < nr; ++i)
    for (i64 k = 0; k < K; ++k)
      out[i * K + k] = (double)s[((r0 + i) / 128) * KB + k / 128] *
                       oracle_e4m3_decode(q[(r0 + i) * K + k]);
  (void)N;
}

void oracle_dequant_cols(const uint8_t* qT, const float* sT, i64 C, i64 R,
                         i64 c0, i64 nc, double* out) {
  init_mag();
#pragma omp parallel for schedule(static)
  for (i64 i = 0; i < nc; ++i)
    for (i64 r = 0; r < R; ++r)
      out[i * R + r] = (double)sT[(r / 128) * C + (c0 + i)] *
                       oracle_e4m3_decode(qT[(c0 + i) * R + r]);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
