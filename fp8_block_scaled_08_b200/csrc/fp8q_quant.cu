// Quantizer kernels of libfp8q (sm_100a): the 1x128 activation quantizer, the
// 128x128 weight quantizer, fused RMSNorm+quantize, fused SwiGLU+quantize, the
// dual (row 1x128 + transposed column 128x1) quantizer of BF16 gradients, the
// transposed 128x1 requantizer of saved FP8 activations, the producers that emit
// both groupings of their BF16 output (RMSNorm, SwiGLU), and the RMSNorm / SwiGLU
// backward in BF16 with the dual gradient quantizer fused behind them.
//
// All of them are HBM-bound: BF16 is read with 16-byte loads that a warp issues as
// contiguous runs, group maxima are taken with warp shuffles, and the codes come from
// the hardware E4M3 conversion (round to nearest even, saturate). A group's scale is
// s = amax/448 by IEEE division (s = 1 for an all-zero group); each code is the E4M3
// value nearest to the IEEE quotient x/s. Where x is a BF16 value (every quantizer
// but the FP8 requantizer) the quotient is formed from the correctly rounded
// reciprocal r = 1/s with one residual correction (q = x*r; e = fma(-q, s, x);
// q = fma(e, r, q); sign of x; the kernels evaluate it as q - (q*s - x)*r, which keeps
// the sign of -0 by itself), which yields the same E4M3 code as the IEEE quotient
// for every BF16 x and every BF16 amax >= |x| with s >= 2^-80 (checked exhaustively by
// the test suite); groups with smaller s use the IEEE division itself.
//
// Method: "Resumen Técnico: Jet-RL" (gist.science, paper 2601.14243), section
// "Esquema de Cuantización" (1x128 activation groups, 128x128 weight blocks,
// FP8 saved activations produced by the preceding operator, BF16 gradients,
// 1x128 / 128x1 WGrad grouping) and section "Implementación" (fused
// activation/RMSNorm and transposition kernels).
#include <algorithm>
#include <atomic>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fp8q_device.cuh"
#include "fp8q_host.h"

namespace fp8q {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kSmallScale = 0x1p-80f;  // below it the quotient uses IEEE division

// ---------------------------------------------------------------------------
// Group scale and quotient
// ---------------------------------------------------------------------------
struct GroupScale {
  float s, rs, ns;  // scale, its correctly rounded reciprocal, -scale
  bool small;       // s < 2^-80 (or a tiny amax): quotients by IEEE division
};

// Scale of a group with an arbitrary fp32 amax: s = amax/448 (IEEE), s = 1 if amax = 0.
__device__ __forceinline__ GroupScale group_scale(float amax) {
  GroupScale g;
  g.s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
  g.rs = __frcp_rn(g.s);
  g.ns = -g.s;
  g.small = g.s < kSmallScale;
  return g;
}

// For amax = (1 + i/128) * 2^E, a normal BF16 value: amax/448 = ((1 + i/128)/7) * 2^(E-6),
// and scaling by a power of two commutes with rounding while the result stays a normal
// float, so fl32(amax/448) = kScaleMant[i] * 2^(E-6) and fl32(1/s) = kRecipMant[i] *
// 2^(6-E), with kScaleMant[i] = fl32((1 + i/128)/7) and kRecipMant[i] =
// fl32(1/kScaleMant[i]) (values below; the test suite re-derives them and checks the
// identity for every BF16 amax with E >= -71).
__constant__ float kScaleMant[128] = {
    0x1.24924ap-3f, 0x1.26db6ep-3f, 0x1.292492p-3f, 0x1.2b6db6p-3f, 0x1.2db6dcp-3f, 0x1.3p-3f,
    0x1.324924p-3f, 0x1.34924ap-3f, 0x1.36db6ep-3f, 0x1.392492p-3f, 0x1.3b6db6p-3f, 0x1.3db6dcp-3f,
    0x1.4p-3f, 0x1.424924p-3f, 0x1.44924ap-3f, 0x1.46db6ep-3f, 0x1.492492p-3f, 0x1.4b6db6p-3f,
    0x1.4db6dcp-3f, 0x1.5p-3f, 0x1.524924p-3f, 0x1.54924ap-3f, 0x1.56db6ep-3f, 0x1.592492p-3f,
    0x1.5b6db6p-3f, 0x1.5db6dcp-3f, 0x1.6p-3f, 0x1.624924p-3f, 0x1.64924ap-3f, 0x1.66db6ep-3f,
    0x1.692492p-3f, 0x1.6b6db6p-3f, 0x1.6db6dcp-3f, 0x1.7p-3f, 0x1.724924p-3f, 0x1.74924ap-3f,
    0x1.76db6ep-3f, 0x1.792492p-3f, 0x1.7b6db6p-3f, 0x1.7db6dcp-3f, 0x1.8p-3f, 0x1.824924p-3f,
    0x1.84924ap-3f, 0x1.86db6ep-3f, 0x1.892492p-3f, 0x1.8b6db6p-3f, 0x1.8db6dcp-3f, 0x1.9p-3f,
    0x1.924924p-3f, 0x1.94924ap-3f, 0x1.96db6ep-3f, 0x1.992492p-3f, 0x1.9b6db6p-3f, 0x1.9db6dcp-3f,
    0x1.ap-3f, 0x1.a24924p-3f, 0x1.a4924ap-3f, 0x1.a6db6ep-3f, 0x1.a92492p-3f, 0x1.ab6db6p-3f,
    0x1.adb6dcp-3f, 0x1.bp-3f, 0x1.b24924p-3f, 0x1.b4924ap-3f, 0x1.b6db6ep-3f, 0x1.b92492p-3f,
    0x1.bb6db6p-3f, 0x1.bdb6dcp-3f, 0x1.cp-3f, 0x1.c24924p-3f, 0x1.c4924ap-3f, 0x1.c6db6ep-3f,
    0x1.c92492p-3f, 0x1.cb6db6p-3f, 0x1.cdb6dcp-3f, 0x1.dp-3f, 0x1.d24924p-3f, 0x1.d4924ap-3f,
    0x1.d6db6ep-3f, 0x1.d92492p-3f, 0x1.db6db6p-3f, 0x1.ddb6dcp-3f, 0x1.ep-3f, 0x1.e24924p-3f,
    0x1.e4924ap-3f, 0x1.e6db6ep-3f, 0x1.e92492p-3f, 0x1.eb6db6p-3f, 0x1.edb6dcp-3f, 0x1.fp-3f,
    0x1.f24924p-3f, 0x1.f4924ap-3f, 0x1.f6db6ep-3f, 0x1.f92492p-3f, 0x1.fb6db6p-3f, 0x1.fdb6dcp-3f,
    0x1p-2f, 0x1.012492p-2f, 0x1.024924p-2f, 0x1.036db6p-2f, 0x1.04924ap-2f, 0x1.05b6dcp-2f,
    0x1.06db6ep-2f, 0x1.08p-2f, 0x1.092492p-2f, 0x1.0a4924p-2f, 0x1.0b6db6p-2f, 0x1.0c924ap-2f,
    0x1.0db6dcp-2f, 0x1.0edb6ep-2f, 0x1.1p-2f, 0x1.112492p-2f, 0x1.124924p-2f, 0x1.136db6p-2f,
    0x1.14924ap-2f, 0x1.15b6dcp-2f, 0x1.16db6ep-2f, 0x1.18p-2f, 0x1.192492p-2f, 0x1.1a4924p-2f,
    0x1.1b6db6p-2f, 0x1.1c924ap-2f, 0x1.1db6dcp-2f, 0x1.1edb6ep-2f, 0x1.2p-2f, 0x1.212492p-2f,
    0x1.224924p-2f, 0x1.236db6p-2f,
};
__constant__ float kRecipMant[128] = {
    0x1.bffffep+2f, 0x1.bc86f2p+2f, 0x1.b91b92p+2f, 0x1.b5bd9p+2f, 0x1.b26c9ap+2f, 0x1.af286cp+2f,
    0x1.abf0b8p+2f, 0x1.a8c536p+2f, 0x1.a5a5a6p+2f, 0x1.a291cp+2f, 0x1.9f8948p+2f, 0x1.9c8bf8p+2f,
    0x1.99999ap+2f, 0x1.96b1eep+2f, 0x1.93d4bap+2f, 0x1.9101cap+2f, 0x1.8e38e4p+2f, 0x1.8b79d4p+2f,
    0x1.88c462p+2f, 0x1.861862p+2f, 0x1.8375ap+2f, 0x1.80dbeap+2f, 0x1.7e4b18p+2f, 0x1.7bc2f8p+2f,
    0x1.79436p+2f, 0x1.76cc2p+2f, 0x1.745d18p+2f, 0x1.71f618p+2f, 0x1.6f96f8p+2f, 0x1.6d3f98p+2f,
    0x1.6aefccp+2f, 0x1.68a774p+2f, 0x1.666666p+2f, 0x1.642c86p+2f, 0x1.61f9aep+2f, 0x1.5fcdbep+2f,
    0x1.5da896p+2f, 0x1.5b8a16p+2f, 0x1.59722p+2f, 0x1.576092p+2f, 0x1.555556p+2f, 0x1.53504ap+2f,
    0x1.51515p+2f, 0x1.4f5854p+2f, 0x1.4d6536p+2f, 0x1.4b77dep+2f, 0x1.49902ep+2f, 0x1.47ae14p+2f,
    0x1.45d174p+2f, 0x1.43fa36p+2f, 0x1.422844p+2f, 0x1.405b88p+2f, 0x1.3e93eap+2f, 0x1.3cd154p+2f,
    0x1.3b13b2p+2f, 0x1.395aeep+2f, 0x1.37a6f4p+2f, 0x1.35f7b2p+2f, 0x1.344d14p+2f, 0x1.32a704p+2f,
    0x1.310572p+2f, 0x1.2f684cp+2f, 0x1.2dcf8p+2f, 0x1.2c3af8p+2f, 0x1.2aaaaap+2f, 0x1.291e82p+2f,
    0x1.27967p+2f, 0x1.26126p+2f, 0x1.24924ap+2f, 0x1.231618p+2f, 0x1.219dbcp+2f, 0x1.20292ap+2f,
    0x1.1eb852p+2f, 0x1.1d4b26p+2f, 0x1.1be196p+2f, 0x1.1a7b96p+2f, 0x1.19191ap+2f, 0x1.17ba1p+2f,
    0x1.165e72p+2f, 0x1.15063p+2f, 0x1.13b13cp+2f, 0x1.125f8ap+2f, 0x1.111112p+2f, 0x1.0fc5c4p+2f,
    0x1.0e7d96p+2f, 0x1.0d387cp+2f, 0x1.0bf66ep+2f, 0x1.0ab75ep+2f, 0x1.097b42p+2f, 0x1.08421p+2f,
    0x1.070bbep+2f, 0x1.05d842p+2f, 0x1.04a79p+2f, 0x1.0379a2p+2f, 0x1.024e6ap+2f, 0x1.0125e2p+2f,
    0x1p+2f, 0x1.fdb976p+1f, 0x1.fb7814p+1f, 0x1.f93bc8p+1f, 0x1.f7047cp+1f, 0x1.f4d22ap+1f,
    0x1.f2a4bap+1f, 0x1.f07c2p+1f, 0x1.ee5848p+1f, 0x1.ec3924p+1f, 0x1.ea1ea4p+1f, 0x1.e808b6p+1f,
    0x1.e5f752p+1f, 0x1.e3ea66p+1f, 0x1.e1e1e2p+1f, 0x1.dfddbap+1f, 0x1.dddddep+1f, 0x1.dbe244p+1f,
    0x1.d9ead6p+1f, 0x1.d7f792p+1f, 0x1.d60864p+1f, 0x1.d41d42p+1f, 0x1.d2361ep+1f, 0x1.d052ecp+1f,
    0x1.ce739ep+1f, 0x1.cc9828p+1f, 0x1.cac082p+1f, 0x1.c8ec9ep+1f, 0x1.c71c72p+1f, 0x1.c54ffp+1f,
    0x1.c3870ep+1f, 0x1.c1c1c4p+1f,
};

// group_scale for an arbitrary fp32 amax, with amax/448 formed as quot does (y =
// fl32(1/448), q = fl32(amax y), q + (amax - q 448) y): the correctly rounded quotient
// (Markstein's theorem) for amax >= 2^-60; below that, and for amax = 0, group_scale.
__device__ __forceinline__ GroupScale group_scale_fma(float amax) {
  if (amax < 0x1p-60f) {
    GroupScale g = group_scale(amax);
    g.small = g.small && amax != 0.0f;  // 0 / 1 is exact on the fast path
    return g;
  }
  constexpr float kY = 1.0f / 448.0f;  // fl32(1/448), rounded once by the compiler
  const float q = __fmul_rn(amax, kY);
  const float e = __fmaf_rn(-q, 448.0f, amax);
  GroupScale g;
  g.s = __fmaf_rn(e, kY, q);
  g.rs = __frcp_rn(g.s);
  g.ns = -g.s;
  g.small = g.s < kSmallScale;
  return g;
}

// Same result as group_scale for every amax that is a BF16 value (the maximum of BF16
// values is one). amax = 0 gives s = 1 directly (its codes are those of 0 / 1 = 0 on
// the fast path too, so an all-zero group, or a lane with no group, does not send its
// warp down the division path); 0 < amax < 2^-71 (s below about 2^-80) and non-finite
// amax (outside the contract) take the division path; the branch is taken per warp,
// only when one of its lanes needs it.
__device__ __forceinline__ GroupScale group_scale_bf16(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ebias = static_cast<int>(b >> 23);  // biased exponent (amax >= 0)
  const bool tiny = (ebias < 127 - 71 && b != 0) || ebias == 255;
  const int e = ebias - 127;
  const uint32_t i = (b >> 16) & 0x7Fu;
  GroupScale g;
  g.s = __uint_as_float(__float_as_uint(kScaleMant[i]) + static_cast<uint32_t>((e - 6) << 23));
  g.rs = __uint_as_float(__float_as_uint(kRecipMant[i]) + static_cast<uint32_t>((6 - e) << 23));
  if (b == 0) g.s = g.rs = 1.0f;  // an all-zero group: s = 1, and 0 / 1 is exact either way
  g.small = false;
  if (__any_sync(kFull, tiny)) {
    if (tiny) {
      g = group_scale(amax);
      g.small = true;
    }
  }
  g.ns = -g.s;
  return g;
}

// group_scale_bf16 with its tables in shared memory (tab[0..127] the scale mantissas,
// tab[128..255] their reciprocals); same result.
__device__ __forceinline__ GroupScale group_scale_bf16_sm(float amax, const float* tab) {
  const uint32_t b = __float_as_uint(amax);
  const int ebias = static_cast<int>(b >> 23);
  const bool tiny = (ebias < 127 - 71 && b != 0) || ebias == 255;
  const int e = ebias - 127;
  const uint32_t i = (b >> 16) & 0x7Fu;
  GroupScale g;
  g.s = __uint_as_float(__float_as_uint(tab[i]) + static_cast<uint32_t>((e - 6) << 23));
  g.rs = __uint_as_float(__float_as_uint(tab[128 + i]) + static_cast<uint32_t>((6 - e) << 23));
  if (b == 0) g.s = g.rs = 1.0f;  // an all-zero group (see group_scale_bf16)
  g.small = false;
  if (__any_sync(kFull, tiny)) {
    if (tiny) {
      g = group_scale(amax);
      g.small = true;
    }
  }
  g.ns = -g.s;
  return g;
}

// Copies the two scale tables into shared memory (256 floats), for group_scale_bf16_sm.
__device__ __forceinline__ void scale_tables_fill(float* tab) {
  for (int i = threadIdx.x; i < 128; i += blockDim.x) {
    tab[i] = kScaleMant[i];
    tab[128 + i] = kRecipMant[i];
  }
}

// x/s for a BF16-valued x (see the file header for why this has the IEEE quotient's
// code): q = x*r, then q - (q*s - x)*r. Written this way the sign of x = -0 survives
// without a separate copy-sign (q*s - x is +0 and q - (+0)*r is -0 + -0).
__device__ __forceinline__ float quot(float x, const GroupScale& g) {
  const float q = __fmul_rn(x, g.rs);
  const float en = __fmaf_rn(q, g.s, -x);
  return __fmaf_rn(en, -g.rs, q);
}

// quot on two values (of groups g0 and g1) with packed fp32 pair instructions: each
// lane of a pair is the same IEEE operation as in quot, so the results are quot's bit
// for bit.
__device__ __forceinline__ void quot2(float x0, float x1, const GroupScale& g0,
                                      const GroupScale& g1, float& t0, float& t1) {
  float q0, q1;
  mul2(q0, q1, x0, x1, g0.rs, g1.rs);
  float e0 = -x0, e1 = -x1;
  fma2(e0, e1, q0, q1, g0.s, g1.s);      // q*s - x
  fma2(q0, q1, e0, e1, -g0.rs, -g1.rs);  // q - (q*s - x)*r
  t0 = q0;
  t1 = q1;
}

// Eight codes of BF16-valued x (packed little-endian into two words). Groups with a
// tiny scale divide; the branch is per warp and only taken when a lane needs it.
__device__ __forceinline__ uint2 codes8(const float (&v)[8], const GroupScale& g) {
  float t[8];
  if (__any_sync(kFull, g.small)) {
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = g.small ? __fdiv_rn(v[i], g.s) : quot(v[i], g);
  } else {
#pragma unroll
    for (int i = 0; i < 8; i += 2) quot2(v[i], v[i + 1], g, g, t[i], t[i + 1]);
  }
  return make_uint2(cvt_e4m3x4(t[0], t[1], t[2], t[3]), cvt_e4m3x4(t[4], t[5], t[6], t[7]));
}

// Lane-wise max of the magnitudes of two packed BF16 pairs (finite inputs).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a & 0x7FFF7FFFu), "r"(b & 0x7FFF7FFFu));
  return r;
}

// Largest magnitude of eight values (balanced tree).
__device__ __forceinline__ float absmax8(const float (&v)[8]) {
  const float a = fmaxf(fabsf(v[0]), fabsf(v[1])), b = fmaxf(fabsf(v[2]), fabsf(v[3]));
  const float c = fmaxf(fabsf(v[4]), fabsf(v[5])), d = fmaxf(fabsf(v[6]), fabsf(v[7]));
  return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

// One 1x128 group of BF16 values held by a half-warp: 16 lanes x 8 values. Returns the
// group scale; writes the 8 codes of this lane. All 32 lanes must call it.
__device__ __forceinline__ float quant_half_warp(const float (&v)[8], uint2& codes) {
  float a = absmax8(v);
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, off));
  const GroupScale g = group_scale_bf16(a);
  codes = codes8(v, g);
  return g.s;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& r, float (&v)[8]) {
  v[0] = bf16_lo(r.x); v[1] = bf16_hi(r.x);
  v[2] = bf16_lo(r.y); v[3] = bf16_hi(r.y);
  v[4] = bf16_lo(r.z); v[5] = bf16_hi(r.z);
  v[6] = bf16_lo(r.w); v[7] = bf16_hi(r.w);
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------
// The method's fixed fp32 exponential: Cody-Waite range reduction (Cody & Waite,
// "Software Manual for the Elementary Functions", 1980) with ln2 split into a
// 12-significant-bit head and an fp32 tail, then the degree-7 Taylor polynomial of
// e^r in Horner form with fused multiply-adds, scaled by 2^n. The argument is
// clamped to [-80, 88], where 2^n stays a normal number; below -80, 1 + e^x is 1 in
// fp32 anyway. Every step is an IEEE-rounded operation, so the result is a fixed
// function of x. Two arguments at a time (packed fp32 pairs).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void exp_cw2(float x0, float x1, float& e0, float& e1) {
  const float kLog2e = 0x1.715476p+0f;
  const float kLn2Hi = 0x1.62ep-1f;
  const float kLn2Lo = 0x1.0bfbe8p-15f;
  // Adding 1.5 * 2^23 to |v| < 2^22 leaves a float whose unit in the last place is 1, so
  // the addition itself rounds v to the nearest integer, ties to even (= rint(v)), and
  // that integer sits in the low mantissa bits: n = bits(t) - bits(1.5 * 2^23). This
  // keeps the rounding and the 2^n exponent on the FMA/ALU pipes.
  const float kShift = 0x1.8p+23f;
  x0 = fminf(fmaxf(x0, -80.0f), 88.0f);
  x1 = fminf(fmaxf(x1, -80.0f), 88.0f);
  float l0, l1;
  mul2(l0, l1, x0, x1, kLog2e, kLog2e);
  const float t0 = __fadd_rn(l0, kShift), t1 = __fadd_rn(l1, kShift);
  const float n0 = __fsub_rn(t0, kShift), n1 = __fsub_rn(t1, kShift);  // rint(l), exact
  float r0 = x0, r1 = x1;
  fma2(r0, r1, -n0, -n1, kLn2Hi, kLn2Hi);
  fma2(r0, r1, -n0, -n1, kLn2Lo, kLn2Lo);
  // Horner: p = ((((((c7 r + c6) r + c5) r + c4) r + c3) r + c2) r + 1) r + 1
  float p0 = 0x1.6c16c2p-10f, p1 = 0x1.6c16c2p-10f;  // starts as c6, then c7*r + c6
  fma2(p0, p1, r0, r1, 0x1.a01a02p-13f, 0x1.a01a02p-13f);
  float c0 = 0x1.111112p-7f, c1 = 0x1.111112p-7f;
  fma2(c0, c1, p0, p1, r0, r1);
  p0 = c0; p1 = c1;
  c0 = 0x1.555556p-5f; c1 = 0x1.555556p-5f;
  fma2(c0, c1, p0, p1, r0, r1);
  p0 = c0; p1 = c1;
  c0 = 0x1.555556p-3f; c1 = 0x1.555556p-3f;
  fma2(c0, c1, p0, p1, r0, r1);
  p0 = c0; p1 = c1;
  c0 = 0.5f; c1 = 0.5f;
  fma2(c0, c1, p0, p1, r0, r1);
  p0 = c0; p1 = c1;
  c0 = 1.0f; c1 = 1.0f;
  fma2(c0, c1, p0, p1, r0, r1);
  p0 = c0; p1 = c1;
  c0 = 1.0f; c1 = 1.0f;
  fma2(c0, c1, p0, p1, r0, r1);
  const int k0 = __float_as_int(t0) - __float_as_int(kShift);
  const int k1 = __float_as_int(t1) - __float_as_int(kShift);
  const float s0 = __int_as_float((k0 + 127) << 23);
  const float s1 = __int_as_float((k1 + 127) << 23);
  mul2(e0, e1, c0, c1, s0, s1);
}

// ---------------------------------------------------------------------------
// Row-group quantizer of SwiGLU (a4), fed by tensor copies. A unit is a box of kRgRows
// rows x one 128-column group of the gate and the same of the up half (2 x 32 KB of
// BF16). A persistent CTA has one producer warp that keeps up to kStages units in flight
// through a ring in shared memory, and kConsumers consumer warps, each quantizing eight
// rows of the box (four lanes per row, 32 values a lane: the row maximum takes two
// shuffles and the scale is formed once per 32 values; a half-warp per row measured 3 %
// slower). The gate factor comes from a per-CTA table (see sg_index). A box past a
// ragged M or K arrives zero-filled (zeros raise no group maximum) and only its valid
// rows and columns are stored.
// ---------------------------------------------------------------------------
#ifndef A4_STAGES
#define A4_STAGES 2
#define A4_CONS 16
#endif
constexpr int kRgRows = 8 * A4_CONS;  // eight rows per consumer warp
constexpr uint32_t kRgBoxBytes = kRgRows * 128 * 2;
template <int kConsumers>
constexpr int rg_threads() { return 32 * (kConsumers + 1); }


// The gate factor sg(g) = fl32(g / fl32(1 + E(-g))) of SwiGLU depends on the BF16 gate
// alone, so each CTA tabulates it, with the same device arithmetic, for every BF16 g with
// 2^-24 <= |g| < 2^7 (biased exponents 103 .. 133, both signs: 7936 values, 31 KB of
// shared memory); a chunk with a gate outside that range computes sg directly.
constexpr uint32_t kSgLoExp = 127 - 24;
constexpr uint32_t kSgExps = 31;
constexpr uint32_t kSgHalf = kSgExps * 128;  // entries per sign
constexpr uint32_t kSgEntries = 2 * kSgHalf;

// Table index of the BF16 gate with bit pattern gb, or kSgEntries when outside the table.
__device__ __forceinline__ uint32_t sg_index(uint32_t gb) {
  const uint32_t rel = (gb & 0x7FFFu) - (kSgLoExp << 7);  // wraps below the range
  return rel < kSgHalf ? rel + (gb >> 15) * kSgHalf : kSgEntries;
}

// sg(g) = fl32(g / fl32(1 + E(-g))) of two gates; h = bf16(fl32(sg(g) u)) then follows.
__device__ __forceinline__ void sg2(float g0, float g1, float& s0, float& s1) {
  float e0, e1;
  exp_cw2(-g0, -g1, e0, e1);
  s0 = __fdiv_rn(g0, __fadd_rn(1.0f, e0));
  s1 = __fdiv_rn(g1, __fadd_rn(1.0f, e1));
}

__device__ __forceinline__ void sg_table_fill(float* tab) {
  for (uint32_t i = threadIdx.x; i < kSgEntries / 2; i += blockDim.x) {
    const uint32_t e0 = 2 * i, e1 = 2 * i + 1;  // entries with the same sign
    const uint32_t sign = e0 / kSgHalf;
    const float g0 = __uint_as_float(((sign << 15) | ((e0 - sign * kSgHalf) + (kSgLoExp << 7))) << 16);
    const float g1 = __uint_as_float(((sign << 15) | ((e1 - sign * kSgHalf) + (kSgLoExp << 7))) << 16);
    sg2(g0, g1, tab[e0], tab[e1]);
  }
}

struct SwigluBoxes {  // a4: h = SwiGLU(gate, up) from the gate box and the up box
  static constexpr int kBoxes = 2;
  __device__ __forceinline__ static void values(const uint16_t* b0, const uint16_t* b1, int off,
                                                const float* tab, float (&v)[8]) {
    const uint4 gw = *reinterpret_cast<const uint4*>(b0 + off);
    float g[8], u[8], sg[8];
    unpack_bf16x8(gw, g);
    unpack_bf16x8(*reinterpret_cast<const uint4*>(b1 + off), u);
    const uint32_t w[4] = {gw.x, gw.y, gw.z, gw.w};
    uint32_t idx[8];
    bool in = true;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      idx[2 * i] = sg_index(w[i] & 0xFFFFu);
      idx[2 * i + 1] = sg_index(w[i] >> 16);
      in = in && idx[2 * i] < kSgEntries && idx[2 * i + 1] < kSgEntries;
    }
    if (__all_sync(kFull, in)) {
#pragma unroll
      for (int i = 0; i < 8; ++i) sg[i] = tab[idx[i]];
    } else {
#pragma unroll
      for (int i = 0; i < 8; i += 2) sg2(g[i], g[i + 1], sg[i], sg[i + 1]);
    }
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      float m0, m1;
      mul2(m0, m1, sg[i], sg[i + 1], u[i], u[i + 1]);
      v[i] = round_bf16(m0);
      v[i + 1] = round_bf16(m1);
    }
  }
};

// (defined with the lane-per-group quantizers below)
__device__ __forceinline__ uint32_t bf16x2_maxabs_xs(uint32_t a, uint32_t b);
__device__ __forceinline__ float bf16x2_hmax_abs(uint32_t m);
template <bool kSmall>
__device__ __forceinline__ uint2 codes8_words(const uint4& w, const GroupScale& g);

template <class B, int kStages>
constexpr size_t rowgroup_tma_smem() {
  return 1024 + static_cast<size_t>(kStages) * B::kBoxes * kRgBoxBytes + 2 * kStages * 8 + 16 +
         kSgEntries * 4 + 256 * 4;
}

// M rows, G = ceil(K / 128) groups of K valid columns; codes q[m * ldq + k], scales
// s[g * lds + m]. tm0 (and tm1) map the [M][K] source(s) with 128 x kRgRows boxes.
template <class B, int kStages, int kConsumers>
__global__ void __launch_bounds__(rg_threads<kConsumers>()) rowgroup_tma_kernel(
    const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1, int64_t M,
    int64_t G, int64_t K, uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ s,
    int64_t lds, unsigned* err, uint64_t limit_ns) {
  static_assert(kStages <= 32, "stage flags are one word");
  constexpr uint32_t kStageBytes = B::kBoxes * kRgBoxBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  int* abort_flag = reinterpret_cast<int*>(empty + kStages);
  float* tab = reinterpret_cast<float*>(empty + kStages + 2);
  const WaitCtl ctl{abort_flag, err, limit_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(full + st, 1);
      mbar_init(empty + st, kConsumers);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  float* stab = tab + kSgEntries;  // scale and reciprocal tables
  sg_table_fill(tab);
  scale_tables_fill(stab);
  __syncthreads();
  // unit u = (row box) * G + group; the host keeps the unit count below 2^31
  const uint32_t units = static_cast<uint32_t>(((M + kRgRows - 1) / kRgRows) * G);
  const uint32_t G32 = static_cast<uint32_t>(G);
  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0, par = 0;  // bit st: stage st has a copy issued / its parity
      bool ok = true;
      int i = 0;
      for (uint32_t t = blockIdx.x; t < units; t += gridDim.x, ++i) {
        const int st = i % kStages;
        const uint32_t ph = static_cast<uint32_t>(i / kStages) & 1u;
        if (i >= kStages && !mbar_wait(empty + st, ph ^ 1u, ctl)) { ok = false; break; }
        const uint32_t tb = t / G32;
        const int32_t x0 = static_cast<int32_t>((t - tb * G32) * 128);
        const int32_t y0 = static_cast<int32_t>(tb * kRgRows);
        mbar_arrive_expect_tx(full + st, kStageBytes);
        tma_load_2d(base + st * kStageBytes, &tm0, x0, y0, full + st);
        if (B::kBoxes == 2) tma_load_2d(base + st * kStageBytes + kRgBoxBytes, &tm1, x0, y0, full + st);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        for (int st = 0; st < kStages; ++st) {
          if (!((issued >> st) & 1u)) continue;
          const uint32_t a = smem_u32(full + st);
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(a, (par >> st) & 1u))
            if (global_timer_ns() - t0 > limit_ns) break;
        }
      }
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  // lane l of consumer warp w: row 8w + l / 4 of the unit, the four 8-column chunks
  // (l % 4) + 4k rotated by the row (no two lanes of a shared-memory phase in one bank)
  static_assert(kRgRows == 8 * kConsumers, "eight rows per consumer warp");
  const int lr = lane >> 2, a = lane & 3;
  const int r = warp * 8 + lr;
  int i = 0;
  for (uint32_t t = blockIdx.x; t < units; t += gridDim.x, ++i) {
    const int st = i % kStages;
    if (!mbar_wait_warp(full + st, static_cast<uint32_t>(i / kStages) & 1u, ctl)) break;
    const uint16_t* b0 = reinterpret_cast<const uint16_t*>(base + st * kStageBytes) + r * 128;
    const uint16_t* b1 = b0 + kRgRows * 128;
    const uint32_t tb = t / G32;
    const int64_t g = t - tb * G32;
    const int64_t m = static_cast<int64_t>(tb) * kRgRows + r;
    uint4 h[4];
    uint32_t mh[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float v[8];
      B::values(b0, b1, ((a + 4 * k + 4 * (lr & 3)) & 15) * 8, tab, v);
      h[k] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                        pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
      mh[0] = bf16x2_maxabs_xs(mh[0], h[k].x);
      mh[1] = bf16x2_maxabs_xs(mh[1], h[k].y);
      mh[2] = bf16x2_maxabs_xs(mh[2], h[k].z);
      mh[3] = bf16x2_maxabs_xs(mh[3], h[k].w);
    }
    __syncwarp();  // every lane's reads of the stage are complete (their values are used)
    if (lane == 0) mbar_arrive(empty + st);  // this warp is done with the stage
    // the row's four lanes are adjacent: two shuffles give its maximum
    uint32_t hm = bf16x2_maxabs_xs(bf16x2_maxabs_xs(mh[0], mh[1]), bf16x2_maxabs_xs(mh[2], mh[3]));
    hm = bf16x2_maxabs_xs(hm, __shfl_xor_sync(kFull, hm, 1));
    hm = bf16x2_maxabs_xs(hm, __shfl_xor_sync(kFull, hm, 2));
    const GroupScale gs = group_scale_bf16_sm(bf16x2_hmax_abs(hm), stab);
    const bool small = __any_sync(kFull, gs.small);
    if (m < M) {
      uint8_t* qr = q + m * ldq + g * 128;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = ((a + 4 * k + 4 * (lr & 3)) & 15) * 8;
        if (g * 128 + c < K)  // K is a multiple of 16: a chunk is in or out
          *reinterpret_cast<uint2*>(qr + c) =
              small ? codes8_words<true>(h[k], gs) : codes8_words<false>(h[k], gs);
      }
      if (a == 0) s[g * lds + m] = gs.s;
    }
  }
}

// ---------------------------------------------------------------------------
// Lane-per-group row quantizer (a1). A unit is kLgRows = 32 rows x one 128-column group;
// each lane of a consumer warp owns one row of it, i.e. one whole 1x128 group, so the
// group maximum needs no shuffles and the scale is formed once per 128 values. A
// producer warp streams units through tensor-copy stages; consumer warp w takes units w,
// w + kConsumers, ... and owns kPer stages of its own (its units rotate through them), so
// that a warp only ever waits on a stage whose previous phase it consumed itself (an
// mbarrier parity wait cannot tell phase k from phase k - 2). The codes go through a per-warp staging box in
// shared memory and leave by a tensor store (which also clips a ragged M or K); the
// scales (one per lane) are one coalesced 128-byte store per unit.
// Rows of a staged unit are 256 bytes apart, so lane r reads its 16-byte chunks in the
// rotated order c = (j + r) mod 16: the 32 lanes of one load then cover 16 distinct chunk
// positions (8 bank groups), 4 wavefronts for 512 bytes, the least possible. Codes are
// staged in the same rotated order (8-byte pieces, 2 wavefronts per 256 bytes).
// ---------------------------------------------------------------------------
#ifndef LG1_PER
#define LG1_PER 2
#define LG1_CONS 10
#endif
constexpr int kLgRows = 32;
constexpr uint32_t kLgBoxBytes = kLgRows * 128 * 2;  // one BF16 box
constexpr uint32_t kLgOutBytes = kLgRows * 128;      // its codes
template <int kConsumers>
constexpr int lg_threads() { return 32 * (kConsumers + 1); }

template <class B, int kPer, int kConsumers>
constexpr size_t lanegroup_smem() {
  return 1024 + static_cast<size_t>(kPer * kConsumers) * B::kBoxes * kLgBoxBytes +
         static_cast<size_t>(kConsumers) * kLgOutBytes + 2 * kPer * kConsumers * 8 + 16;
}

// Lane-wise max(|a|, |b|) of two packed BF16 pairs; the sign bits of the result are the
// XOR of the operands' (max.xorsign.abs), so only the magnitudes are meaningful.
__device__ __forceinline__ uint32_t bf16x2_maxabs_xs(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Magnitude of the larger half of a packed pair from bf16x2_maxabs_xs.
__device__ __forceinline__ float bf16x2_hmax_abs(uint32_t m) {
  return fmaxf(fabsf(bf16_lo(m)), fabsf(bf16_hi(m)));
}

// Codes of 8 BF16 values (four packed words) of one group; kSmall: some lane of the warp
// has a tiny scale (the division path).
template <bool kSmall>
__device__ __forceinline__ uint2 codes8_words(const uint4& w, const GroupScale& g) {
  float v[8];
  unpack_bf16x8(w, v);
  float t[8];
  if (kSmall) {
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = g.small ? __fdiv_rn(v[i], g.s) : quot(v[i], g);
  } else {
#pragma unroll
    for (int i = 0; i < 8; i += 2) quot2(v[i], v[i + 1], g, g, t[i], t[i + 1]);
  }
  return make_uint2(cvt_e4m3x4(t[0], t[1], t[2], t[3]), cvt_e4m3x4(t[4], t[5], t[6], t[7]));
}

struct ActLane {  // a1: the staged values themselves
  static constexpr int kBoxes = 1;
  __device__ __forceinline__ static uint4 chunk(const uint16_t* b0, const uint16_t*, int off) {
    return *reinterpret_cast<const uint4*>(b0 + off);
  }
};


// M rows, G = ceil(K / 128) groups of K valid columns. tm0 (and tm1) map the [M][K]
// source(s) with 128 x kLgRows boxes; tmQ maps the [M][K] codes (same box); scales go to
// s[g * lds + m]. The host keeps the unit count below 2^31.
template <class B, int kPer, int kConsumers>
__global__ void __launch_bounds__(lg_threads<kConsumers>(), 1) lanegroup_kernel(
    const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
    const __grid_constant__ CUtensorMap tmQ, int64_t M, int64_t G, float* __restrict__ s,
    int64_t lds, unsigned* err, uint64_t limit_ns) {
  constexpr int kStages = kPer * kConsumers;
  static_assert(kStages <= 32, "stage flags are one word");
  constexpr uint32_t kStageBytes = B::kBoxes * kLgBoxBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* outs = base + kStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(outs + kConsumers * kLgOutBytes);
  uint64_t* empty = full + kStages;
  int* abort_flag = reinterpret_cast<int*>(empty + kStages);
  const WaitCtl ctl{abort_flag, err, limit_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(full + st, 1);
      mbar_init(empty + st, 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const uint32_t units = static_cast<uint32_t>(((M + kLgRows - 1) / kLgRows) * G);
  const uint32_t G32 = static_cast<uint32_t>(G);
  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0, par = 0;  // bit st: stage st has a copy issued / its parity
      bool ok = true;
      int i = 0;
      for (uint32_t t = blockIdx.x; t < units; t += gridDim.x, ++i) {
        const int li = i / kConsumers;  // the unit's index among its warp's units
        const int st = (i % kConsumers) * kPer + li % kPer;
        const uint32_t ph = static_cast<uint32_t>(li / kPer) & 1u;
        if (li >= kPer && !mbar_wait(empty + st, ph ^ 1u, ctl)) { ok = false; break; }
        const uint32_t tb = t / G32;
        const int32_t x0 = static_cast<int32_t>((t - tb * G32) * 128);
        const int32_t y0 = static_cast<int32_t>(tb * kLgRows);
        mbar_arrive_expect_tx(full + st, kStageBytes);
        tma_load_2d(base + st * kStageBytes, &tm0, x0, y0, full + st);
        if (B::kBoxes == 2) tma_load_2d(base + st * kStageBytes + kLgBoxBytes, &tm1, x0, y0, full + st);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        for (int st = 0; st < kStages; ++st) {
          if (!((issued >> st) & 1u)) continue;
          const uint32_t a = smem_u32(full + st);
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(a, (par >> st) & 1u))
            if (global_timer_ns() - t0 > limit_ns) break;
        }
      }
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  uint8_t* out = outs + warp * kLgOutBytes;
  bool stored = false;
  int li = 0;
  for (uint32_t t = blockIdx.x + warp * gridDim.x; t < units; t += kConsumers * gridDim.x, ++li) {
    const int st = warp * kPer + li % kPer;
    if (!mbar_wait_warp(full + st, static_cast<uint32_t>(li / kPer) & 1u, ctl)) break;
    const uint16_t* row0 = reinterpret_cast<const uint16_t*>(base + st * kStageBytes) + lane * 128;
    const uint16_t* row1 = row0 + kLgRows * 128;
    uint4 w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = B::chunk(row0, row1, ((j + lane) & 15) * 8);
    uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      m[0] = bf16x2_maxabs_xs(m[0], w[j].x);
      m[1] = bf16x2_maxabs_xs(m[1], w[j].y);
      m[2] = bf16x2_maxabs_xs(m[2], w[j].z);
      m[3] = bf16x2_maxabs_xs(m[3], w[j].w);
    }
    const float amax =
        bf16x2_hmax_abs(bf16x2_maxabs_xs(bf16x2_maxabs_xs(m[0], m[1]), bf16x2_maxabs_xs(m[2], m[3])));
    __syncwarp();  // every lane's reads of the stage are complete (their values are used)
    if (lane == 0) mbar_arrive(empty + st);
    const GroupScale g = group_scale_bf16(amax);
    const uint32_t tb = t / G32;
    const int32_t x0 = static_cast<int32_t>((t - tb * G32) * 128);
    const int32_t y0 = static_cast<int32_t>(tb * kLgRows);
    if (stored) {  // the previous unit's store must have read the staging box
      if (lane == 0) tma_store_wait_read();
      __syncwarp();
    }
    uint8_t* orow = out + lane * 128;
    if (__any_sync(kFull, g.small)) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        *reinterpret_cast<uint2*>(orow + ((j + lane) & 15) * 8) = codes8_words<true>(w[j], g);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        *reinterpret_cast<uint2*>(orow + ((j + lane) & 15) * 8) = codes8_words<false>(w[j], g);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&tmQ, out, x0, y0);
      tma_store_commit();
    }
    stored = true;
    const int64_t mrow = static_cast<int64_t>(y0) + lane;
    if (mrow < M) s[static_cast<int64_t>(x0 / 128) * lds + mrow] = g.s;
  }
  if (stored && lane == 0) tma_store_wait_all();
}

// ---------------------------------------------------------------------------
// a3: RMSNorm + 1x128 quantization.
// Batches of more than 1024 rows: one warp per row in two passes (the sum of squares,
// a warp reduction, then the row again from L2 to form and quantize y), 8 rows per CTA.
// Small batches: one CTA (256 threads) per row, the row held in registers.
// Thread t of the row owns 8-element chunks t, t+T, ... (T = threads per row), so
// that each half-warp covers one 128-group.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float rstd_from_ss(double ss, int64_t H, float eps) {
  const double ms = __ddiv_rn(ss, static_cast<double>(H));
  const double rr = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, static_cast<double>(eps))));
  return __double2float_rn(rr);
}

// Sum of squares of this thread's chunks c = first + stride*j (c < nch) in fp64. Each
// square of a BF16 value is exact in fp64; eight partial sums (one per position in the
// chunk) keep the dependent chains short. The order differs from a sequential sum only
// in the last bits of the fp64 result.
template <int kChunks>
__device__ __forceinline__ double sum_squares(const uint4 (&raw)[kChunks], int64_t first,
                                              int64_t stride, int64_t nch) {
  double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int j = 0; j < kChunks; ++j) {
    if (first + stride * j < nch) {
      float v[8];
      unpack_bf16x8(raw[j], v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const double d = static_cast<double>(v[i]);
        acc[i] = __fma_rn(d, d, acc[i]);
      }
    }
  }
  return __dadd_rn(__dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3])),
                   __dadd_rn(__dadd_rn(acc[4], acc[5]), __dadd_rn(acc[6], acc[7])));
}

// y = bf16(fl32(fl32(x r) g)) for one chunk (gamma staged in shared memory), then the
// half-warp group quantization.
__device__ __forceinline__ void norm_quant_chunk(const uint4& xr, const uint16_t* gamma, int64_t c,
                                                 bool act, float r, uint8_t* qrow, float* s,
                                                 int64_t lds, int64_t m, int lane) {
  float v[8];
  if (act) {
    float xv[8], gv[8];
    unpack_bf16x8(xr, xv);
    unpack_bf16x8(*reinterpret_cast<const uint4*>(gamma + c * 8), gv);  // shared memory
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      float a0, a1, b0, b1;
      mul2(a0, a1, xv[i], xv[i + 1], r, r);
      mul2(b0, b1, a0, a1, gv[i], gv[i + 1]);
      v[i] = round_bf16(b0);
      v[i + 1] = round_bf16(b1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.0f;
  }
  uint2 codes;
  const float sc = quant_half_warp(v, codes);
  if (act) {
    *reinterpret_cast<uint2*>(qrow + c * 8) = codes;
    if ((lane & 15) == 0) s[(c >> 4) * lds + m] = sc;
  }
}

// One warp per row in two passes: the fp64 sum of squares with four 16-byte loads in
// flight per lane (the partial sums and their order are those of sum_squares, so r is
// the same), then the row again (from L2: a warp's row is a few KB, read moments
// before) to form y and quantize it. Holding no whole row in registers keeps the
// kernel small enough for several CTAs per SM.
__global__ void __launch_bounds__(256) rmsnorm_quant_warp2_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ gamma, int64_t M, int64_t H,
    int64_t ldx, float eps, uint8_t* __restrict__ q, float* __restrict__ s, int64_t lds) {
  extern __shared__ uint4 gamma_sm[];  // H BF16 values, shared by every row
  const int lane = threadIdx.x & 31;
  const int64_t nch = H >> 3;
  for (int64_t i = threadIdx.x; i < nch; i += blockDim.x) gamma_sm[i] = ld_nc_v4(gamma + i * 8);
  __syncthreads();
  const int64_t wglobal = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t m = wglobal; m < M; m += nw) {
    const uint16_t* row = x + m * ldx;
    double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    for (int64_t c0 = 0; c0 < nch; c0 += 128) {
      uint4 raw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t c = c0 + lane + 32 * u;
        if (c < nch) raw[u] = ld_nc_v4(row + c * 8);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (c0 + lane + 32 * u < nch) {
          float v[8];
          unpack_bf16x8(raw[u], v);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const double d = static_cast<double>(v[i]);
            acc[i] = __fma_rn(d, d, acc[i]);
          }
        }
      }
    }
    double ss = __dadd_rn(__dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3])),
                          __dadd_rn(__dadd_rn(acc[4], acc[5]), __dadd_rn(acc[6], acc[7])));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(kFull, ss, off));
    const float r = rstd_from_ss(ss, H, eps);
    for (int64_t c0 = 0; c0 < nch; c0 += 128) {
      uint4 raw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t c = c0 + lane + 32 * u;
        if (c < nch) raw[u] = *reinterpret_cast<const uint4*>(row + c * 8);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (c0 + 32 * u >= nch) break;  // warp-uniform; lanes past nch hold zeros
        const int64_t c = c0 + lane + 32 * u;
        norm_quant_chunk(raw[u], reinterpret_cast<const uint16_t*>(gamma_sm), c, c < nch, r,
                         q + m * H, s, lds, m, lane);
      }
    }
  }
}

constexpr int kNormThreads = 256;
constexpr int kNormMaxChunks = 8;  // CTA-per-row path: H <= 8 * 8 * 256 = 16384

__global__ void __launch_bounds__(kNormThreads) rmsnorm_quant_cta_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ gamma, int64_t M, int64_t H,
    int64_t ldx, float eps, uint8_t* __restrict__ q, float* __restrict__ s, int64_t lds) {
  __shared__ double red[kNormThreads / 32];
  __shared__ float r_sh;
  extern __shared__ uint4 gamma_sm[];  // H BF16 values, shared by every row
  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;
  const int64_t nch = H >> 3;
  for (int64_t i = tid; i < nch; i += kNormThreads) gamma_sm[i] = ld_nc_v4(gamma + i * 8);
  __syncthreads();
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const uint16_t* row = x + m * ldx;
    uint4 raw[kNormMaxChunks];
#pragma unroll
    for (int j = 0; j < kNormMaxChunks; ++j) {
      const int64_t c = tid + j * kNormThreads;
      if (c < nch) raw[j] = ld_nc_v4(row + c * 8);
    }
    double ss = sum_squares<kNormMaxChunks>(raw, tid, kNormThreads, nch);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(kFull, ss, off));
    if (lane == 0) red[wid] = ss;
    __syncthreads();
    if (tid == 0) {
      double tot = 0.0;
      for (int w = 0; w < kNormThreads / 32; ++w) tot = __dadd_rn(tot, red[w]);
      r_sh = rstd_from_ss(tot, H, eps);
    }
    __syncthreads();
    const float r = r_sh;
#pragma unroll
    for (int j = 0; j < kNormMaxChunks; ++j) {
      const int64_t c0 = static_cast<int64_t>(j) * kNormThreads + (tid & ~31);
      if (c0 >= nch) break;  // warp-uniform; lanes past nch (a partial group) hold zeros
      const int64_t c = tid + j * kNormThreads;
      norm_quant_chunk(raw[j], reinterpret_cast<const uint16_t*>(gamma_sm), c, c < nch, r,
                       q + m * H, s, lds, m, lane);
    }
    __syncthreads();  // red / r_sh are reused by the next row
  }
}

// Lane-per-group RMSNorm + quantization (H a multiple of 128, at most 64 groups): a unit
// is one row, staged whole by one tensor copy (a [M][G][128] view); consumer warp w takes
// rows w, w + kConsumers, ... of the CTA's share. Lane l owns groups l, l + 32, ...: it
// adds its groups' squares in fp64 (eight partial sums, one per position in a chunk), a
// butterfly over the warp gives the row's sum, and from r each lane forms y = bf16(fl32(
// fl32(x r) g)) of its group as packed BF16 words, takes their maximum, and writes the
// codes into the warp's staging row, which leaves by a tensor store. Each consumer warp
// owns `per` row stages (set by the host from the shared-memory budget; stages are per
// warp for the reason given at lanegroup_kernel). Groups are 256 bytes apart
// in a staged row, so lanes read their chunks in the rotated order of lanegroup_kernel.
template <int kConsumers>
__global__ void __launch_bounds__(32 * (kConsumers + 1), 1) rmsnorm_lane_kernel(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
    const uint16_t* __restrict__ gamma, int64_t M, int G, int per, float eps,
    float* __restrict__ s, int64_t lds, unsigned* err, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  const int nst = per * kConsumers;
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t row_bytes = static_cast<uint32_t>(G) * 256;
  const uint16_t* gam = reinterpret_cast<const uint16_t*>(base);
  uint8_t* ring = base + row_bytes;
  uint8_t* outs = ring + static_cast<uint32_t>(nst) * row_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(outs + kConsumers * (row_bytes / 2));
  uint64_t* empty = full + nst;
  int* abort_flag = reinterpret_cast<int*>(empty + nst);
  const WaitCtl ctl{abort_flag, err, limit_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t H = static_cast<int64_t>(G) * 128;
  for (int i = threadIdx.x; i < G * 16; i += blockDim.x)
    reinterpret_cast<uint4*>(base)[i] = ld_nc_v4(gamma + i * 8);
  if (threadIdx.x == 0) {
    for (int st = 0; st < nst; ++st) {
      mbar_init(full + st, 1);
      mbar_init(empty + st, 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint64_t issued = 0, par = 0;  // bit st: stage st has a copy issued / its parity
      bool ok = true;
      int i = 0;
      for (int64_t t = blockIdx.x; t < M; t += gridDim.x, ++i) {
        const int li = i / kConsumers;  // the row's index among its warp's rows
        const int st = (i % kConsumers) * per + li % per;
        const uint32_t ph = static_cast<uint32_t>(li / per) & 1u;
        if (li >= per && !mbar_wait(empty + st, ph ^ 1u, ctl)) { ok = false; break; }
        mbar_arrive_expect_tx(full + st, row_bytes);
        tma_load_3d(ring + st * row_bytes, &tmX, 0, 0, static_cast<int32_t>(t), full + st);
        issued |= uint64_t{1} << st;
        par = (par & ~(uint64_t{1} << st)) | (static_cast<uint64_t>(ph) << st);
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        for (int st = 0; st < nst; ++st) {
          if (!((issued >> st) & 1u)) continue;
          const uint32_t a = smem_u32(full + st);
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(a, static_cast<uint32_t>(par >> st) & 1u))
            if (global_timer_ns() - t0 > limit_ns) break;
        }
      }
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  uint8_t* out = outs + warp * (row_bytes / 2);
  // lane l takes half h = l % 2 (64 values) of groups l/2, l/2 + 16, ...; chunk j of the
  // half is read in the rotated order h*8 + (j + l/2) % 8
  const int gl = lane >> 1, hh = lane & 1;
  const int rounds = (G + 15) >> 4;
  bool stored = false;
  int li = 0;
  for (int64_t t = blockIdx.x + static_cast<int64_t>(warp) * gridDim.x; t < M;
       t += static_cast<int64_t>(kConsumers) * gridDim.x, ++li) {
    const int st = warp * per + li % per;
    if (!mbar_wait_warp(full + st, static_cast<uint32_t>(li / per) & 1u, ctl)) break;
    const uint16_t* xr = reinterpret_cast<const uint16_t*>(ring + st * row_bytes);
    double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    for (int k = 0; k < rounds; ++k) {
      const int g = gl + 16 * k;
      if (g < G) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float v[8];
          unpack_bf16x8(*reinterpret_cast<const uint4*>(xr + g * 128 + (hh * 8 + ((j + gl) & 7)) * 8), v);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const double d = static_cast<double>(v[e]);
            acc[e] = __fma_rn(d, d, acc[e]);
          }
        }
      }
    }
    double ss = __dadd_rn(__dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3])),
                          __dadd_rn(__dadd_rn(acc[4], acc[5]), __dadd_rn(acc[6], acc[7])));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(kFull, ss, off));
    const float r = rstd_from_ss(ss, H, eps);
    if (stored) {  // the previous row's store must have read the staging row
      if (lane == 0) tma_store_wait_read();
      __syncwarp();
    }
    for (int k = 0; k < rounds; ++k) {
      const int g = gl + 16 * k;
      const bool act = g < G;
      const int gg = act ? g : 0;
      uint4 y[8];
      uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int off = gg * 128 + (hh * 8 + ((j + gl) & 7)) * 8;
        float xv[8], gv[8], b[8];
        unpack_bf16x8(*reinterpret_cast<const uint4*>(xr + off), xv);
        unpack_bf16x8(*reinterpret_cast<const uint4*>(gam + off), gv);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          float a0, a1;
          mul2(a0, a1, xv[e], xv[e + 1], r, r);
          mul2(b[e], b[e + 1], a0, a1, gv[e], gv[e + 1]);
        }
        y[j] = act ? make_uint4(pack_bf16x2(b[0], b[1]), pack_bf16x2(b[2], b[3]),
                                pack_bf16x2(b[4], b[5]), pack_bf16x2(b[6], b[7]))
                   : make_uint4(0u, 0u, 0u, 0u);
        m[0] = bf16x2_maxabs_xs(m[0], y[j].x);
        m[1] = bf16x2_maxabs_xs(m[1], y[j].y);
        m[2] = bf16x2_maxabs_xs(m[2], y[j].z);
        m[3] = bf16x2_maxabs_xs(m[3], y[j].w);
      }
      uint32_t mh = bf16x2_maxabs_xs(bf16x2_maxabs_xs(m[0], m[1]), bf16x2_maxabs_xs(m[2], m[3]));
      mh = bf16x2_maxabs_xs(mh, __shfl_xor_sync(kFull, mh, 1));  // the group's other half
      const GroupScale gs = group_scale_bf16(bf16x2_hmax_abs(mh));
      uint8_t* orow = out + gg * 128;
      if (__any_sync(kFull, gs.small)) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint2 c = codes8_words<true>(y[j], gs);
          if (act) *reinterpret_cast<uint2*>(orow + (hh * 8 + ((j + gl) & 7)) * 8) = c;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint2 c = codes8_words<false>(y[j], gs);
          if (act) *reinterpret_cast<uint2*>(orow + (hh * 8 + ((j + gl) & 7)) * 8) = c;
        }
      }
      if (act && hh == 0) s[static_cast<int64_t>(g) * lds + t] = gs.s;
    }
    __syncwarp();  // every lane is done with the stage and has staged its codes
    if (lane == 0) mbar_arrive(empty + st);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(&tmQ, out, 0, 0, static_cast<int32_t>(t));
      tma_store_commit();
    }
    stored = true;
  }
  if (stored && lane == 0) tma_store_wait_all();
}

// ---------------------------------------------------------------------------
// 128x128 tile helpers of the FP8 requantizer (a8) and of the fused dual producers:
// persistent CTAs of 256 threads. Tiles arrive in shared memory by TMA into a double
// buffer, so the next tile loads while this one is processed; a tile's arrival is an
// mbarrier that thread 0 waits on with the bounded wait (the CTA stops if it gives up,
// after letting issued copies land). Row pass: thread t owns rows t/16 + 16j (j = 0..7)
// and the 8 columns 8*(t%16) .. +7 of the staged tile (a half-warp reads one 256-byte
// row), so each row is one 1x128 group. Column pass: thread t owns the column pair
// 2*(t%64), +1 and the 32 rows 32*(t/64) .. +31; a warp reads 32 consecutive column pairs
// of one row per load (no bank conflicts) and each thread writes 2 x 32 consecutive codes
// of the transposed output as two 32-byte runs. (a2 and a6 have kernels of their own.)
// ---------------------------------------------------------------------------
constexpr int kTileElems = 128 * 128;

struct TileSmem {
  uint8_t* buf[2];
  uint64_t* bar;  // [2]
  float* red;     // [4 * 128]
  int* flag;
};

// Thread 0 waits for tile buffer b (bounded); every thread then acquires it. Returns
// false, uniformly across the CTA, if the wait gave up.
__device__ __forceinline__ bool tile_acquire(const TileSmem& sm, int b, uint32_t parity,
                                             const WaitCtl& ctl) {
  if (threadIdx.x == 0) *sm.flag = mbar_wait(sm.bar + b, parity, ctl) ? 1 : 0;
  __syncthreads();
  if (!*sm.flag) return false;
  mbar_try_wait(smem_u32(sm.bar + b), parity);  // completed: acquires the TMA writes
  return true;
}

// Codes of a column pair's kR values (lo / hi halves of w[]), four per word.
template <bool kMaybeSmall, int kR>
__device__ __forceinline__ void col_codes(const uint32_t (&w)[kR], const GroupScale& g0,
                                          const GroupScale& g1, uint32_t (&o0)[kR / 4],
                                          uint32_t (&o1)[kR / 4]) {
#pragma unroll
  for (int k = 0; k < kR / 4; ++k) {
    float t0[4], t1[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float x0 = bf16_lo(w[4 * k + i]), x1 = bf16_hi(w[4 * k + i]);
      if (kMaybeSmall) {
        t0[i] = g0.small ? __fdiv_rn(x0, g0.s) : quot(x0, g0);
        t1[i] = g1.small ? __fdiv_rn(x1, g1.s) : quot(x1, g1);
      } else {
        quot2(x0, x1, g0, g1, t0[i], t1[i]);
      }
    }
    o0[k] = cvt_e4m3x4(t0[0], t0[1], t0[2], t0[3]);
    o1[k] = cvt_e4m3x4(t1[0], t1[1], t1[2], t1[3]);
  }
}

// Column pass over a staged BF16 tile Ts[128][128] (dense rows) by a CTA of kThreads
// threads: thread t takes column pair t % 64 over kR = 128 / (kThreads / 64) consecutive
// rows. Column scales: computed per column (per_col; red holds kThreads / 64 x 128
// floats) or the given block scale. Codes go to dst[c * ldd + r] for tile column c and
// tile row r; per-column scales to scol[c]. Only the first `rows` rows and `cols`
// columns exist (a partial tile at the end of a ragged tensor, both multiples of 16;
// the staged tile holds zeros beyond them); nothing is stored outside them.
template <int kThreads = 256>
__device__ __forceinline__ void tile_cols_bf16(const uint16_t* Ts, float* red, bool per_col,
                                               const GroupScale& blk, uint8_t* __restrict__ dst,
                                               int64_t ldd, float* __restrict__ scol,
                                               const float* tab, int rows = 128,
                                               int cols = 128) {
  constexpr int kQ = kThreads / 64, kR = 128 / kQ;
  static_assert(kQ * 64 == kThreads && kR % 16 == 0, "column pass: 256 or 512 threads");
  const int tid = threadIdx.x;
  const int cp = tid & 63, rq = tid >> 6;
  uint32_t w[kR];
#pragma unroll
  for (int r = 0; r < kR; ++r) w[r] = *reinterpret_cast<const uint32_t*>(Ts + (kR * rq + r) * 128 + 2 * cp);
  GroupScale g0 = blk, g1 = blk;
  if (per_col) {
    // column maxima of the kR rows on packed pairs (four interleaved chains)
    uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int r = 0; r < kR; ++r) m[r & 3] = bf16x2_absmax(m[r & 3], w[r]);
    const uint32_t mm = bf16x2_absmax(bf16x2_absmax(m[0], m[1]), bf16x2_absmax(m[2], m[3]));
    red[rq * 128 + 2 * cp] = bf16_lo(mm);
    red[rq * 128 + 2 * cp + 1] = bf16_hi(mm);
    __syncthreads();
    float c0 = red[2 * cp], c1 = red[2 * cp + 1];
#pragma unroll
    for (int q = 1; q < kQ; ++q) {
      c0 = fmaxf(c0, red[q * 128 + 2 * cp]);
      c1 = fmaxf(c1, red[q * 128 + 2 * cp + 1]);
    }
    g0 = group_scale_bf16_sm(c0, tab);  // 32 different entries per warp: shared memory
    g1 = group_scale_bf16_sm(c1, tab);
    if (rq == 0 && scol && 2 * cp < cols)
      *reinterpret_cast<float2*>(scol + 2 * cp) = make_float2(g0.s, g1.s);
  }
  uint32_t o0[kR / 4], o1[kR / 4];
  if (__any_sync(kFull, g0.small || g1.small))
    col_codes<true, kR>(w, g0, g1, o0, o1);
  else
    col_codes<false, kR>(w, g0, g1, o0, o1);
  if (2 * cp >= cols) return;  // cols is even: the pair is in or out together
  uint4* d0 = reinterpret_cast<uint4*>(dst + (2 * cp) * ldd + kR * rq);
  uint4* d1 = reinterpret_cast<uint4*>(dst + (2 * cp + 1) * ldd + kR * rq);
#pragma unroll
  for (int k = 0; k < kR / 16; ++k) {
    if (kR * rq + 16 * k >= rows) break;  // rows is a multiple of 16
    d0[k] = make_uint4(o0[4 * k], o0[4 * k + 1], o0[4 * k + 2], o0[4 * k + 3]);
    d1[k] = make_uint4(o1[4 * k], o1[4 * k + 1], o1[4 * k + 2], o1[4 * k + 3]);
  }
}

// Shared memory of the FP8 tile kernel (a8): two (16 KB codes + 512 B row scales) buffers.
constexpr size_t kTileSmemFP8 = 1024 + 2 * (kTileElems + 512) + 4 * 128 * 4 + 64;

__device__ __forceinline__ TileSmem carve_tiles(uint8_t* raw, int buf_bytes,
                                               int red_floats = 4 * 128) {
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
  TileSmem sm;
  sm.buf[0] = base;
  sm.buf[1] = base + buf_bytes;
  sm.red = reinterpret_cast<float*>(base + 2 * buf_bytes);
  sm.bar = reinterpret_cast<uint64_t*>(base + 2 * buf_bytes + red_floats * 4);
  sm.flag = reinterpret_cast<int*>(sm.bar + 2);
  return sm;
}

// Shared prologue / epilogue of the persistent tile loops. `issue(b, t)` starts the
// copies of tile t into buffer b (thread 0 only).
template <class Issue>
__device__ __forceinline__ void tiles_prologue(const TileSmem& sm, int64_t tiles, Issue issue) {
  if (threadIdx.x == 0) {
    mbar_init(sm.bar, 1);
    mbar_init(sm.bar + 1, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int j = 0; j < 2; ++j) {
      const int64_t t = blockIdx.x + static_cast<int64_t>(j) * gridDim.x;
      if (t < tiles) issue(j, t);
    }
  }
}

// At the start of tile number i >= 1, right after its acquire barrier (so every thread
// has finished tile i - 1): refill buffer (i + 1) & 1, which held tile i - 1, with tile
// i + 1. The prologue already issued tiles 0 and 1. One load stays in flight while a
// tile is processed, and no barrier is needed at the end of a tile.
template <class Issue>
__device__ __forceinline__ void tiles_refill(int64_t t, int64_t tiles, int i, Issue issue) {
  if (i == 0) return;
  const int64_t tn = t + static_cast<int64_t>(gridDim.x);
  if (threadIdx.x == 0 && tn < tiles) issue((i + 1) & 1, tn);
}

// If the loop stopped at tile number i_stop (its wait gave up), let the copies still in
// flight land before exiting: tile i_stop, and tile 1 as well if i_stop is 0.
__device__ __forceinline__ void tiles_drain(const TileSmem& sm, int64_t t_stop, int64_t tiles,
                                            int i_stop, uint64_t limit_ns) {
  if (threadIdx.x != 0) return;
  for (int j = 0; j < (i_stop == 0 ? 2 : 1); ++j) {
    const int i = i_stop + j;
    const int64_t t = t_stop + static_cast<int64_t>(j) * gridDim.x;
    if (t < tiles) {
      const uint32_t a = smem_u32(sm.bar + (i & 1));
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(a, (i >> 1) & 1)) {
        if (global_timer_ns() - t0 > limit_ns) break;
      }
    }
  }
}


// ---------------------------------------------------------------------------
// Option B for saved activations (the producer emits both groupings from BF16, no FP8
// requantization): the producer's BF16 output is formed 128 x 128 tile by tile in shared
// memory and both groupings are quantized from it: the RMSNorm inside a6_tile_kernel
// with the TileRms source (after its per-row reciprocal RMS), the SwiGLU by
// swiglu_dual_tile_kernel.
// ---------------------------------------------------------------------------

// Per-row reciprocal RMS, r = (float)(1/sqrt(ss/H + eps)) with the fp64 sum of squares
// of the RMSNorm kernels (eight partial sums per lane, then a warp reduction).
__global__ void __launch_bounds__(256) rmsnorm_rstd_kernel(const uint16_t* __restrict__ x,
                                                           int64_t M, int64_t H, int64_t ldx,
                                                           float eps, float* __restrict__ rstd) {
  const int lane = threadIdx.x & 31;
  const int64_t nch = H >> 3;
  const int64_t wglobal = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t m = wglobal; m < M; m += nw) {
    const uint16_t* row = x + m * ldx;
    double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    int64_t c = lane;
    for (; c + 96 < nch; c += 128) {  // four 16-byte loads in flight per lane
      uint4 raw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) raw[u] = ld_nc_v4(row + (c + 32 * u) * 8);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float v[8];
        unpack_bf16x8(raw[u], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double d = static_cast<double>(v[i]);
          acc[i] = __fma_rn(d, d, acc[i]);
        }
      }
    }
    for (; c < nch; c += 32) {
      float v[8];
      unpack_bf16x8(ld_nc_v4(row + c * 8), v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const double d = static_cast<double>(v[i]);
        acc[i] = __fma_rn(d, d, acc[i]);
      }
    }
    double ss = __dadd_rn(__dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3])),
                          __dadd_rn(__dadd_rn(acc[4], acc[5]), __dadd_rn(acc[6], acc[7])));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(kFull, ss, off));
    if (lane == 0) rstd[m] = rstd_from_ss(ss, H, eps);
  }
}

// ---------------------------------------------------------------------------
// Tensors quantized both ways from a BF16 value formed on the fly (1x128 rows, and
// 128x1 columns stored transposed), one 128 x 128 unit at a time: a6 itself (the value
// is the input), the option-B forward producers, and the backward producers in BF16
// with a6 fused behind them (the gradient handed to the preceding linear layer never
// makes a BF16 round trip through HBM).
// ---------------------------------------------------------------------------

// SwiGLU backward per element, every step one IEEE fp32 operation (the exponential and
// silu as in the forward producer):
//   e = E(-g), d = 1 + e, silu = g / d, sig = 1 / d,
//   d_up = bf16(dh silu), d_gate = bf16((dh u) (sig (1 + g (1 - sig)))).
// silu and ds = sig (1 + g (1 - sig)) depend on the gate alone; sgb2 computes them for
// two gates.
__device__ __forceinline__ void sgb2(float g0, float g1, float& silu0, float& silu1, float& ds0,
                                     float& ds1) {
  float e0, e1;
  exp_cw2(-g0, -g1, e0, e1);
  const float d0 = __fadd_rn(1.0f, e0), d1 = __fadd_rn(1.0f, e1);
  const float sig0 = __frcp_rn(d0), sig1 = __frcp_rn(d1);
  // silu = g / d from sig = RN(1/d): q = g sig, t = q d - g, silu = q - t sig. For every
  // BF16 g (d = fl32(1 + E(-g))) this equals the IEEE quotient, signed zeros included
  // (exhaustive proof in the CPU tests); it replaces a second division.
  float q0, q1, t0 = -g0, t1 = -g1;
  mul2(q0, q1, g0, g1, sig0, sig1);
  fma2(t0, t1, q0, q1, d0, d1);
  silu0 = q0;
  silu1 = q1;
  fma2(silu0, silu1, t0, t1, -sig0, -sig1);
  const float t10 = __fsub_rn(1.0f, sig0), t11 = __fsub_rn(1.0f, sig1);
  float t20, t21;
  mul2(t20, t21, g0, g1, t10, t11);
  const float t30 = __fadd_rn(1.0f, t20), t31 = __fadd_rn(1.0f, t21);
  mul2(ds0, ds1, sig0, sig1, t30, t31);
}

// The products with dh and u for two columns, rounded to BF16.
__device__ __forceinline__ void swiglu_bwd_out2(float dh0, float dh1, float u0, float u1,
                                                float silu0, float silu1, float ds0, float ds1,
                                                float& dg0, float& dg1, float& du0, float& du1) {
  float a0, a1, b0, b1, c0, c1;
  mul2(a0, a1, dh0, dh1, silu0, silu1);
  mul2(b0, b1, dh0, dh1, u0, u1);
  mul2(c0, c1, b0, b1, ds0, ds1);
  dg0 = round_bf16(c0);
  dg1 = round_bf16(c1);
  du0 = round_bf16(a0);
  du1 = round_bf16(a1);
}

// A chunk: 8 consecutive gate, up and dh values of one row; v[0] receives d_gate, v[1]
// d_up.
__device__ __forceinline__ void swiglu_bwd8(const uint4& gw, const uint4& uw, const uint4& dw,
                                            float (&v)[2][8]) {
  float g[8], u[8], dh[8];
  unpack_bf16x8(gw, g);
  unpack_bf16x8(uw, u);
  unpack_bf16x8(dw, dh);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    float s0, s1, d0, d1;
    sgb2(g[i], g[i + 1], s0, s1, d0, d1);
    swiglu_bwd_out2(dh[i], dh[i + 1], u[i], u[i + 1], s0, s1, d0, d1, v[0][i], v[0][i + 1],
                    v[1][i], v[1][i + 1]);
  }
}

// The (silu, ds) pair of every BF16 gate in the table range of sg_index (62 KB), with
// the arithmetic of sgb2.
__device__ __forceinline__ void sgb_table_fill(float2* tab) {
  for (uint32_t i = threadIdx.x; i < kSgEntries / 2; i += blockDim.x) {
    const uint32_t e0 = 2 * i, e1 = 2 * i + 1;  // entries with the same sign
    const uint32_t sign = e0 / kSgHalf;
    const float g0 = __uint_as_float(((sign << 15) | ((e0 - sign * kSgHalf) + (kSgLoExp << 7))) << 16);
    const float g1 = __uint_as_float(((sign << 15) | ((e1 - sign * kSgHalf) + (kSgLoExp << 7))) << 16);
    float s0, s1, d0, d1;
    sgb2(g0, g1, s0, s1, d0, d1);
    tab[e0] = make_float2(s0, d0);
    tab[e1] = make_float2(s1, d1);
  }
}

// swiglu_bwd8 with silu and ds looked up in the table when every gate of the warp's
// chunks lies in its range (computed otherwise).
__device__ __forceinline__ void swiglu_bwd8_tab(const uint4& gw, const uint4& uw, const uint4& dw,
                                                const float2* tab, float (&v)[2][8]) {
  const uint32_t w[4] = {gw.x, gw.y, gw.z, gw.w};
  uint32_t idx[8];
  bool in = true;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    idx[2 * i] = sg_index(w[i] & 0xFFFFu);
    idx[2 * i + 1] = sg_index(w[i] >> 16);
    in = in && idx[2 * i] < kSgEntries && idx[2 * i + 1] < kSgEntries;
  }
  if (__all_sync(kFull, in)) {
    float u[8], dh[8];
    unpack_bf16x8(uw, u);
    unpack_bf16x8(dw, dh);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float2 t0 = tab[idx[i]], t1 = tab[idx[i + 1]];
      swiglu_bwd_out2(dh[i], dh[i + 1], u[i], u[i + 1], t0.x, t1.x, t0.y, t1.y, v[0][i],
                      v[0][i + 1], v[1][i], v[1][i + 1]);
    }
  } else {
    swiglu_bwd8(gw, uw, dw, v);
  }
}

// ---------------------------------------------------------------------------
// Exact sums of fp32 terms (the two reductions of the RMSNorm backward). A finite fp32
// value is m * 2^(e - 149) with an integer m < 2^24 and e in [0, 253] (subnormals:
// e = 0, no implicit bit). Bin b = e / 16 holds integers in units of 2^(16 b - 149); a
// term is m << (e % 16) (< 2^39) of them. Integer additions are exact, so the bins'
// total is the exact sum of the terms, whatever order the additions take (with fewer
// than 2^24 terms no bin can overflow). The total is rounded once at the end.
// ---------------------------------------------------------------------------
constexpr int kXBins = 16;

// One exact sum per thread: the two bins last added to are cached in registers (the
// terms of one sum usually span one or two bins); a bin that leaves the cache goes to
// spill(bin, units), an atomic add into integer bins in shared or global memory (rare).
// A cached bin is a double: the terms of bin b are integer multiples of its unit
// 2^(16 b - 149) below 2^39 units, and a double holds every such integer below 2^53
// exactly, so the fp64 additions of up to 2^14 terms are exact (no rounding) and
// cheaper than splitting each term into a bin and a 64-bit integer. The integer is
// formed once, when the bin leaves the cache.
struct XPair {
  double a0 = 0.0, a1 = 0.0;
  int b0 = -1, b1 = -1;
  // bin b's cached sum in units of 2^(16 b - 149) (an exact scaling by a power of two)
  static __device__ __forceinline__ long long units(double a, int b) {
    const double scale = __longlong_as_double(static_cast<long long>(1023 + 149 - 16 * b) << 52);
    return __double2ll_rn(__dmul_rn(a, scale));
  }
  template <class Spill>
  __device__ __forceinline__ void add(float t, Spill&& spill) {
    if (t == 0.0f) return;
    const uint32_t E = (__float_as_uint(t) >> 23) & 0xFFu;
    const int bin = (E ? static_cast<int>(E) - 1 : 0) >> 4;
    const double d = static_cast<double>(t);
    if (bin == b0) {
      a0 = __dadd_rn(a0, d);
    } else if (bin == b1) {
      a1 = __dadd_rn(a1, d);
    } else {
      if (b1 >= 0 && a1 != 0.0) spill(b1, units(a1, b1));
      b1 = b0;
      a1 = a0;
      b0 = bin;
      a0 = d;
    }
  }
  // bit b set where this lane's cache holds bin b
  __device__ __forceinline__ uint32_t mask() const {
    return (b0 >= 0 ? 1u << b0 : 0u) | (b1 >= 0 ? 1u << b1 : 0u);
  }
  __device__ __forceinline__ long long value(int b) const {
    return (b0 == b ? units(a0, b0) : 0) + (b1 == b ? units(a1, b1) : 0);
  }
};

// The value sum_b A[b] * 2^(16 b - 149) rounded once to a double: to nearest, ties to
// even, or, with `odd`, to odd (the last mantissa bit set when a lower bit is dropped;
// a double rounded to odd and then rounded to nearest fp32 is the fp32 nearest to the
// exact value, as 53 >= 24 + 2). An exact zero gives +0. Needs |A[b]| < 2^62.
__device__ double xbins_round(const long long (&A)[kXBins], bool odd) {
  // base-2^16 digits D[0..18] of the magnitude: the low 15 from a carry pass, the top bin
  // (with its carry, < 2^63) split into four more
  uint32_t D[kXBins + 3];
  long long carry = 0;
#pragma unroll
  for (int b = 0; b < kXBins - 1; ++b) carry = (carry + A[b]) >> 16;
  const bool neg = A[kXBins - 1] + carry < 0;
  carry = 0;
#pragma unroll
  for (int b = 0; b < kXBins - 1; ++b) {
    const long long t = (neg ? -A[b] : A[b]) + carry;
    D[b] = static_cast<uint32_t>(t & 0xFFFF);
    carry = t >> 16;  // arithmetic: the low digit stays in [0, 2^16)
  }
  unsigned long long top =
      static_cast<unsigned long long>((neg ? -A[kXBins - 1] : A[kXBins - 1]) + carry);
#pragma unroll
  for (int i = 0; i < 4; ++i) D[kXBins - 1 + i] = static_cast<uint32_t>((top >> (16 * i)) & 0xFFFF);
  int h = -1;
#pragma unroll
  for (int i = 0; i < kXBins + 3; ++i)
    if (D[i]) h = i;
  if (h < 0) return 0.0;
  // 64-bit window of digits h .. h-3 (missing digits are 0), left-aligned with bits of
  // digit h-4; everything below is the sticky bit
  unsigned long long w = 0;
  for (int i = h; i > h - 4; --i) w = (w << 16) | (i >= 0 ? D[i] : 0u);
  const uint32_t nxt = h - 4 >= 0 ? D[h - 4] : 0u;
  bool sticky = false;
  for (int i = h - 5; i >= 0; --i) sticky |= D[i] != 0;
  const int lz = __clzll(static_cast<long long>(w));  // 0..15: digit h is non-zero
  if (lz) {
    w = (w << lz) | (nxt >> (16 - lz));
    sticky |= (nxt & ((1u << (16 - lz)) - 1u)) != 0;
  } else {
    sticky |= nxt != 0;
  }
  // bit 63 of w has weight 2^e_top
  int e_top = 16 * (h - 3) - lz - 149 + 63;
  unsigned long long mant = w >> 11;  // 53 bits
  const uint32_t rem = static_cast<uint32_t>(w & 0x7FF);
  if (odd) {
    if (rem || sticky) mant |= 1ull;
  } else if (rem > 0x400u || (rem == 0x400u && (sticky || (mant & 1ull)))) {
    ++mant;
    if (mant >> 53) {
      mant >>= 1;
      ++e_top;
    }
  }
  // normal double (e_top >= -149): sign, biased exponent, 52 fraction bits
  const unsigned long long bits = (static_cast<unsigned long long>(neg) << 63) |
                                  (static_cast<unsigned long long>(e_top + 1023) << 52) |
                                  (mant & ((1ull << 52) - 1));
  return __longlong_as_double(static_cast<long long>(bits));
}

// Per-row scalars of the RMSNorm backward: r (as in the forward producer) and
// k = (float)((((c r) r) r) / H) in fp64, c = the exact sum of the fp32 products
// fl32(fl32(gamma_j dy_j) x_j) rounded once to a double. One warp per row.
__global__ void __launch_bounds__(256) rmsnorm_bwd_rows_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ gamma,
    const uint16_t* __restrict__ dy, int64_t M, int64_t H, float eps, float* __restrict__ r_out,
    float* __restrict__ k_out) {
  const int lane = threadIdx.x & 31;
  const int64_t nch = H >> 3;
  const int64_t wglobal = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  // bins evicted from the lanes' register caches, one set per warp
  __shared__ unsigned long long wbins[8][kXBins];
  unsigned long long* wb = wbins[threadIdx.x >> 5];
  auto spill = [&](int b, long long v) { atomicAdd(wb + b, static_cast<unsigned long long>(v)); };
  for (int64_t m = wglobal; m < M; m += nw) {
    const uint16_t* xr = x + m * H;
    const uint16_t* dr = dy + m * H;
    double ss[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    if (lane < kXBins) wb[lane] = 0ull;
    __syncwarp();
    XPair cc;
    int64_t c = lane;
    for (; c + 32 < nch; c += 64) {  // two chunks of each operand in flight per lane
      uint4 rx[2], rd[2], rg[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        rx[u] = ld_nc_v4(xr + (c + 32 * u) * 8);
        rd[u] = ld_nc_v4(dr + (c + 32 * u) * 8);
        rg[u] = __ldg(reinterpret_cast<const uint4*>(gamma + (c + 32 * u) * 8));
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float xv[8], dv[8], gv[8];
        unpack_bf16x8(rx[u], xv);
        unpack_bf16x8(rd[u], dv);
        unpack_bf16x8(rg[u], gv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double xd = static_cast<double>(xv[i]);
          ss[i] = __fma_rn(xd, xd, ss[i]);
          cc.add(__fmul_rn(__fmul_rn(gv[i], dv[i]), xv[i]), spill);
        }
      }
    }
    for (; c < nch; c += 32) {
      float xv[8], dv[8], gv[8];
      unpack_bf16x8(ld_nc_v4(xr + c * 8), xv);
      unpack_bf16x8(ld_nc_v4(dr + c * 8), dv);
      unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(gamma + c * 8)), gv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const double xd = static_cast<double>(xv[i]);
        ss[i] = __fma_rn(xd, xd, ss[i]);
        cc.add(__fmul_rn(__fmul_rn(gv[i], dv[i]), xv[i]), spill);
      }
    }
    double s2 = __dadd_rn(__dadd_rn(__dadd_rn(ss[0], ss[1]), __dadd_rn(ss[2], ss[3])),
                          __dadd_rn(__dadd_rn(ss[4], ss[5]), __dadd_rn(ss[6], ss[7])));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) s2 = __dadd_rn(s2, __shfl_xor_sync(kFull, s2, off));
    // the cached bins summed over the warp, bin by bin, plus the evicted ones
    __syncwarp();  // every eviction is in wb
    long long A[kXBins];
#pragma unroll
    for (int b = 0; b < kXBins; ++b) A[b] = static_cast<long long>(wb[b]);
    for (uint32_t used = __reduce_or_sync(kFull, cc.mask()); used; used &= used - 1) {
      const int b = __ffs(used) - 1;
      long long v = cc.value(b);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
      A[b] += v;
    }
    __syncwarp();  // wb is read before the next row clears it
    const double c2 = xbins_round(A, false);
    if (lane == 0) {
      const float r = rstd_from_ss(s2, H, eps);
      const double rd = static_cast<double>(r);
      double kd = __dmul_rn(c2, rd);
      kd = __dmul_rn(kd, rd);
      kd = __dmul_rn(kd, rd);
      kd = __ddiv_rn(kd, static_cast<double>(H));
      r_out[m] = r;
      k_out[m] = __double2float_rn(kd);
    }
  }
}

// RMSNorm backward per element: out = bf16(bf16(dx) + dres) with
// dx = fl32(fl32(r fl32(gamma dy)) - fl32(k x)) (dgamma has a kernel of its own). A
// thread's chunk: 8 consecutive x, dy (and dres) values of one row.
struct RmsBwd {
  const uint16_t* x;
  const uint16_t* dy;
  const uint16_t* dres;  // may be NULL
  const float* r;
  const float* k;
  const uint16_t* gamma;
  int64_t H;
  static constexpr int kOut = 1;
  static constexpr bool kHeavy = false;
  static constexpr bool kTails = false;  // ragged M / N accepted by its entry point
  struct In { uint4 x, d, res; };
  struct Col { float g[8]; };
  __device__ __forceinline__ Col column(int64_t c) const {
    Col k;
    unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(gamma + c)), k.g);
    return k;
  }
  __device__ __forceinline__ In load(int64_t m, int64_t col) const {
    In in;
    in.x = ld_nc_v4(x + m * H + col);
    in.d = ld_nc_v4(dy + m * H + col);
    in.res = dres ? ld_nc_v4(dres + m * H + col) : make_uint4(0u, 0u, 0u, 0u);
    return in;
  }
  __device__ __forceinline__ void form(const In& in, int64_t m, const Col& col,
                                       float (&v)[1][8]) const {
    const float(&gv)[8] = col.g;
    float xv[8], dv[8], rv[8];
    unpack_bf16x8(in.x, xv);
    unpack_bf16x8(in.d, dv);
    unpack_bf16x8(in.res, rv);
    const float rr = __ldg(r + m), kk = __ldg(k + m);
    const bool res = dres != nullptr;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      float gd0, gd1, a0, a1, b0, b1;
      mul2(gd0, gd1, gv[i], gv[i + 1], dv[i], dv[i + 1]);
      mul2(a0, a1, gd0, gd1, rr, rr);
      mul2(b0, b1, xv[i], xv[i + 1], kk, kk);
      float o0 = round_bf16(__fsub_rn(a0, b0)), o1 = round_bf16(__fsub_rn(a1, b1));
      if (res) {
        o0 = round_bf16(__fadd_rn(o0, rv[i]));
        o1 = round_bf16(__fadd_rn(o1, rv[i + 1]));
      }
      v[0][i] = o0;
      v[0][i + 1] = o1;
    }
  }
};

// Rows loaded per batch and the occupancy the backward kernels are compiled for.
constexpr int kBwdBatch = 2;
constexpr int kBwdMinBlocks = 3;

// Shared memory of the unit kernels: the formed BF16 output tile(s) and one column
// reduction per output tile.
template <class X>
constexpr size_t direct_smem_bytes() {
  return X::kOut * (kTileElems * 2 + 4 * 128 * 4) + 256 * 4;
}

// One 128 x 128 unit of direct_dual_kernel (described there). kEdge: the unit may reach
// past a ragged M or N; loads past them read zeros and nothing past them is stored.
template <class X, int kBatch, bool kEdge>
__device__ __forceinline__ void dual_unit(const X& xf, int64_t mb, int64_t nb, int64_t M, int64_t N,
                                          uint16_t* __restrict__ bf16_out,
                                          uint8_t* __restrict__ q_row, float* __restrict__ s_row,
                                          int64_t lds_row, uint8_t* __restrict__ q_colT,
                                          float* __restrict__ s_col, uint16_t* tile, float* red,
                                          const float* stab) {
  constexpr int kOut = X::kOut;
  const int64_t Nout = kOut * N;
  const int tid = threadIdx.x;
  const int rr = tid >> 4, c8 = (tid & 15) * 8;
  const GroupScale unused{1.0f, 1.0f, -1.0f, false};
  {
    const int64_t col = nb * 128 + c8;
    const bool col_ok = !kEdge || col < N;  // N is a multiple of 8: a chunk is in or out
    const typename X::Col cs = xf.column(col_ok ? col : 0);
    // unrolled for short forms; a long form (the SwiGLU exponential and divisions) stays
    // rolled, which keeps the kernel inside the instruction cache (measured faster)
    constexpr int kOuterUnroll = X::kHeavy ? 1 : 8 / kBatch;
#pragma unroll kOuterUnroll
    for (int h = 0; h < 8 / kBatch; ++h) {
      typename X::In in[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int64_t m = mb * 128 + rr + 16 * (h * kBatch + j);
        if (!kEdge || (m < M && col_ok)) in[j] = xf.load(m, col);
        else in[j] = typename X::In{};
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int r = rr + 16 * (h * kBatch + j);
        const int64_t m = mb * 128 + r;
        const bool ok = !kEdge || (m < M && col_ok);
        float v[kOut][8];
        xf.form(in[j], ok ? m : 0, cs, v);
#pragma unroll
        for (int o = 0; o < kOut; ++o) {
          const int64_t oc = o * N + nb * 128 + c8;  // output column of this chunk
          const uint4 pk = make_uint4(pack_bf16x2(v[o][0], v[o][1]), pack_bf16x2(v[o][2], v[o][3]),
                                      pack_bf16x2(v[o][4], v[o][5]), pack_bf16x2(v[o][6], v[o][7]));
          *reinterpret_cast<uint4*>(tile + o * kTileElems + r * 128 + c8) = pk;
          if (bf16_out && ok) *reinterpret_cast<uint4*>(bf16_out + m * Nout + oc) = pk;
          if (q_row) {
            uint2 codes;
            const float sc = quant_half_warp(v[o], codes);  // every lane takes part
            if (ok) *reinterpret_cast<uint2*>(q_row + m * Nout + oc) = codes;
            if ((tid & 15) == 0 && (!kEdge || m < M)) s_row[((o * N) / 128 + nb) * lds_row + m] = sc;
          }
        }
      }
    }
    __syncthreads();
    // Each column pass reads its tile into registers before its own barrier, so once
    // every thread is past the last one the tiles may be overwritten by the next unit.
    const int rows = kEdge && M - mb * 128 < 128 ? static_cast<int>(M - mb * 128) : 128;
    const int cols = kEdge && N - nb * 128 < 128 ? static_cast<int>(N - nb * 128) : 128;
#pragma unroll
    for (int o = 0; o < kOut; ++o) {
      const int64_t oc0 = o * N + nb * 128;
      tile_cols_bf16<256>(tile + o * kTileElems, red + o * 4 * 128, true, unused,
                          q_colT + oc0 * M + mb * 128, M, s_col + mb * Nout + oc0, stab, rows,
                          cols);
    }
  }
}

// The checked unit out of line, so that the rare edge path does not take registers from
// the common one.
template <class X, int kBatch>
__device__ __noinline__ void dual_unit_edge(const X& xf, int64_t mb, int64_t nb, int64_t M,
                                            int64_t N, uint16_t* bf16_out, uint8_t* q_row,
                                            float* s_row, int64_t lds_row, uint8_t* q_colT,
                                            float* s_col, uint16_t* tile, float* red,
                                            const float* stab) {
  dual_unit<X, kBatch, true>(xf, mb, nb, M, N, bf16_out, q_row, s_row, lds_row, q_colT, s_col,
                             tile, red, stab);
}

// Persistent over the ceil(M/128) x NB units (NB = ceil(N/128)); unit t covers rows
// (t / NB) * 128 and input columns (t % NB) * 128. Each thread loads its chunks (rows
// rr + 16 j, columns c8..c8+7) straight into registers, kBatch rows at a time, forms the
// gradient, stores it in the output tile(s) in shared memory (and in bf16_out if given)
// and quantizes its rows; after one barrier the column pass runs on the staged tile(s).
// Output tile o covers columns o * N + nb * 128 of the [M, Nout] output (Nout = kOut *
// N): for the SwiGLU d_gate and d_up, for the RMSNorm the gradient itself. M and N must
// be multiples of 16; the chunks of a partial unit past them are zeros (they raise no
// group maximum) and are not stored.
template <class X, int kBatch, int kMinBlocks>
__global__ void __launch_bounds__(256, kMinBlocks) direct_dual_kernel(
    X xf, int64_t M, int64_t N, uint16_t* __restrict__ bf16_out, uint8_t* __restrict__ q_row,
    float* __restrict__ s_row, int64_t lds_row, uint8_t* __restrict__ q_colT,
    float* __restrict__ s_col) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  constexpr int kOut = X::kOut;
  uint16_t* tile = reinterpret_cast<uint16_t*>(smem_raw);
  float* red = reinterpret_cast<float*>(smem_raw + kOut * kTileElems * 2);
  // the scale tables, after the tiles
  float* stab = reinterpret_cast<float*>(smem_raw + kOut * (kTileElems * 2 + 4 * 128 * 4));
  scale_tables_fill(stab);
  const X& xs = xf;
  __syncthreads();
  const int64_t NB = (N + 127) >> 7;
  const int64_t tiles = ((M + 127) >> 7) * NB;
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
    const int64_t mb = t / NB, nb = t % NB;
    // a unit past the end of a ragged M or N (only sources that accept one) takes the
    // checked path; whole units take the unchecked one
    if (X::kTails && (mb * 128 + 128 > M || nb * 128 + 128 > N))
      dual_unit_edge<X, kBatch>(xs, mb, nb, M, N, bf16_out, q_row, s_row, lds_row, q_colT, s_col,
                                tile, red, stab);
    else
      dual_unit<X, kBatch, false>(xs, mb, nb, M, N, bf16_out, q_row, s_row, lds_row, q_colT,
                                  s_col, tile, red, stab);
  }
}

// a6 for a BF16 gradient that is already formed, and the producers that form their BF16
// value from staged inputs (option B's RMSNorm and SwiGLU, the SwiGLU backward): both
// groupings from one 128 x 128 tile staged by tensor copies, persistent CTAs of 17 warps.
//   warps 0-7  1x128 rows: lane l of warp w holds half of row 16w + (l % 16) of the tile
//              (columns 64 (l / 16) .. +63; the halves meet by one shuffle). A forming
//              source has these warps form their rows from the staged inputs first and
//              write them over the first box(es). Codes leave through a per-warp staging
//              box and a tensor store, one scale store per row.
//   warps 8-15 128x1 columns: warp 8 + 4h + q reads rows 32q .. 32q+31 of the column
//              pairs 64h + (2l, 2l+1), l the lane (one 4-byte word per row and lane, 128
//              consecutive bytes per warp load). Partial maxima of the four row quarters
//              meet in shared memory; every lane then forms the scales of its two columns
//              and quantizes its 2 columns x 32 rows into a transposed [128 columns][128
//              rows] staging tile (128-byte swizzle, 2-way bank conflicts at most), which
//              one tensor store writes to q_colT.
//   warp 16    producer: tiles into a ring of stages of kBoxes boxes each.
// The scale tables sit in shared memory here: the column scales look up 32 different
// entries per warp load, which the constant cache would serve one at a time.
#ifndef A6_STAGES
#define A6_STAGES 4
#endif
constexpr int kA6Stages = A6_STAGES;  // boxes in the ring of a one- or two-box source
constexpr uint32_t kA6Tile = 128 * 128 * 2;
constexpr int kA6Threads = 17 * 32;
template <class Src>
struct A6Layout {
  static constexpr int kStages = kA6Stages / Src::kBoxes;
  static constexpr uint32_t kStageBytes = Src::kBoxes * kA6Tile;
  static constexpr uint32_t kOffCol = kStages * kStageBytes;  // transposed codes, 16 KB
  static constexpr uint32_t kOffRow = kOffCol + 128 * 128;    // 8 x (16 x 128) row codes
  static constexpr uint32_t kOffRed = kOffRow + 128 * 128;    // [4][64] partial maxima
  static constexpr uint32_t kOffTab = kOffRed + 4 * 64 * 4;  // scale and reciprocal tables
  static constexpr uint32_t kOffBar = kOffTab + 256 * 4;     // full, empty, formed, csync
  static constexpr size_t kSmem = 1024 + kOffBar + (3 * kStages + 1) * 8 + 16;
};
template <class Src>
constexpr size_t a6_smem() {
  return A6Layout<Src>::kSmem;
}

// Sources of the tile kernel. kBoxes tensor copies per tile (the ring then holds
// kA6Stages / kBoxes tiles); with kForm the row warps form the BF16 value from them and
// write it over box 0, where the column warps read it once all eight row warps are done.
struct TileGrad {  // a6: the BF16 gradient itself (no forming step)
  static constexpr int kBoxes = 1;
  static constexpr bool kForm = false;
};

struct TileRms {  // option B, RMSNorm: y = bf16(fl32(fl32(x r) g)), r from the pre-pass
  const float* rstd;
  const uint16_t* gamma;
  static constexpr int kBoxes = 1;
  static constexpr bool kForm = true;
  __device__ __forceinline__ float row_factor(int64_t m) const { return __ldg(rstd + m); }
  // 8 values at x0 (staged), output columns col .. col + 7
  __device__ __forceinline__ uint4 form(const uint16_t* x0, const uint16_t*, int64_t col,
                                        float r) const {
    float xv[8], gv[8], b[8];
    unpack_bf16x8(*reinterpret_cast<const uint4*>(x0), xv);
    unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(gamma + col)), gv);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      float a0, a1;
      mul2(a0, a1, xv[i], xv[i + 1], r, r);
      mul2(b[i], b[i + 1], a0, a1, gv[i], gv[i + 1]);
    }
    return make_uint4(pack_bf16x2(b[0], b[1]), pack_bf16x2(b[2], b[3]), pack_bf16x2(b[4], b[5]),
                      pack_bf16x2(b[6], b[7]));
  }
};


// Group maximum from a lane's four running bf16x2 maxima and its partner's (lane ^ 16).
__device__ __forceinline__ float half_row_amax_finish(const uint32_t (&m)[4]) {
  uint32_t mh = bf16x2_maxabs_xs(bf16x2_maxabs_xs(m[0], m[1]), bf16x2_maxabs_xs(m[2], m[3]));
  mh = bf16x2_maxabs_xs(mh, __shfl_xor_sync(kFull, mh, 16));
  return bf16x2_hmax_abs(mh);
}

// Group maximum of a lane's 64 values w and its partner's.
__device__ __forceinline__ float half_row_amax(const uint4 (&w)[8]) {
  uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    m[0] = bf16x2_maxabs_xs(m[0], w[j].x);
    m[1] = bf16x2_maxabs_xs(m[1], w[j].y);
    m[2] = bf16x2_maxabs_xs(m[2], w[j].z);
    m[3] = bf16x2_maxabs_xs(m[3], w[j].w);
  }
  return half_row_amax_finish(m);
}

// A lane's 64 codes of w (scale g) at orow, chunk j at position (j + lane) % 8.
__device__ __forceinline__ void half_row_codes(const uint4 (&w)[8], const GroupScale& g,
                                               uint8_t* orow, int lane) {
  if (__any_sync(kFull, g.small)) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint2*>(orow + ((j + lane) & 7) * 8) = codes8_words<true>(w[j], g);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint2*>(orow + ((j + lane) & 7) * 8) = codes8_words<false>(w[j], g);
  }
}

template <class Src, bool kRows>
__global__ void __launch_bounds__(kA6Threads, 1) a6_tile_kernel(
    const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmD1,
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQT, Src src,
    int64_t M, int64_t N, float* __restrict__ s_row, int64_t lds_row, float* __restrict__ s_col,
    unsigned* err, uint64_t limit_ns) {
  using L = A6Layout<Src>;
  constexpr int kStages = L::kStages;
  constexpr uint32_t kStageBytes = L::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* tab = reinterpret_cast<float*>(base + L::kOffTab);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L::kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* formed = empty + kStages;  // kForm: the eight row warps have written the tile
  uint64_t* csync = formed + kStages;  // the column warps' rendezvous (bounded, unlike bar.sync)
  int* abort_flag = reinterpret_cast<int*>(csync + 1);
  const WaitCtl ctl{abort_flag, err, limit_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 128) {
    tab[threadIdx.x] = kScaleMant[threadIdx.x];
    tab[128 + threadIdx.x] = kRecipMant[threadIdx.x];
  }
  if (threadIdx.x == 0) {
    for (int b = 0; b < kStages; ++b) {
      mbar_init(full + b, 1);
      mbar_init(empty + b, 16);
      mbar_init(formed + b, 8);
    }
    mbar_init(csync, 8);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t NB = (N + 127) >> 7;
  const int64_t tiles = ((M + 127) >> 7) * NB;
  if (warp == 16) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0, par = 0;
      bool ok = true;
      int i = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
        const int b = i % kStages;
        const uint32_t ph = static_cast<uint32_t>(i / kStages) & 1u;
        if (i >= kStages && !mbar_wait(empty + b, ph ^ 1u, ctl)) { ok = false; break; }
        const int64_t mb = t / NB, nb = t - mb * NB;
        mbar_arrive_expect_tx(full + b, kStageBytes);
        tma_load_2d(base + b * kStageBytes, &tmD, static_cast<int32_t>(nb * 128),
                    static_cast<int32_t>(mb * 128), full + b);
        if (Src::kBoxes == 2)
          tma_load_2d(base + b * kStageBytes + kA6Tile, &tmD1, static_cast<int32_t>(nb * 128),
                      static_cast<int32_t>(mb * 128), full + b);
        issued |= 1u << b;
        par = (par & ~(1u << b)) | (ph << b);
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        for (int b = 0; b < kStages; ++b) {
          if (!((issued >> b) & 1u)) continue;
          const uint32_t a = smem_u32(full + b);
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(a, (par >> b) & 1u))
            if (global_timer_ns() - t0 > limit_ns) break;
        }
      }
    }
    return;
  }
  bool stored = false;
  if (warp < 8) {
    // ------------------------------------------------------------ 1x128 rows
    // lane l of warp w: row 16w + (l % 16) of the tile, chunks 8 (l / 16) .. + 7 of it
    uint8_t* out = base + L::kOffRow + warp * (16 * 128);
    const int rl = lane & 15, hh = lane >> 4;
    int i = 0;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int b = i % kStages;
      if (!mbar_wait_warp(full + b, static_cast<uint32_t>(i / kStages) & 1u, ctl)) break;
      if (!kRows && !Src::kForm) {
        if (lane == 0) mbar_arrive(empty + b);
        continue;
      }
      const int64_t mb = t / NB, nb = t - mb * NB;
      const int roff = (warp * 16 + rl) * 128 + hh * 64;
      uint16_t* row = reinterpret_cast<uint16_t*>(base + b * kStageBytes) + roff;
      uint4 w[8];
      if constexpr (Src::kForm) {
        // form the value from the staged inputs and write it over box 0 (same rotated
        // order as the reads: no bank conflicts)
        const uint16_t* row1 = reinterpret_cast<const uint16_t*>(base + b * kStageBytes + kA6Tile) + roff;
        const float rf = src.row_factor(mb * 128 + warp * 16 + rl);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int off = ((j + lane) & 7) * 8;
          w[j] = src.form(row + off, row1 + off, nb * 128 + hh * 64 + off, rf);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(row + ((j + lane) & 7) * 8) = w[j];
        __syncwarp();
        if (lane == 0) mbar_arrive(formed + b);  // release: the column warps may read it
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = *reinterpret_cast<const uint4*>(row + ((j + lane) & 7) * 8);
      }
      const float amax = half_row_amax(w);
      __syncwarp();  // every lane's reads of the tile are complete (their values are used)
      if (lane == 0) mbar_arrive(empty + b);
      if (!kRows) continue;
      const GroupScale g = group_scale_bf16_sm(amax, tab);
      if (stored) {
        if (lane == 0) tma_store_wait_read();
        __syncwarp();
      }
      half_row_codes(w, g, out + rl * 128 + hh * 64, lane);
      fence_proxy_async_smem();
      __syncwarp();
      const int64_t m0 = mb * 128 + warp * 16;
      if (lane == 0) {
        tma_store_2d(&tmQ, out, static_cast<int32_t>(nb * 128), static_cast<int32_t>(m0));
        tma_store_commit();
      }
      stored = true;
      if (hh == 0 && m0 + rl < M) s_row[nb * lds_row + m0 + rl] = g.s;
    }
  } else {
    // ------------------------------------------------------------ 128x1 columns
    const int cw = warp - 8;
    const int q4 = cw & 3;                // row quarter: rows 32 q4 .. 32 q4 + 31
    const int c0 = 64 * (cw >> 2) + 2 * lane;  // this lane's column pair c0, c0 + 1
    uint32_t* red = reinterpret_cast<uint32_t*>(base + L::kOffRed);
    uint8_t* colst = base + L::kOffCol;
    // The eight column warps meet twice a tile: each warp's lanes finish their shared-
    // memory writes, lane 0 arrives, and the warp waits (bounded) for the phase.
    uint32_t nsync = 0;
    auto col_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(csync);
      return mbar_wait_warp(csync, (nsync++) & 1u, ctl);
    };
    int i = 0;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int b = i % kStages;
      if (!mbar_wait_warp(Src::kForm ? formed + b : full + b,
                          static_cast<uint32_t>(i / kStages) & 1u, ctl))
        break;
      const uint32_t* tw = reinterpret_cast<const uint32_t*>(base + b * kStageBytes) + q4 * 32 * 64 + (c0 >> 1);
      uint32_t w[32];  // columns c0, c0 + 1 of rows 32 q4 + k
#pragma unroll
      for (int k = 0; k < 32; ++k) w[k] = tw[k * 64];
      uint32_t m0 = 0u, m1 = 0u;
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        m0 = bf16x2_maxabs_xs(m0, w[k]);
        m1 = bf16x2_maxabs_xs(m1, w[k + 1]);
      }
      __syncwarp();  // every lane's reads of the tile are complete (their values are used)
      if (lane == 0) mbar_arrive(empty + b);
      red[q4 * 64 + (c0 >> 1)] = bf16x2_maxabs_xs(m0, m1);
      if (stored && cw == 0 && lane == 0) tma_store_wait_read();  // the staging tile is free
      if (!col_sync()) break;
      const int64_t mb = t / NB, nb = t - mb * NB;
      uint32_t mm = 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) mm = bf16x2_maxabs_xs(mm, red[q * 64 + (c0 >> 1)]);
      const GroupScale g0 = group_scale_bf16_sm(fabsf(bf16_lo(mm)), tab);
      const GroupScale g1 = group_scale_bf16_sm(fabsf(bf16_hi(mm)), tab);
      if (q4 == 0 && nb * 128 + c0 < N)
        *reinterpret_cast<float2*>(s_col + mb * N + nb * 128 + c0) = make_float2(g0.s, g1.s);
      uint32_t o0[8], o1[8];
      if (__any_sync(kFull, g0.small || g1.small))
        col_codes<true, 32>(w, g0, g1, o0, o1);
      else
        col_codes<false, 32>(w, g0, g1, o0, o1);
      // staging row c holds column c's 128 codes; 16-byte chunk k of the row (rows 16k ..
      // 16k+15 of the tile) sits at position k ^ (c & 7) (the 128-byte swizzle)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = c0 + e;
        const uint32_t* o = e ? o1 : o0;
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int k = 2 * q4 + k2;
          *reinterpret_cast<uint4*>(colst + c * 128 + ((k ^ (c & 7)) << 4)) =
              make_uint4(o[4 * k2], o[4 * k2 + 1], o[4 * k2 + 2], o[4 * k2 + 3]);
        }
      }
      fence_proxy_async_smem();
      if (!col_sync()) break;
      if (cw == 0 && lane == 0) {
        tma_store_2d(&tmQT, colst, static_cast<int32_t>(mb * 128), static_cast<int32_t>(nb * 128));
        tma_store_commit();
      }
      stored = true;
    }
  }
  if (stored && lane == 0) tma_store_wait_all();
}

// ---------------------------------------------------------------------------
// Option B's SwiGLU producer (f2): h = bf16(fl32(sg(g) u)) in both groupings, on the
// layout of the SwiGLU backward's kernel below: a stage holds the gate and up boxes of a
// 128 x 128 tile (two stages), sg comes from a4's per-CTA table, and all sixteen
// consumer warps form eight rows each (four lanes per row, chunks rotated by the row),
// write h over the gate box, store their rows' codes from registers and arrive on
// `formed`; then every warp quantizes 16 rows x 2 columns of the tile (warp w: rows
// 16 (w % 8) .. +15, column pairs 64 (w / 8) + 2 lane), the eight partial maxima of a
// column meet in shared memory, and the transposed codes are staged over the first half
// of the gate box for one tensor store.
// ---------------------------------------------------------------------------
constexpr int kSfStages = 2;
constexpr uint32_t kSfStageBytes = 2 * kA6Tile;               // gate and up boxes
constexpr uint32_t kSfOffGate = kSfStages * kSfStageBytes;    // sg per gate
constexpr uint32_t kSfOffRed = kSfOffGate + kSgEntries * 4;   // [8][64] partial maxima
constexpr uint32_t kSfOffTab = kSfOffRed + 8 * 64 * 4;        // scale and reciprocal tables
constexpr uint32_t kSfOffBar = kSfOffTab + 256 * 4;           // full, empty, formed, csync
constexpr size_t kSfSmem = 1024 + kSfOffBar + (3 * kSfStages + 1) * 8 + 16;

__global__ void __launch_bounds__(kA6Threads, 1) swiglu_dual_tile_kernel(
    const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmU,
    const __grid_constant__ CUtensorMap tmQT, uint8_t* __restrict__ q_row, int64_t M, int64_t I,
    float* __restrict__ s_row, int64_t lds_row, float* __restrict__ s_col, unsigned* err,
    uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* gtab = reinterpret_cast<float*>(base + kSfOffGate);
  float* tab = reinterpret_cast<float*>(base + kSfOffTab);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kSfOffBar);
  uint64_t* empty = full + kSfStages;
  uint64_t* formed = empty + kSfStages;  // all sixteen warps have formed their rows
  uint64_t* csync = formed + kSfStages;  // the sixteen warps' column rendezvous
  int* abort_flag = reinterpret_cast<int*>(csync + 1);
  const WaitCtl ctl{abort_flag, err, limit_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 128) {
    tab[threadIdx.x] = kScaleMant[threadIdx.x];
    tab[128 + threadIdx.x] = kRecipMant[threadIdx.x];
  }
  sg_table_fill(gtab);
  if (threadIdx.x == 0) {
    for (int b = 0; b < kSfStages; ++b) {
      mbar_init(full + b, 1);
      mbar_init(empty + b, 16);
      mbar_init(formed + b, 16);
    }
    mbar_init(csync, 16);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t NB = I >> 7;
  const int64_t tiles = (M >> 7) * NB;
  if (warp == 16) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0, par = 0;
      bool ok = true;
      int i = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
        const int b = i % kSfStages;
        const uint32_t ph = static_cast<uint32_t>(i / kSfStages) & 1u;
        if (i >= kSfStages && !mbar_wait(empty + b, ph ^ 1u, ctl)) { ok = false; break; }
        const int64_t mb = t / NB, nb = t - mb * NB;
        const int32_t x = static_cast<int32_t>(nb * 128), y = static_cast<int32_t>(mb * 128);
        uint8_t* st = base + b * kSfStageBytes;
        mbar_arrive_expect_tx(full + b, kSfStageBytes);
        tma_load_2d(st, &tmG, x, y, full + b);
        tma_load_2d(st + kA6Tile, &tmU, x, y, full + b);
        issued |= 1u << b;
        par = (par & ~(1u << b)) | (ph << b);
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        for (int b = 0; b < kSfStages; ++b) {
          if (!((issued >> b) & 1u)) continue;
          const uint32_t a = smem_u32(full + b);
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(a, (par >> b) & 1u))
            if (global_timer_ns() - t0 > limit_ns) break;
        }
      }
    }
    return;
  }
  // row phase: tile row r = 8 warp + lr, chunks (a + 4k + 4 (lr % 4)) % 16, k = 0 .. 3
  const int lr = lane >> 2, a = lane & 3;
  const int r = warp * 8 + lr;
  auto chunk = [&](int k) { return (a + 4 * k + 4 * (lr & 3)) & 15; };
  // column phase: rows 16 q8 .. +15, column pair c0, c0 + 1
  const int q8 = warp & 7;
  const int c0 = 64 * (warp >> 3) + 2 * lane;
  uint32_t* red = reinterpret_cast<uint32_t*>(base + kSfOffRed);
  uint32_t nsync = 0;
  auto col_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(csync);
    return mbar_wait_warp(csync, (nsync++) & 1u, ctl);
  };
  bool stored = false;
  int i = 0;
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
    const int b = i % kSfStages;
    const uint32_t ph = static_cast<uint32_t>(i / kSfStages) & 1u;
    if (!mbar_wait_warp(full + b, ph, ctl)) break;
    const int64_t mb = t / NB, nb = t - mb * NB;
    uint8_t* st = base + b * kSfStageBytes;
    // ---------------------------------------------------------------- rows
    {
      uint16_t* rg = reinterpret_cast<uint16_t*>(st) + r * 128;
      const uint16_t* ru = reinterpret_cast<const uint16_t*>(st + kA6Tile) + r * 128;
      uint4 h[4];
      uint32_t mh[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int off = chunk(k) * 8;
        float v[8];
        SwigluBoxes::values(rg, ru, off, gtab, v);
        h[k] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                          pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
        *reinterpret_cast<uint4*>(rg + off) = h[k];
        mh[0] = bf16x2_maxabs_xs(mh[0], h[k].x);
        mh[1] = bf16x2_maxabs_xs(mh[1], h[k].y);
        mh[2] = bf16x2_maxabs_xs(mh[2], h[k].z);
        mh[3] = bf16x2_maxabs_xs(mh[3], h[k].w);
      }
      fence_proxy_async_smem();  // the stage is written by tensor copies and read by a store later
      __syncwarp();
      if (lane == 0) mbar_arrive(formed + b);  // release: the column pass may read the rows
      // the row's four lanes are adjacent: two shuffles give its maximum
      uint32_t hm = bf16x2_maxabs_xs(bf16x2_maxabs_xs(mh[0], mh[1]), bf16x2_maxabs_xs(mh[2], mh[3]));
      hm = bf16x2_maxabs_xs(hm, __shfl_xor_sync(kFull, hm, 1));
      hm = bf16x2_maxabs_xs(hm, __shfl_xor_sync(kFull, hm, 2));
      const GroupScale g = group_scale_bf16_sm(bf16x2_hmax_abs(hm), tab);
      const int64_t m = mb * 128 + r;
      uint8_t* qr = q_row + m * I + nb * 128;
      if (__any_sync(kFull, g.small)) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint2*>(qr + chunk(k) * 8) = codes8_words<true>(h[k], g);
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint2*>(qr + chunk(k) * 8) = codes8_words<false>(h[k], g);
      }
      if (a == 0) s_row[nb * lds_row + m] = g.s;
    }
    if (!mbar_wait_warp(formed + b, ph, ctl)) break;
    // ---------------------------------------------------------------- columns
    {
      const uint32_t* tw = reinterpret_cast<const uint32_t*>(st) + q8 * 16 * 64 + (c0 >> 1);
      uint32_t w[16];  // columns c0, c0 + 1 of rows 16 q8 + k
#pragma unroll
      for (int k = 0; k < 16; ++k) w[k] = tw[k * 64];
      uint32_t m0 = 0u, m1 = 0u;
#pragma unroll
      for (int k = 0; k < 16; k += 2) {
        m0 = bf16x2_maxabs_xs(m0, w[k]);
        m1 = bf16x2_maxabs_xs(m1, w[k + 1]);
      }
      red[q8 * 64 + (c0 >> 1)] = bf16x2_maxabs_xs(m0, m1);
      if (!col_sync()) break;  // every warp's reads of the tile are done: it may be overwritten
      uint32_t mm = 0u;
#pragma unroll
      for (int q = 0; q < 8; ++q) mm = bf16x2_maxabs_xs(mm, red[q * 64 + (c0 >> 1)]);
      const GroupScale g0 = group_scale_bf16_sm(fabsf(bf16_lo(mm)), tab);
      const GroupScale g1 = group_scale_bf16_sm(fabsf(bf16_hi(mm)), tab);
      if (q8 == 0)
        *reinterpret_cast<float2*>(s_col + mb * I + nb * 128 + c0) = make_float2(g0.s, g1.s);
      uint32_t o0[4], o1[4];
      if (__any_sync(kFull, g0.small || g1.small))
        col_codes<true, 16>(w, g0, g1, o0, o1);
      else
        col_codes<false, 16>(w, g0, g1, o0, o1);
      // staging (first 16 KB of the gate box): row c holds column c's 128 codes, 16-byte
      // chunk q8 at position q8 ^ (c & 7) (the 128-byte swizzle)
      *reinterpret_cast<uint4*>(st + c0 * 128 + ((q8 ^ (c0 & 7)) << 4)) =
          make_uint4(o0[0], o0[1], o0[2], o0[3]);
      *reinterpret_cast<uint4*>(st + (c0 + 1) * 128 + ((q8 ^ ((c0 + 1) & 7)) << 4)) =
          make_uint4(o1[0], o1[1], o1[2], o1[3]);
      fence_proxy_async_smem();
      if (!col_sync()) break;  // (red is free again too)
      if (lane == 0) {
        if (warp == 0) {
          tma_store_2d(&tmQT, st, static_cast<int32_t>(mb * 128), static_cast<int32_t>(nb * 128));
          tma_store_commit();
          tma_store_wait_read();  // the stage may be refilled once the store has read it
          stored = true;
        }
        mbar_arrive(empty + b);
      }
    }
  }
  if (stored && lane == 0) tma_store_wait_all();
}

// ---------------------------------------------------------------------------
// SwiGLU backward with both groupings of [d_gate | d_up] (f1), on the tile layout: a
// stage holds the 128 x 128 gate and up boxes of one tile (64 KB, two stages); dh comes
// straight from HBM into registers, the next tile's while this one is quantized. All
// sixteen consumer warps first form eight rows each (lane l: row 8w + l / 4, the four
// 8-column chunks (l % 4) + 4k, rotated by the row so that no two lanes of a shared-
// memory phase meet in a bank), with silu and ds from a per-CTA table of every BF16
// gate in range, write d_gate over the gate box and d_up over the up box, take the row
// maxima by two shuffles and store their rows' codes (and the BF16 gradient) from
// registers: four lanes cover a row's 128 codes, so every store fills whole sectors.
// Once all rows are formed, warps 0-7 quantize d_gate's columns and warps 8-15 d_up's,
// as the column warps of a6_tile_kernel do, staging the transposed codes over the first
// half of the box they read (each group meets on its own bounded barrier after its
// reads). Warp 16 is the producer.
// ---------------------------------------------------------------------------
constexpr int kSbStages = 2;
constexpr uint32_t kSbStageBytes = 2 * kA6Tile;                // gate and up boxes
constexpr uint32_t kSbOffGate = kSbStages * kSbStageBytes;     // (silu, ds) per gate
constexpr uint32_t kSbOffRed = kSbOffGate + kSgEntries * 8;    // [2 outputs][4][64] maxima
constexpr uint32_t kSbOffTab = kSbOffRed + 2 * 4 * 64 * 4;     // scale and reciprocal tables
constexpr uint32_t kSbOffBar = kSbOffTab + 256 * 4;            // full, empty, formed, csync[2]
constexpr size_t kSbSmem = 1024 + kSbOffBar + (3 * kSbStages + 2) * 8 + 16;

__global__ void __launch_bounds__(kA6Threads, 1) swiglu_bwd_tile_kernel(
    const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmU,
    const __grid_constant__ CUtensorMap tmQT, const uint16_t* __restrict__ dh,
    uint16_t* __restrict__ dgu, uint8_t* __restrict__ q_row, int64_t M, int64_t I,
    float* __restrict__ s_row, int64_t lds_row, float* __restrict__ s_col, unsigned* err,
    uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const float2* gtab = reinterpret_cast<const float2*>(base + kSbOffGate);
  float* tab = reinterpret_cast<float*>(base + kSbOffTab);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kSbOffBar);
  uint64_t* empty = full + kSbStages;
  uint64_t* formed = empty + kSbStages;  // all sixteen warps have formed their rows
  uint64_t* csync = formed + kSbStages;  // [2]: each column group's rendezvous
  int* abort_flag = reinterpret_cast<int*>(csync + 2);
  const WaitCtl ctl{abort_flag, err, limit_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 128) {
    tab[threadIdx.x] = kScaleMant[threadIdx.x];
    tab[128 + threadIdx.x] = kRecipMant[threadIdx.x];
  }
  sgb_table_fill(reinterpret_cast<float2*>(base + kSbOffGate));
  if (threadIdx.x == 0) {
    for (int b = 0; b < kSbStages; ++b) {
      mbar_init(full + b, 1);
      mbar_init(empty + b, 16);
      mbar_init(formed + b, 16);
    }
    mbar_init(csync, 8);
    mbar_init(csync + 1, 8);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t NB = I >> 7;
  const int64_t tiles = (M >> 7) * NB;
  if (warp == 16) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0, par = 0;
      bool ok = true;
      int i = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
        const int b = i % kSbStages;
        const uint32_t ph = static_cast<uint32_t>(i / kSbStages) & 1u;
        if (i >= kSbStages && !mbar_wait(empty + b, ph ^ 1u, ctl)) { ok = false; break; }
        const int64_t mb = t / NB, nb = t - mb * NB;
        const int32_t x = static_cast<int32_t>(nb * 128), y = static_cast<int32_t>(mb * 128);
        uint8_t* st = base + b * kSbStageBytes;
        mbar_arrive_expect_tx(full + b, kSbStageBytes);
        tma_load_2d(st, &tmG, x, y, full + b);
        tma_load_2d(st + kA6Tile, &tmU, x, y, full + b);
        issued |= 1u << b;
        par = (par & ~(1u << b)) | (ph << b);
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        for (int b = 0; b < kSbStages; ++b) {
          if (!((issued >> b) & 1u)) continue;
          const uint32_t a = smem_u32(full + b);
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(a, (par >> b) & 1u))
            if (global_timer_ns() - t0 > limit_ns) break;
        }
      }
    }
    return;
  }
  // row phase: tile row r = 8 warp + lr, chunks (a + 4k + 4 (lr % 4)) % 16, k = 0 .. 3
  const int lr = lane >> 2, a = lane & 3;
  const int r = warp * 8 + lr;
  // column phase: output grp, row quarter q4, column pair c0, c0 + 1
  const int grp = warp >> 3, cw = warp & 7, q4 = cw & 3;
  const int c0 = 64 * (cw >> 2) + 2 * lane;
  uint32_t* red = reinterpret_cast<uint32_t*>(base + kSbOffRed) + grp * 256;
  uint32_t nsync = 0;
  auto col_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(csync + grp);
    return mbar_wait_warp(csync + grp, (nsync++) & 1u, ctl);
  };
  auto chunk = [&](int k) { return (a + 4 * k + 4 * (lr & 3)) & 15; };
  // this lane's dh chunks of tile t
  uint4 dcur[4];
  auto load_dh = [&](int64_t t) {
    const int64_t mb = t / NB, nb = t - mb * NB;
    const uint16_t* row = dh + (mb * 128 + r) * I + nb * 128;
#pragma unroll
    for (int k = 0; k < 4; ++k) dcur[k] = ld_nc_v4(row + chunk(k) * 8);
  };
  if (static_cast<int64_t>(blockIdx.x) < tiles) load_dh(blockIdx.x);
  bool stored = false;
  int i = 0;
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
    const int b = i % kSbStages;
    const uint32_t ph = static_cast<uint32_t>(i / kSbStages) & 1u;
    if (!mbar_wait_warp(full + b, ph, ctl)) break;
    const int64_t mb = t / NB, nb = t - mb * NB;
    uint8_t* st = base + b * kSbStageBytes;
    // ---------------------------------------------------------------- rows
    {
      uint16_t* rg = reinterpret_cast<uint16_t*>(st) + r * 128;
      uint16_t* ru = reinterpret_cast<uint16_t*>(st + kA6Tile) + r * 128;
      uint32_t ma[4] = {0u, 0u, 0u, 0u}, mu[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int off = chunk(k) * 8;
        float v[2][8];
        swiglu_bwd8_tab(*reinterpret_cast<const uint4*>(rg + off),
                        *reinterpret_cast<const uint4*>(ru + off), dcur[k], gtab, v);
        const uint4 dg = make_uint4(pack_bf16x2(v[0][0], v[0][1]), pack_bf16x2(v[0][2], v[0][3]),
                                    pack_bf16x2(v[0][4], v[0][5]), pack_bf16x2(v[0][6], v[0][7]));
        const uint4 du = make_uint4(pack_bf16x2(v[1][0], v[1][1]), pack_bf16x2(v[1][2], v[1][3]),
                                    pack_bf16x2(v[1][4], v[1][5]), pack_bf16x2(v[1][6], v[1][7]));
        *reinterpret_cast<uint4*>(rg + off) = dg;
        *reinterpret_cast<uint4*>(ru + off) = du;
        ma[0] = bf16x2_maxabs_xs(ma[0], dg.x);
        ma[1] = bf16x2_maxabs_xs(ma[1], dg.y);
        ma[2] = bf16x2_maxabs_xs(ma[2], dg.z);
        ma[3] = bf16x2_maxabs_xs(ma[3], dg.w);
        mu[0] = bf16x2_maxabs_xs(mu[0], du.x);
        mu[1] = bf16x2_maxabs_xs(mu[1], du.y);
        mu[2] = bf16x2_maxabs_xs(mu[2], du.z);
        mu[3] = bf16x2_maxabs_xs(mu[3], du.w);
      }
      // the next tile's dh while this one is quantized
      if (t + gridDim.x < tiles) load_dh(t + gridDim.x);
      // the row's four lanes are adjacent: two shuffles give its maximum
      uint32_t hg = bf16x2_maxabs_xs(bf16x2_maxabs_xs(ma[0], ma[1]), bf16x2_maxabs_xs(ma[2], ma[3]));
      uint32_t hu = bf16x2_maxabs_xs(bf16x2_maxabs_xs(mu[0], mu[1]), bf16x2_maxabs_xs(mu[2], mu[3]));
      hg = bf16x2_maxabs_xs(hg, __shfl_xor_sync(kFull, hg, 1));
      hu = bf16x2_maxabs_xs(hu, __shfl_xor_sync(kFull, hu, 1));
      hg = bf16x2_maxabs_xs(hg, __shfl_xor_sync(kFull, hg, 2));
      hu = bf16x2_maxabs_xs(hu, __shfl_xor_sync(kFull, hu, 2));
      const GroupScale g0 = group_scale_bf16_sm(bf16x2_hmax_abs(hg), tab);
      const GroupScale g1 = group_scale_bf16_sm(bf16x2_hmax_abs(hu), tab);
      const int64_t m = mb * 128 + r;
      uint8_t* qr = q_row + m * 2 * I + nb * 128;
      uint16_t* br = dgu ? dgu + m * 2 * I + nb * 128 : nullptr;
      const bool small = __any_sync(kFull, g0.small || g1.small);
      // the codes from the formed values (this lane's own writes) before the rows are
      // released: the column groups stage their codes over these boxes afterwards
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = chunk(k) * 8;
        const uint4 dg = *reinterpret_cast<const uint4*>(rg + c);
        const uint4 du = *reinterpret_cast<const uint4*>(ru + c);
        uint2 q0, q1;
        if (small) {
          q0 = codes8_words<true>(dg, g0);
          q1 = codes8_words<true>(du, g1);
        } else {
          q0 = codes8_words<false>(dg, g0);
          q1 = codes8_words<false>(du, g1);
        }
        *reinterpret_cast<uint2*>(qr + c) = q0;
        *reinterpret_cast<uint2*>(qr + I + c) = q1;
        if (br) {
          *reinterpret_cast<uint4*>(br + c) = dg;
          *reinterpret_cast<uint4*>(br + I + c) = du;
        }
      }
      if (a == 0) {
        s_row[nb * lds_row + m] = g0.s;
        s_row[(NB + nb) * lds_row + m] = g1.s;
      }
      fence_proxy_async_smem();  // the stage is refilled by tensor copies later
      __syncwarp();
      if (lane == 0) mbar_arrive(formed + b);  // release: the column warps may read the rows
    }
    if (!mbar_wait_warp(formed + b, ph, ctl)) break;
    // ---------------------------------------------------------------- columns of output grp
    {
      uint8_t* box = st + grp * kA6Tile;
      const uint32_t* tw = reinterpret_cast<const uint32_t*>(box) + q4 * 32 * 64 + (c0 >> 1);
      uint32_t w[32];  // columns c0, c0 + 1 of rows 32 q4 + k
#pragma unroll
      for (int k = 0; k < 32; ++k) w[k] = tw[k * 64];
      uint32_t m0 = 0u, m1 = 0u;
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        m0 = bf16x2_maxabs_xs(m0, w[k]);
        m1 = bf16x2_maxabs_xs(m1, w[k + 1]);
      }
      red[q4 * 64 + (c0 >> 1)] = bf16x2_maxabs_xs(m0, m1);
      if (stored && cw == 0 && lane == 0) tma_store_wait_read();  // (earlier stages' stores)
      if (!col_sync()) break;  // the group's reads of the box are done: it may be overwritten
      uint32_t mm = 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) mm = bf16x2_maxabs_xs(mm, red[q * 64 + (c0 >> 1)]);
      const GroupScale g0 = group_scale_bf16_sm(fabsf(bf16_lo(mm)), tab);
      const GroupScale g1 = group_scale_bf16_sm(fabsf(bf16_hi(mm)), tab);
      if (q4 == 0)
        *reinterpret_cast<float2*>(s_col + mb * 2 * I + grp * I + nb * 128 + c0) =
            make_float2(g0.s, g1.s);
      uint32_t o0[8], o1[8];
      if (__any_sync(kFull, g0.small || g1.small))
        col_codes<true, 32>(w, g0, g1, o0, o1);
      else
        col_codes<false, 32>(w, g0, g1, o0, o1);
      // staging (first 16 KB of the box): row c holds column c's 128 codes, 16-byte chunk
      // k at position k ^ (c & 7) (the 128-byte swizzle)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = c0 + e;
        const uint32_t* oc = e ? o1 : o0;
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int k = 2 * q4 + k2;
          *reinterpret_cast<uint4*>(box + c * 128 + ((k ^ (c & 7)) << 4)) =
              make_uint4(oc[4 * k2], oc[4 * k2 + 1], oc[4 * k2 + 2], oc[4 * k2 + 3]);
        }
      }
      fence_proxy_async_smem();
      if (!col_sync()) break;
      if (lane == 0) {
        if (cw == 0) {
          tma_store_2d(&tmQT, box, static_cast<int32_t>(mb * 128),
                       static_cast<int32_t>(grp * I + nb * 128));
          tma_store_commit();
          tma_store_wait_read();  // the stage may be refilled once the store has read it
          stored = true;
        }
        mbar_arrive(empty + b);
      }
    }
  }
  if (stored && lane == 0) tma_store_wait_all();
}

// dgamma_j = the exact sum over rows of fl32(dy_mj * fl32(x_mj * r_m)), rounded once to
// fp32. A warp takes a strip of 32 8-column chunks (one per lane) over kDgRows rows, keeps
// each of its 8 columns as an exact sum, and adds each column's bins into the global
// bins [H][kXBins] with 64-bit integer atomics: integer additions, so the order in which
// the warps land does not matter.
#ifndef DG_ROWS
#define DG_ROWS 64
#define DG_BATCH 4
#endif
constexpr int kDgRows = DG_ROWS;
constexpr int kDgBatch = DG_BATCH;  // rows whose loads are in flight together

__global__ void __launch_bounds__(256, 2) dgamma_exact_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ dy, const float* __restrict__ r,
    int64_t M, int64_t H, unsigned long long* __restrict__ bins) {
  const int lane = threadIdx.x & 31;
  const int64_t nch = H >> 3;
  const int64_t strips = (nch + 31) / 32;
  const int64_t rblocks = (M + kDgRows - 1) / kDgRows;
  const int64_t wglobal = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t u = wglobal; u < strips * rblocks; u += nw) {
    const int64_t ch = (u % strips) * 32 + lane;
    const int64_t m0 = (u / strips) * kDgRows;
    const int64_t m1 = m0 + kDgRows < M ? m0 + kDgRows : M;
    if (ch >= nch) continue;  // lanes past the last chunk (H not a multiple of 256)
    unsigned long long* col = bins + ch * 8 * kXBins;  // this lane's 8 columns' bins
    XPair acc[8];
    int64_t m = m0;
    // kDgBatch rows' loads in flight before their terms are added
    for (; m + kDgBatch <= m1; m += kDgBatch) {
      uint4 xr[kDgBatch], dr[kDgBatch];
      float rm[kDgBatch];
#pragma unroll
      for (int e = 0; e < kDgBatch; ++e) {
        xr[e] = ld_nc_v4(x + (m + e) * H + ch * 8);
        dr[e] = ld_nc_v4(dy + (m + e) * H + ch * 8);
        rm[e] = __ldg(r + m + e);
      }
#pragma unroll
      for (int e = 0; e < kDgBatch; ++e) {
        float xv[8], dv[8];
        unpack_bf16x8(xr[e], xv);
        unpack_bf16x8(dr[e], dv);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          acc[q].add(__fmul_rn(dv[q], __fmul_rn(xv[q], rm[e])), [&](int b, long long v) {
            atomicAdd(col + q * kXBins + b, static_cast<unsigned long long>(v));
          });
      }
    }
    for (; m < m1; ++m) {
      float xv[8], dv[8];
      unpack_bf16x8(ld_nc_v4(x + m * H + ch * 8), xv);
      unpack_bf16x8(ld_nc_v4(dy + m * H + ch * 8), dv);
      const float rm = __ldg(r + m);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        acc[q].add(__fmul_rn(dv[q], __fmul_rn(xv[q], rm)), [&](int b, long long v) {
          atomicAdd(col + q * kXBins + b, static_cast<unsigned long long>(v));
        });
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (acc[q].b0 >= 0 && acc[q].a0 != 0.0)
        atomicAdd(col + q * kXBins + acc[q].b0,
                  static_cast<unsigned long long>(XPair::units(acc[q].a0, acc[q].b0)));
      if (acc[q].b1 >= 0 && acc[q].a1 != 0.0)
        atomicAdd(col + q * kXBins + acc[q].b1,
                  static_cast<unsigned long long>(XPair::units(acc[q].a1, acc[q].b1)));
    }
  }
}

// dgamma from the bins (two's complement in the unsigned words), one thread per column.
__global__ void __launch_bounds__(256) dgamma_round_kernel(const unsigned long long* __restrict__ bins,
                                                           int64_t H, float* __restrict__ dgamma) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= H) return;
  long long A[kXBins];
#pragma unroll
  for (int b = 0; b < kXBins; ++b) A[b] = static_cast<long long>(bins[j * kXBins + b]);
  dgamma[j] = __double2float_rn(xbins_round(A, true));
}

// a8: saved FP8 activation tiles (1x128 groups) -> xhat = fl32(s * dec(q)) -> 128x1
// groups along M, stored transposed; persistent over the (M/128) x (K/128) tiles.
// Each buffer holds the 16 KB code tile and its 128 row scales. xhat is an arbitrary
// fp32 value here (not a BF16 one), so the quotient must be the IEEE quotient itself:
// quot's q + (x - q s) y with y = fl32(1/s) and q = fl32(x y) is fl32(x / s) for every
// x and s of fp32 without underflow (Markstein's theorem: y within half an ulp of 1/s,
// q within one ulp of x/s, the residual exact by the FMA). Scales below 2^-80 divide.
__global__ void __launch_bounds__(256) transpose_quant_fp8_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS, int64_t M,
    int64_t K, uint8_t* __restrict__ qT, float* __restrict__ sT, unsigned* err,
    uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  const TileSmem sm = carve_tiles(smem_raw, kTileElems + 512);
  __shared__ int abort_flag;
  const WaitCtl ctl{&abort_flag, err, limit_ns};
  if (threadIdx.x == 0) abort_flag = 0;
  const int64_t KB = (K + 127) >> 7;
  const int64_t tiles = ((M + 127) >> 7) * KB;
  const int tid = threadIdx.x;
  auto issue = [&](int b, int64_t t) {
    const int32_t mx = static_cast<int32_t>((t / KB) * 128), kx = static_cast<int32_t>(t % KB);
    mbar_arrive_expect_tx(sm.bar + b, kTileElems + 512);
    tma_load_2d(sm.buf[b], &tmQ, kx * 128, mx, sm.bar + b);
    tma_load_2d(sm.buf[b] + kTileElems, &tmS, mx, kx, sm.bar + b);
  };
  tiles_prologue(sm, tiles, issue);
  const int cp = tid & 63, rq = tid >> 6;
  int i = 0;
  int64_t t = blockIdx.x;
  for (; t < tiles; t += gridDim.x, ++i) {
    if (!tile_acquire(sm, i & 1, (i >> 1) & 1, ctl)) break;
    tiles_refill(t, tiles, i, issue);
    const uint8_t* Tq = sm.buf[i & 1];
    const float* rsc = reinterpret_cast<const float*>(Tq + kTileElems);
    const int64_t mb = t / KB, kb = t % KB;
    float x0[32], x1[32];
#pragma unroll
    for (int r4 = 0; r4 < 32; r4 += 4) {
      const float4 sr4 = *reinterpret_cast<const float4*>(rsc + 32 * rq + r4);  // broadcast
      const float sr[4] = {sr4.x, sr4.y, sr4.z, sr4.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = r4 + k;
        const uint16_t two = *reinterpret_cast<const uint16_t*>(Tq + (32 * rq + r) * 128 + 2 * cp);
        const float2 d = e4m3x2_to_f32(two);
        x0[r] = __fmul_rn(sr[k], d.x);
        x1[r] = __fmul_rn(sr[k], d.y);
      }
    }
    float c0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, c1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      c0[r & 3] = fmaxf(c0[r & 3], fabsf(x0[r]));
      c1[r & 3] = fmaxf(c1[r & 3], fabsf(x1[r]));
    }
    float a0 = fmaxf(fmaxf(c0[0], c0[1]), fmaxf(c0[2], c0[3]));
    float a1 = fmaxf(fmaxf(c1[0], c1[1]), fmaxf(c1[2], c1[3]));
    sm.red[rq * 128 + 2 * cp] = a0;
    sm.red[rq * 128 + 2 * cp + 1] = a1;
    __syncthreads();
    a0 = fmaxf(fmaxf(sm.red[2 * cp], sm.red[128 + 2 * cp]),
               fmaxf(sm.red[256 + 2 * cp], sm.red[384 + 2 * cp]));
    a1 = fmaxf(fmaxf(sm.red[2 * cp + 1], sm.red[128 + 2 * cp + 1]),
               fmaxf(sm.red[256 + 2 * cp + 1], sm.red[384 + 2 * cp + 1]));
    const GroupScale g0 = group_scale_fma(a0), g1 = group_scale_fma(a1);
    const float s0 = g0.s, s1 = g1.s;
    // a partial tile (ragged M or K) arrived zero-filled; store only its valid part
    const int rows = M - mb * 128 < 128 ? static_cast<int>(M - mb * 128) : 128;
    const bool col_ok = kb * 128 + 2 * cp < K;  // K is even: the pair is in or out
    if (rq == 0 && col_ok)
      *reinterpret_cast<float2*>(sT + mb * K + kb * 128 + 2 * cp) = make_float2(s0, s1);
    uint32_t o0[8], o1[8];
    if (__any_sync(kFull, g0.small || g1.small)) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float t0[4], t1[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          t0[e] = g0.small ? __fdiv_rn(x0[4 * k + e], g0.s) : quot(x0[4 * k + e], g0);
          t1[e] = g1.small ? __fdiv_rn(x1[4 * k + e], g1.s) : quot(x1[4 * k + e], g1);
        }
        o0[k] = cvt_e4m3x4(t0[0], t0[1], t0[2], t0[3]);
        o1[k] = cvt_e4m3x4(t1[0], t1[1], t1[2], t1[3]);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float t0[4], t1[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) quot2(x0[4 * k + e], x1[4 * k + e], g0, g1, t0[e], t1[e]);
        o0[k] = cvt_e4m3x4(t0[0], t0[1], t0[2], t0[3]);
        o1[k] = cvt_e4m3x4(t1[0], t1[1], t1[2], t1[3]);
      }
    }
    uint8_t* dst = qT + (kb * 128) * M + mb * 128;
    uint4* d0 = reinterpret_cast<uint4*>(dst + (2 * cp) * M + 32 * rq);
    uint4* d1 = reinterpret_cast<uint4*>(dst + (2 * cp + 1) * M + 32 * rq);
    if (col_ok && 32 * rq < rows) {  // rows is a multiple of 16
      d0[0] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
      d1[0] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
    }
    if (col_ok && 32 * rq + 16 < rows) {
      d0[1] = make_uint4(o0[4], o0[5], o0[6], o0[7]);
      d1[1] = make_uint4(o1[4], o1[5], o1[6], o1[7]);
    }
  }
  if (t < tiles) tiles_drain(sm, t, tiles, i, limit_ns);
}

// a2 on a tile ring. The block scale is shared by a block and its transpose, so qT is the
// byte transpose of q: the codes are formed once, staged in shared memory, and leave twice
// by tensor stores, the second time after an in-register 8x8 byte transpose.
//   warps 0-7  thread t: rows t/16 + 16j (j < 8), columns 8(t%16) .. +7 of the tile (a
//              half-warp reads one 256-byte row); the warps' maxima meet in shared memory
//              (bounded rendezvous), every thread forms the block scale and its codes and
//              stores them in the q staging tile; then thread t transposes the 8x8 code
//              block (row block t%16, column block (t%16 + t/16) % 16) into the qT staging
//              tile. Both staging tiles use the 128-byte swizzle, which with this diagonal
//              assignment keeps the 8-byte reads and writes free of bank conflicts.
//   warp 8     producer: tiles into a ring of kA2Stages buffers.
// A partial block at the end of a ragged N or K arrives zero-filled (zeros raise no
// maximum) and the tensor stores write only its valid part.
#ifndef A2_STAGES
#define A2_STAGES 4
#endif
constexpr int kA2Stages = A2_STAGES;
constexpr uint32_t kA2Tile = 128 * 128 * 2;
constexpr uint32_t kA2OffQ = kA2Stages * kA2Tile;     // q staging, 16 KB
constexpr uint32_t kA2OffQT = kA2OffQ + 128 * 128;    // qT staging, 16 KB
constexpr uint32_t kA2OffRed = kA2OffQT + 128 * 128;  // [8] warp maxima
constexpr uint32_t kA2OffTab = kA2OffRed + 64;        // scale and reciprocal tables
constexpr uint32_t kA2OffBar = kA2OffTab + 256 * 4;   // full[], empty[], csync
constexpr size_t kA2Smem = 1024 + kA2OffBar + (2 * kA2Stages + 1) * 8 + 16;
constexpr int kA2Threads = 9 * 32;

// 4x4 byte transpose: word i holds row i (byte k = column k); returns word k = column k.
__device__ __forceinline__ void transpose_4x4_bytes(uint32_t& a, uint32_t& b, uint32_t& c,
                                                    uint32_t& d) {
  const uint32_t t0 = __byte_perm(a, b, 0x5140), t1 = __byte_perm(a, b, 0x7362);
  const uint32_t t2 = __byte_perm(c, d, 0x5140), t3 = __byte_perm(c, d, 0x7362);
  a = __byte_perm(t0, t2, 0x5410);
  b = __byte_perm(t0, t2, 0x7632);
  c = __byte_perm(t1, t3, 0x5410);
  d = __byte_perm(t1, t3, 0x7632);
}

// Byte offset of (row r, byte column c) in a [128][128]-byte tile with the 128-byte
// swizzle (16-byte chunk index XOR row % 8), the layout a swizzled tensor store reads.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((((c >> 4) ^ r) & 7) << 4) + (c & 15));
}

__global__ void __launch_bounds__(kA2Threads, 1) a2_tile_kernel(
    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmQ,
    const __grid_constant__ CUtensorMap tmQT, int64_t N, int64_t K, float* __restrict__ s,
    bool want_t, unsigned* err, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* red = reinterpret_cast<float*>(base + kA2OffRed);
  float* tab = reinterpret_cast<float*>(base + kA2OffTab);
  uint8_t* qs = base + kA2OffQ;
  uint8_t* qts = base + kA2OffQT;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kA2OffBar);
  uint64_t* empty = full + kA2Stages;
  uint64_t* csync = empty + kA2Stages;  // the compute warps' rendezvous (bounded)
  int* abort_flag = reinterpret_cast<int*>(csync + 1);
  const WaitCtl ctl{abort_flag, err, limit_ns};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid < 128) {
    tab[tid] = kScaleMant[tid];
    tab[128 + tid] = kRecipMant[tid];
  }
  if (tid == 0) {
    for (int b = 0; b < kA2Stages; ++b) {
      mbar_init(full + b, 1);
      mbar_init(empty + b, 8);
    }
    mbar_init(csync, 8);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t KB = (K + 127) >> 7;
  const int64_t tiles = ((N + 127) >> 7) * KB;
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0, par = 0;
      bool ok = true;
      int i = 0;
      for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
        const int b = i % kA2Stages;
        const uint32_t ph = static_cast<uint32_t>(i / kA2Stages) & 1u;
        if (i >= kA2Stages && !mbar_wait(empty + b, ph ^ 1u, ctl)) { ok = false; break; }
        const int64_t nb = t / KB, kb = t - nb * KB;
        mbar_arrive_expect_tx(full + b, kA2Tile);
        tma_load_2d(base + b * kA2Tile, &tmW, static_cast<int32_t>(kb * 128),
                    static_cast<int32_t>(nb * 128), full + b);
        issued |= 1u << b;
        par = (par & ~(1u << b)) | (ph << b);
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        for (int b = 0; b < kA2Stages; ++b) {
          if (!((issued >> b) & 1u)) continue;
          const uint32_t a = smem_u32(full + b);
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(a, (par >> b) & 1u))
            if (global_timer_ns() - t0 > limit_ns) break;
        }
      }
    }
    return;
  }
  uint32_t nsync = 0;
  auto sync8 = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(csync);
    return mbar_wait_warp(csync, (nsync++) & 1u, ctl);
  };
  const int rr = tid >> 4, c8 = (tid & 15) * 8;
  const int tbr = tid & 15, tbc = ((tid & 15) + (tid >> 4)) & 15;  // transposed 8x8 block
  bool stored = false;
  int i = 0;
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
    const int b = i % kA2Stages;
    if (!mbar_wait_warp(full + b, static_cast<uint32_t>(i / kA2Stages) & 1u, ctl)) break;
    const uint16_t* Ts = reinterpret_cast<const uint16_t*>(base + b * kA2Tile);
    uint4 raw[8];
    uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      raw[j] = *reinterpret_cast<const uint4*>(Ts + (rr + 16 * j) * 128 + c8);
      m[0] = bf16x2_maxabs_xs(m[0], raw[j].x);
      m[1] = bf16x2_maxabs_xs(m[1], raw[j].y);
      m[2] = bf16x2_maxabs_xs(m[2], raw[j].z);
      m[3] = bf16x2_maxabs_xs(m[3], raw[j].w);
    }
    float a = bf16x2_hmax_abs(bf16x2_maxabs_xs(bf16x2_maxabs_xs(m[0], m[1]), bf16x2_maxabs_xs(m[2], m[3])));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, off));
    if (lane == 0) {
      red[warp] = a;
      mbar_arrive(empty + b);  // the lanes' reads of the tile are complete (values used)
    }
    if (stored && tid == 0) tma_store_wait_read();  // both staging tiles are free
    if (!sync8()) break;
    float amax = red[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) amax = fmaxf(amax, red[k]);
    const GroupScale g = group_scale_bf16_sm(amax, tab);
    const int64_t nb = t / KB, kb = t - nb * KB;
    if (tid == 0) s[nb * KB + kb] = g.s;
    if (g.small) {  // uniform over the CTA
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint2*>(qs + sw128(rr + 16 * j, c8)) = codes8_words<true>(raw[j], g);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint2*>(qs + sw128(rr + 16 * j, c8)) = codes8_words<false>(raw[j], g);
    }
    fence_proxy_async_smem();
    if (!sync8()) break;
    if (tid == 0) {
      tma_store_2d(&tmQ, qs, static_cast<int32_t>(kb * 128), static_cast<int32_t>(nb * 128));
      tma_store_commit();
    }
    if (want_t) {
      // rows 8 tbr .. +7, bytes 8 tbc .. +7 of q  ->  rows 8 tbc .. +7, bytes 8 tbr .. +7 of qT
      uint32_t lo[8], hi[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const uint2 v = *reinterpret_cast<const uint2*>(qs + sw128(8 * tbr + r, 8 * tbc));
        lo[r] = v.x;
        hi[r] = v.y;
      }
      transpose_4x4_bytes(lo[0], lo[1], lo[2], lo[3]);
      transpose_4x4_bytes(lo[4], lo[5], lo[6], lo[7]);
      transpose_4x4_bytes(hi[0], hi[1], hi[2], hi[3]);
      transpose_4x4_bytes(hi[4], hi[5], hi[6], hi[7]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        *reinterpret_cast<uint2*>(qts + sw128(8 * tbc + c, 8 * tbr)) = make_uint2(lo[c], lo[4 + c]);
        *reinterpret_cast<uint2*>(qts + sw128(8 * tbc + 4 + c, 8 * tbr)) = make_uint2(hi[c], hi[4 + c]);
      }
      fence_proxy_async_smem();
      if (!sync8()) break;
      if (tid == 0) {
        tma_store_2d(&tmQT, qts, static_cast<int32_t>(nb * 128), static_cast<int32_t>(kb * 128));
        tma_store_commit();
      }
    }
    stored = true;
  }
  if (stored && tid == 0) tma_store_wait_all();
}

// Resident CTAs per SM of a kernel (cached per device), for grid-stride/persistent grids.
template <class Kernel>
// `cache` is a per-device table owned by the caller; host threads may race to fill an
// entry (with the same value), so entries are atomics.
int resident_ctas(Kernel k, int threads, size_t dyn_smem, std::atomic<int>* cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  if (const int known = cache[dev].load(std::memory_order_acquire)) return known;
  if (dyn_smem > 48 * 1024)
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn_smem));
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, dyn_smem) != cudaSuccess || n < 1)
    n = 1;
  cudaGetLastError();
  cache[dev].store(n, std::memory_order_release);
  return n;
}

// Opt a kernel in to the largest dynamic shared memory of an sm_100 CTA, once per device.
// `done` is a per-device table owned by the caller, one per kernel (kernels of the same
// signature share a function-pointer type, so a table inside this template would be
// shared between them).
constexpr size_t kMaxDynSmem = 232448;
// Tensor-copy coordinates are signed 32-bit: the kernels fed by them take extents below this.
constexpr int64_t kMaxTmaCoord = int64_t{1} << 31;
template <class Kernel>
bool allow_max_smem(Kernel k, std::atomic<int>* done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (done[dev].load(std::memory_order_acquire)) return true;
  const cudaError_t e =
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kMaxDynSmem));
  if (e != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(max dynamic smem)", e);
    cudaGetLastError();
    return false;
  }
  done[dev].store(1, std::memory_order_release);
  return true;
}

int grid_for(int64_t ctas_needed, int per_sm) {
  const int64_t cap = static_cast<int64_t>(sm100_sm_count()) * per_sm;
  const int64_t g = ctas_needed < cap ? ctas_needed : cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" fp8q_status fp8q_quant_act_1x128(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                            uint8_t* q, float* s, int64_t lds, void* stream) {
  if (!x || !q || !s) return FP8Q_ERR_NULL;
  if (M <= 0 || K <= 0 || K % 16 || ldx < K || lds < M || lds % 4) return FP8Q_ERR_SHAPE;
  if (M >= kMaxTmaCoord || K >= kMaxTmaCoord) return FP8Q_ERR_SHAPE;  // 32-bit tensor coordinates
  if (!aligned16(x) || !aligned16(q) || !aligned16(s) || ldx % 8) return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  const int64_t G = (K + 127) / 128;
  const int64_t units = ((M + kLgRows - 1) / kLgRows) * G;
  if (units >= (int64_t{1} << 31)) return FP8Q_ERR_SHAPE;
  CUtensorMap tm, tmq;
  if (!encode_tmap_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, ldx * 2, 128, kLgRows,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, M, K, 128, kLgRows,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
    return FP8Q_ERR_UNSUPPORTED;
  unsigned* err = device_error_word();
  if (!err) return FP8Q_ERR_CUDA;
  constexpr int kPer = LG1_PER, kConsumers = LG1_CONS;
  auto kern = lanegroup_kernel<ActLane, kPer, kConsumers>;
  constexpr size_t smem = lanegroup_smem<ActLane, kPer, kConsumers>();
  static std::atomic<int> occ[64];
  const int per_sm = resident_ctas(kern, lg_threads<kConsumers>(), smem, occ);
  kern<<<grid_for((units + kConsumers - 1) / kConsumers, per_sm), lg_threads<kConsumers>(), smem,
         static_cast<cudaStream_t>(stream)>>>(tm, tm, tmq, M, G, s, lds, err, kWaitLimitNs);
  return launch_status("quant_act_1x128 launch");
}

extern "C" fp8q_status fp8q_swiglu_quant(const uint16_t* gu, int64_t M, int64_t I, int64_t ldgu,
                                         uint8_t* q, float* s, int64_t lds, void* stream) {
  if (!gu || !q || !s) return FP8Q_ERR_NULL;
  if (M <= 0 || I <= 0 || I % 16 || ldgu < 2 * I || lds < M || lds % 4) return FP8Q_ERR_SHAPE;
  if (!aligned16(gu) || !aligned16(q) || !aligned16(s) || ldgu % 8) return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  const int64_t G = (I + 127) / 128;
  if (((M + kRgRows - 1) / kRgRows) * G >= (int64_t{1} << 31)) return FP8Q_ERR_SHAPE;
  // the gate and the up halves as two [M][I] tensors, so that a partial last group of
  // the gate reads zeros, not the first up columns
  CUtensorMap tmG, tmU;
  if (!encode_tmap_2d(&tmG, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gu, I, M, ldgu * 2, 128, kRgRows,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmU, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gu + I, I, M, ldgu * 2, 128, kRgRows,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
    return FP8Q_ERR_UNSUPPORTED;
  unsigned* err = device_error_word();
  if (!err) return FP8Q_ERR_CUDA;
  constexpr int kStages = A4_STAGES, kConsumers = A4_CONS;
  auto kern = rowgroup_tma_kernel<SwigluBoxes, kStages, kConsumers>;
  constexpr size_t smem = rowgroup_tma_smem<SwigluBoxes, kStages>();
  static std::atomic<int> occ[64];
  const int per_sm = resident_ctas(kern, rg_threads<kConsumers>(), smem, occ);
  kern<<<grid_for(((M + kRgRows - 1) / kRgRows) * G, per_sm), rg_threads<kConsumers>(), smem,
         static_cast<cudaStream_t>(stream)>>>(tmG, tmU, M, G, I, q, I, s, lds, err, kWaitLimitNs);
  return launch_status("swiglu_quant launch");
}

namespace fp8q {
namespace {
// a3 through rmsnorm_lane_kernel<kConsumers> with `per` row stages per warp as the shared
// memory allows; FP8Q_ERR_SHAPE (nothing launched) when not even one stage per warp fits.
template <int kConsumers>
fp8q_status launch_rmsnorm_lane(const uint16_t* x, const uint16_t* gamma, int64_t M, int64_t H,
                                int64_t ldx, float eps, uint8_t* q, float* s, int64_t lds,
                                int sms, cudaStream_t st) {
  const int G = static_cast<int>(H / 128);
  const size_t row_bytes = static_cast<size_t>(G) * 256;
  const size_t fixed = 1024 + row_bytes + kConsumers * (row_bytes / 2) + 16;
  if (fixed >= kMaxDynSmem) return FP8Q_ERR_SHAPE;
  const int per = static_cast<int>(
      std::min<size_t>(2, (kMaxDynSmem - fixed) / (kConsumers * (row_bytes + 16))));
  if (per < 1) return FP8Q_ERR_SHAPE;
  const int nst = per * kConsumers;
  const uint64_t dx[3] = {128, static_cast<uint64_t>(G), static_cast<uint64_t>(M)};
  const uint64_t sx[2] = {256, static_cast<uint64_t>(ldx) * 2};
  const uint64_t sq[2] = {128, static_cast<uint64_t>(H)};
  const uint32_t box[3] = {128, static_cast<uint32_t>(G), 1};
  CUtensorMap tmx, tmq;
  if (!encode_tmap_3d(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, dx, sx, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_3d(&tmq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, dx, sq, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
    return FP8Q_ERR_UNSUPPORTED;
  unsigned* err = device_error_word();
  if (!err) return FP8Q_ERR_CUDA;
  auto kern = rmsnorm_lane_kernel<kConsumers>;
  static std::atomic<int> smem_ok[64];  // per instantiation, so per kernel
  if (!allow_max_smem(kern, smem_ok)) return FP8Q_ERR_CUDA;
  const size_t smem = fixed + static_cast<size_t>(nst) * (row_bytes + 16);
  const int64_t ctas = (M + kConsumers - 1) / kConsumers;
  kern<<<static_cast<int>(ctas < sms ? ctas : sms), 32 * (kConsumers + 1), smem, st>>>(
      tmx, tmq, gamma, M, G, per, eps, s, lds, err, kWaitLimitNs);
  return launch_status("rmsnorm_quant launch");
}
}  // namespace
}  // namespace fp8q

extern "C" fp8q_status fp8q_rmsnorm_quant(const uint16_t* x, const uint16_t* gamma, int64_t M,
                                          int64_t H, int64_t ldx, float eps, uint8_t* q, float* s,
                                          int64_t lds, void* stream) {
  if (!x || !gamma || !q || !s) return FP8Q_ERR_NULL;
  if (M <= 0 || H <= 0 || H % 16 || H > 8 * kNormMaxChunks * kNormThreads || ldx < H ||
      lds < M || lds % 4 || !(eps >= 0.0f))
    return FP8Q_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(q) || !aligned16(s) || ldx % 8)
    return FP8Q_ERR_ALIGN;
  const int sms = sm100_sm_count();
  if (!sms) return FP8Q_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t gsm = static_cast<size_t>(H) * 2;  // gamma in shared memory
  // One warp per row needs many rows to fill the GPU; up to 1024 rows one CTA per row
  // is faster (measured 3x at 16-256 rows, equal at 8192).
  if (M > 1024 && M < kMaxTmaCoord && H % 128 == 0 && H <= 64 * 128) {
    // 16 consumer warps where their row stages fit in shared memory, else 8
    const fp8q_status r16 = launch_rmsnorm_lane<16>(x, gamma, M, H, ldx, eps, q, s, lds, sms, st);
    if (r16 != FP8Q_ERR_SHAPE) return r16;
    const fp8q_status r8 = launch_rmsnorm_lane<8>(x, gamma, M, H, ldx, eps, q, s, lds, sms, st);
    if (r8 != FP8Q_ERR_SHAPE) return r8;
  }
  if (M > 1024) {
    const int64_t ctas = (M + 7) / 8;  // one warp per row
    static std::atomic<int> occ[64];
    const int per_sm = resident_ctas(rmsnorm_quant_warp2_kernel, 256, gsm, occ);
    rmsnorm_quant_warp2_kernel<<<grid_for(ctas, per_sm), 256, gsm, st>>>(x, gamma, M, H, ldx, eps,
                                                                         q, s, lds);
  } else {
    const int64_t grid = M < static_cast<int64_t>(sms) * 64 ? M : static_cast<int64_t>(sms) * 64;
    rmsnorm_quant_cta_kernel<<<static_cast<int>(grid), kNormThreads, gsm, st>>>(x, gamma, M, H,
                                                                                ldx, eps, q, s, lds);
  }
  return launch_status("rmsnorm_quant launch");
}

extern "C" fp8q_status fp8q_quant_weight_128x128(const uint16_t* w, int64_t N, int64_t K,
                                                 int64_t ldw, uint8_t* q, float* s, uint8_t* qT,
                                                 void* stream) {
  if (!w || !q || !s) return FP8Q_ERR_NULL;
  if (N <= 0 || K <= 0 || N % 16 || K % 16 || ldw < K) return FP8Q_ERR_SHAPE;
  if (N >= kMaxTmaCoord || K >= kMaxTmaCoord) return FP8Q_ERR_SHAPE;  // 32-bit tensor coordinates
  if (!aligned16(w) || !aligned16(q) || !aligned16(s) || (qT && !aligned16(qT)) || ldw % 8)
    return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  CUtensorMap tm, tmq, tmqt;
  if (!encode_tmap_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, K, N, ldw * 2, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, N, K, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8Q_ERR_UNSUPPORTED;
  if (qT && !encode_tmap_2d(&tmqt, CU_TENSOR_MAP_DATA_TYPE_UINT8, qT, N, K, N, 128, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8Q_ERR_UNSUPPORTED;
  if (!qT) tmqt = tmq;  // unused
  unsigned* err = device_error_word();
  if (!err) return FP8Q_ERR_CUDA;
  static std::atomic<int> occ[64];
  const int per_sm = resident_ctas(a2_tile_kernel, kA2Threads, kA2Smem, occ);
  a2_tile_kernel<<<grid_for(((N + 127) / 128) * ((K + 127) / 128), per_sm), kA2Threads, kA2Smem,
                   static_cast<cudaStream_t>(stream)>>>(tm, tmq, tmqt, N, K, s, qT != nullptr, err,
                                                        kWaitLimitNs);
  return launch_status("quant_weight_128x128 launch");
}

extern "C" fp8q_status fp8q_transpose_quant_bf16(const uint16_t* dy, int64_t M, int64_t N,
                                                 int64_t lddy, uint8_t* q_row, float* s_row,
                                                 int64_t lds_row, uint8_t* q_colT, float* s_col,
                                                 void* stream) {
  if (!dy || !q_colT || !s_col || (q_row != nullptr) != (s_row != nullptr)) return FP8Q_ERR_NULL;
  if (M <= 0 || N <= 0 || M % 16 || N % 16 || lddy < N || (q_row && (lds_row < M || lds_row % 4)))
    return FP8Q_ERR_SHAPE;
  if (M >= kMaxTmaCoord || N >= kMaxTmaCoord) return FP8Q_ERR_SHAPE;  // 32-bit tensor coordinates
  if (!aligned16(dy) || !aligned16(q_colT) || !aligned16(s_col) || lddy % 8 ||
      (q_row && (!aligned16(q_row) || !aligned16(s_row))))
    return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  CUtensorMap tmd, tmq, tmqt;
  if (!encode_tmap_2d(&tmd, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dy, N, M, lddy * 2, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmqt, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_colT, M, N, M, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8Q_ERR_UNSUPPORTED;
  if (q_row && !encode_tmap_2d(&tmq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_row, N, M, N, 128, 16,
                               CU_TENSOR_MAP_SWIZZLE_NONE))
    return FP8Q_ERR_UNSUPPORTED;
  if (!q_row) tmq = tmqt;  // unused
  unsigned* err = device_error_word();
  if (!err) return FP8Q_ERR_CUDA;
  const int64_t tiles = ((M + 127) / 128) * ((N + 127) / 128);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  constexpr size_t kSmem = a6_smem<TileGrad>();
  if (q_row) {
    static std::atomic<int> occ[64];
    const int per_sm = resident_ctas(a6_tile_kernel<TileGrad, true>, kA6Threads, kSmem, occ);
    a6_tile_kernel<TileGrad, true><<<grid_for(tiles, per_sm), kA6Threads, kSmem, st>>>(
        tmd, tmd, tmq, tmqt, TileGrad{}, M, N, s_row, lds_row, s_col, err, kWaitLimitNs);
  } else {
    static std::atomic<int> occ[64];
    const int per_sm = resident_ctas(a6_tile_kernel<TileGrad, false>, kA6Threads, kSmem, occ);
    a6_tile_kernel<TileGrad, false><<<grid_for(tiles, per_sm), kA6Threads, kSmem, st>>>(
        tmd, tmd, tmq, tmqt, TileGrad{}, M, N, s_row, lds_row, s_col, err, kWaitLimitNs);
  }
  return launch_status("transpose_quant_bf16 launch");
}

extern "C" fp8q_status fp8q_transpose_quant_fp8(const uint8_t* q, const float* s, int64_t M,
                                                int64_t K, int64_t lds, uint8_t* qT, float* sT,
                                                void* stream) {
  if (!q || !s || !qT || !sT) return FP8Q_ERR_NULL;
  if (M <= 0 || K <= 0 || M % 16 || K % 16 || lds < M) return FP8Q_ERR_SHAPE;
  if (M >= kMaxTmaCoord || K >= kMaxTmaCoord) return FP8Q_ERR_SHAPE;  // 32-bit tensor coordinates
  if (!aligned16(q) || !aligned16(s) || !aligned16(qT) || !aligned16(sT) || lds % 4)
    return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  const int64_t KB = (K + 127) / 128;
  CUtensorMap tmq, tms;
  if (!encode_tmap_2d(&tmq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, M, K, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, s, M, KB, lds * 4, 128, 1,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
    return FP8Q_ERR_UNSUPPORTED;
  unsigned* err = device_error_word();
  if (!err) return FP8Q_ERR_CUDA;
  static std::atomic<int> occ[64];
  const int per_sm = resident_ctas(transpose_quant_fp8_kernel, 256, kTileSmemFP8, occ);
  transpose_quant_fp8_kernel<<<grid_for(((M + 127) / 128) * KB, per_sm), 256, kTileSmemFP8,
                               static_cast<cudaStream_t>(stream)>>>(tmq, tms, M, K, qT, sT, err,
                                                                    kWaitLimitNs);
  return launch_status("transpose_quant_fp8 launch");
}

extern "C" fp8q_status fp8q_rmsnorm_quant_dual(const uint16_t* x, const uint16_t* gamma,
                                               int64_t M, int64_t H, int64_t ldx, float eps,
                                               uint8_t* q_row, float* s_row, int64_t lds_row,
                                               uint8_t* q_colT, float* s_col, float* rstd,
                                               void* stream) {
  if (!x || !gamma || !q_row || !s_row || !q_colT || !s_col || !rstd) return FP8Q_ERR_NULL;
  if (M <= 0 || H <= 0 || M % 128 || H % 128 || ldx < H || lds_row < M || lds_row % 4 ||
      !(eps >= 0.0f))
    return FP8Q_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(q_row) || !aligned16(s_row) ||
      !aligned16(q_colT) || !aligned16(s_col) || !aligned16(rstd) || ldx % 8)
    return FP8Q_ERR_ALIGN;
  const int sms = sm100_sm_count();
  if (!sms) return FP8Q_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the reciprocal RMS of every row first (one warp per row), then the tiles
  const int64_t rstd_ctas = std::min<int64_t>((M + 7) / 8, static_cast<int64_t>(sms) * 8);
  if (M >= kMaxTmaCoord || H >= kMaxTmaCoord) return FP8Q_ERR_SHAPE;  // 32-bit coordinates
  CUtensorMap tmx, tmq, tmqt;
  if (!encode_tmap_2d(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, H, M, ldx * 2, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_row, H, M, H, 128, 16,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmqt, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_colT, M, H, M, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8Q_ERR_UNSUPPORTED;
  unsigned* err = device_error_word();
  if (!err) return FP8Q_ERR_CUDA;
  rmsnorm_rstd_kernel<<<static_cast<int>(rstd_ctas), 256, 0, st>>>(x, M, H, ldx, eps, rstd);
  const fp8q_status s1 = launch_status("rmsnorm_rstd launch");
  if (s1 != FP8Q_OK) return s1;
  constexpr size_t kSmem = a6_smem<TileRms>();
  auto kern = a6_tile_kernel<TileRms, true>;
  static std::atomic<int> occ[64];
  const int per_sm = resident_ctas(kern, kA6Threads, kSmem, occ);
  kern<<<grid_for((M / 128) * (H / 128), per_sm), kA6Threads, kSmem, st>>>(
      tmx, tmx, tmq, tmqt, TileRms{rstd, gamma}, M, H, s_row, lds_row, s_col, err, kWaitLimitNs);
  return launch_status("rmsnorm_quant_dual launch");
}

extern "C" fp8q_status fp8q_swiglu_quant_dual(const uint16_t* gu, int64_t M, int64_t I,
                                              int64_t ldgu, uint8_t* q_row, float* s_row,
                                              int64_t lds_row, uint8_t* q_colT, float* s_col,
                                              void* stream) {
  if (!gu || !q_row || !s_row || !q_colT || !s_col) return FP8Q_ERR_NULL;
  if (M <= 0 || I <= 0 || M % 128 || I % 128 || ldgu < 2 * I || lds_row < M || lds_row % 4)
    return FP8Q_ERR_SHAPE;
  if (!aligned16(gu) || !aligned16(q_row) || !aligned16(s_row) || !aligned16(q_colT) ||
      !aligned16(s_col) || ldgu % 8)
    return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  if (M >= kMaxTmaCoord || I >= kMaxTmaCoord) return FP8Q_ERR_SHAPE;  // 32-bit coordinates
  // the gate and the up halves as two [M][I] tensors
  CUtensorMap tmg, tmu, tmqt;
  if (!encode_tmap_2d(&tmg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gu, I, M, ldgu * 2, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gu + I, I, M, ldgu * 2, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmqt, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_colT, M, I, M, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8Q_ERR_UNSUPPORTED;
  unsigned* err = device_error_word();
  if (!err) return FP8Q_ERR_CUDA;
  auto kern = swiglu_dual_tile_kernel;
  static std::atomic<int> occ[64];
  const int per_sm = resident_ctas(kern, kA6Threads, kSfSmem, occ);
  kern<<<grid_for((M / 128) * (I / 128), per_sm), kA6Threads, kSfSmem, static_cast<cudaStream_t>(stream)>>>(
      tmg, tmu, tmqt, q_row, M, I, s_row, lds_row, s_col, err, kWaitLimitNs);
  return launch_status("swiglu_quant_dual launch");
}

extern "C" fp8q_status fp8q_swiglu_bwd_quant_dual(const uint16_t* gu, const uint16_t* dh,
                                                  int64_t M, int64_t I, uint16_t* dgu,
                                                  uint8_t* q_row, float* s_row, int64_t lds_row,
                                                  uint8_t* q_colT, float* s_col, void* stream) {
  if (!gu || !dh || !q_row || !s_row || !q_colT || !s_col) return FP8Q_ERR_NULL;
  if (M <= 0 || I <= 0 || M % 128 || I % 128 || lds_row < M || lds_row % 4) return FP8Q_ERR_SHAPE;
  if (!aligned16(gu) || !aligned16(dh) || (dgu && !aligned16(dgu)) || !aligned16(q_row) ||
      !aligned16(s_row) || !aligned16(q_colT) || !aligned16(s_col))
    return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  if (M >= kMaxTmaCoord || 2 * I >= kMaxTmaCoord) return FP8Q_ERR_SHAPE;  // 32-bit coordinates
  // the gate and the up halves as two [M][I] tensors; the column codes [2I][M]
  CUtensorMap tmg, tmu, tmqt;
  if (!encode_tmap_2d(&tmg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gu, I, M, I * 4, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gu + I, I, M, I * 4, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_tmap_2d(&tmqt, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_colT, M, 2 * I, M, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8Q_ERR_UNSUPPORTED;
  unsigned* err = device_error_word();
  if (!err) return FP8Q_ERR_CUDA;
  auto kern = swiglu_bwd_tile_kernel;
  static std::atomic<int> occ[64];
  const int per_sm = resident_ctas(kern, kA6Threads, kSbSmem, occ);
  kern<<<grid_for((M / 128) * (I / 128), per_sm), kA6Threads, kSbSmem, static_cast<cudaStream_t>(stream)>>>(
      tmg, tmu, tmqt, dh, dgu, q_row, M, I, s_row, lds_row, s_col, err, kWaitLimitNs);
  return launch_status("swiglu_bwd_quant_dual launch");
}

namespace {
int64_t rmsnorm_bwd_ws_scalars(int64_t M) { return (8 * M + 255) / 256 * 256; }
// dgamma's exact bins hold fewer than 2^23 terms of < 2^39 each: no int64 overflow
constexpr int64_t kRmsBwdMaxRows = int64_t{1} << 23;
// a lane's cached fp64 bin of a row's sum takes at most H / 32 terms: exact up to 2^14
constexpr int64_t kRmsBwdMaxCols = int64_t{1} << 19;
}  // namespace

extern "C" int64_t fp8q_rmsnorm_bwd_workspace_bytes(int64_t M, int64_t H) {
  if (M <= 0 || H <= 0 || M % 128 || H % 128 || M > kRmsBwdMaxRows || H > kRmsBwdMaxCols)
    return -1;
  return rmsnorm_bwd_ws_scalars(M) + H * kXBins * 8;
}

extern "C" fp8q_status fp8q_rmsnorm_bwd_quant_dual(
    const uint16_t* x, const uint16_t* gamma, const uint16_t* dy, const uint16_t* dres, int64_t M,
    int64_t H, float eps, uint16_t* out, uint8_t* q_row, float* s_row, int64_t lds_row,
    uint8_t* q_colT, float* s_col, float* dgamma, void* workspace, int64_t workspace_bytes,
    void* stream) {
  if (!x || !gamma || !dy || !out || !q_row || !s_row || !q_colT || !s_col || !workspace)
    return FP8Q_ERR_NULL;
  if (M <= 0 || H <= 0 || M % 128 || H % 128 || lds_row < M || lds_row % 4 || !(eps >= 0.0f) ||
      M > kRmsBwdMaxRows || H > kRmsBwdMaxCols)
    return FP8Q_ERR_SHAPE;
  if (workspace_bytes < fp8q_rmsnorm_bwd_workspace_bytes(M, H)) {
    set_last_error_text("rmsnorm_bwd_quant_dual: workspace smaller than "
                        "fp8q_rmsnorm_bwd_workspace_bytes(M, H)");
    return FP8Q_ERR_SHAPE;
  }
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(dy) || (dres && !aligned16(dres)) ||
      !aligned16(out) || !aligned16(q_row) || !aligned16(s_row) || !aligned16(q_colT) ||
      !aligned16(s_col) || (dgamma && !aligned16(dgamma)) || !aligned16(workspace))
    return FP8Q_ERR_ALIGN;
  const int sms = sm100_sm_count();
  if (!sms) return FP8Q_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* r = reinterpret_cast<float*>(ws);
  float* k = r + M;
  unsigned long long* bins = reinterpret_cast<unsigned long long*>(ws + rmsnorm_bwd_ws_scalars(M));
  // per-row r and k first (one warp per row), then the tiles, then dgamma
  const int64_t row_ctas = std::min<int64_t>((M + 7) / 8, static_cast<int64_t>(sms) * 8);
  rmsnorm_bwd_rows_kernel<<<static_cast<int>(row_ctas), 256, 0, st>>>(x, gamma, dy, M, H, eps, r, k);
  fp8q_status s1 = launch_status("rmsnorm_bwd_rows launch");
  if (s1 != FP8Q_OK) return s1;
  constexpr size_t kSmem = direct_smem_bytes<RmsBwd>();
  auto kern = direct_dual_kernel<RmsBwd, kBwdBatch, kBwdMinBlocks>;
  static std::atomic<int> occ[64];
  const int per_sm = resident_ctas(kern, 256, kSmem, occ);
  kern<<<grid_for((M / 128) * (H / 128), per_sm), 256, kSmem, st>>>(
      RmsBwd{x, dy, dres, r, k, gamma, H}, M, H, out, q_row, s_row, lds_row, q_colT, s_col);
  s1 = launch_status("rmsnorm_bwd_quant_dual launch");
  if (s1 != FP8Q_OK || !dgamma) return s1;
  // exact dgamma: the bins start at zero, the warps add into them, one thread per
  // column rounds
  if (cudaMemsetAsync(bins, 0, static_cast<size_t>(H) * kXBins * 8, st) != cudaSuccess)
    return launch_status("dgamma bins clear");
  const int64_t dg_warps = ((H / 8 + 31) / 32) * ((M + kDgRows - 1) / kDgRows);
  const int64_t dg_ctas = std::min<int64_t>((dg_warps + 7) / 8, static_cast<int64_t>(sms) * 8);
  dgamma_exact_kernel<<<static_cast<int>(dg_ctas), 256, 0, st>>>(x, dy, r, M, H, bins);
  s1 = launch_status("dgamma_exact launch");
  if (s1 != FP8Q_OK) return s1;
  dgamma_round_kernel<<<static_cast<int>((H + 255) / 256), 256, 0, st>>>(bins, H, dgamma);
  return launch_status("dgamma_round launch");
}
