// Quantizer kernels of libfp8q (sm_100a): the 1x128 activation quantizer, the
// 128x128 weight quantizer, fused RMSNorm+quantize, fused SwiGLU+quantize, the
// dual (row 1x128 + transposed column 128x1) quantizer of BF16 gradients and the
// transposed 128x1 requantizer of saved FP8 activations.
//
// All of them are HBM-bound: BF16 is read with 16-byte loads that a warp issues as
// contiguous runs, group maxima are taken with warp shuffles, and the codes come from
// the hardware E4M3 conversion (round to nearest even, saturate). A group's scale is
// s = amax/448 by IEEE division (s = 1 for an all-zero group); each code is the E4M3
// value nearest to the IEEE quotient x/s. Where x is a BF16 value (every quantizer
// but the FP8 requantizer) the quotient is formed from the correctly rounded
// reciprocal r = 1/s with one residual correction (q = x*r; e = fma(-q, s, x);
// q = fma(e, r, q); sign of x), which yields the same E4M3 code as the IEEE quotient
// for every BF16 x and every BF16 amax >= |x| with s >= 2^-80 (checked exhaustively by
// the test suite); groups with smaller s use the IEEE division itself.
//
// Method: "Resumen Técnico: Jet-RL" (gist.science, paper 2601.14243), section
// "Esquema de Cuantización" (1x128 activation groups, 128x128 weight blocks,
// FP8 saved activations produced by the preceding operator, BF16 gradients,
// 1x128 / 128x1 WGrad grouping) and section "Implementación" (fused
// activation/RMSNorm and transposition kernels).
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
  float s, rs;
  bool small;
};

__device__ __forceinline__ GroupScale group_scale(float amax) {
  GroupScale g;
  g.s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
  g.rs = __frcp_rn(g.s);
  g.small = g.s < kSmallScale;
  return g;
}

__device__ __forceinline__ float copy_sign(float v, float sgn) {
  return __uint_as_float((__float_as_uint(v) & 0x7FFFFFFFu) | (__float_as_uint(sgn) & 0x80000000u));
}

// Two quotients x/s of BF16-valued x (see the file header for why this equals the
// IEEE quotient's code).
__device__ __forceinline__ void quotient2(float x0, float x1, const GroupScale& g, float& t0,
                                          float& t1) {
  if (g.small) {
    t0 = __fdiv_rn(x0, g.s);
    t1 = __fdiv_rn(x1, g.s);
    return;
  }
  float q0, q1;
  mul2(q0, q1, x0, x1, g.rs, g.rs);      // q = x * r
  float e0 = x0, e1 = x1;
  fma2(e0, e1, -q0, -q1, g.s, g.s);      // e = fma(-q, s, x), exact
  fma2(q0, q1, e0, e1, g.rs, g.rs);      // q = fma(e, r, q)
  t0 = copy_sign(q0, x0);
  t1 = copy_sign(q1, x1);
}

// Eight codes of BF16-valued x (packed little-endian into two words).
__device__ __forceinline__ uint2 codes8(const float (&v)[8], const GroupScale& g) {
  float t[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) quotient2(v[i], v[i + 1], g, t[i], t[i + 1]);
  return make_uint2(cvt_e4m3x4(t[0], t[1], t[2], t[3]), cvt_e4m3x4(t[4], t[5], t[6], t[7]));
}

// One 1x128 group held by a half-warp: 16 lanes x 8 values. Returns the group scale;
// writes the 8 codes of this lane. All 32 lanes must call it (full-mask shuffles).
__device__ __forceinline__ float quant_half_warp(const float (&v)[8], uint2& codes) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, off));
  const GroupScale g = group_scale(a);
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
  x0 = fminf(fmaxf(x0, -80.0f), 88.0f);
  x1 = fminf(fmaxf(x1, -80.0f), 88.0f);
  float l0, l1;
  mul2(l0, l1, x0, x1, kLog2e, kLog2e);
  const float n0 = rintf(l0), n1 = rintf(l1);
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
  const float s0 = __int_as_float((static_cast<int>(n0) + 127) << 23);
  const float s1 = __int_as_float((static_cast<int>(n1) + 127) << 23);
  mul2(e0, e1, c0, c1, s0, s1);
}

// h = bf16( fl32( fl32(g / fl32(1 + E(-g))) * u ) ), two at a time.
__device__ __forceinline__ void swiglu2(float g0, float g1, float u0, float u1, float& h0,
                                        float& h1) {
  float e0, e1;
  exp_cw2(-g0, -g1, e0, e1);
  const float d0 = __fadd_rn(1.0f, e0), d1 = __fadd_rn(1.0f, e1);
  const float s0 = __fdiv_rn(g0, d0), s1 = __fdiv_rn(g1, d1);
  float m0, m1;
  mul2(m0, m1, s0, s1, u0, u1);
  h0 = round_bf16(m0);
  h1 = round_bf16(m1);
}

// ---------------------------------------------------------------------------
// Row-group quantizers (a1, a4): one warp handles a pair of 1x128 groups of one
// row per step (lane l owns columns 8*(l%16) .. +7 of group 2*pair + l/16).
// Sources supply raw 16-byte loads first (so several are in flight) and turn
// them into the 8 fp32 values afterwards.
// ---------------------------------------------------------------------------
struct ActSrc {
  const uint16_t* x;
  int64_t ldx;
  struct Raw { uint4 a; };
  __device__ __forceinline__ Raw fetch(int64_t m, int64_t col) const {
    return Raw{ld_nc_v4(x + m * ldx + col)};
  }
  __device__ __forceinline__ void values(const Raw& r, float (&v)[8]) const {
    unpack_bf16x8(r.a, v);
  }
};

struct SwigluSrc {
  const uint16_t* gu;
  int64_t ldgu, I;
  struct Raw { uint4 g, u; };
  __device__ __forceinline__ Raw fetch(int64_t m, int64_t col) const {
    const uint16_t* row = gu + m * ldgu;
    return Raw{ld_nc_v4(row + col), ld_nc_v4(row + I + col)};
  }
  __device__ __forceinline__ void values(const Raw& r, float (&v)[8]) const {
    float g[8], u[8];
    unpack_bf16x8(r.g, g);
    unpack_bf16x8(r.u, u);
#pragma unroll
    for (int i = 0; i < 8; i += 2) swiglu2(g[i], g[i + 1], u[i], u[i + 1], v[i], v[i + 1]);
  }
};

template <class Src, int kUnroll>
__global__ void __launch_bounds__(256) rowgroup_quant_kernel(Src src, int64_t M, int64_t G,
                                                             uint8_t* __restrict__ q, int64_t ldq,
                                                             float* __restrict__ s, int64_t lds) {
  const int64_t pairs = (G + 1) >> 1;
  const int64_t units = M * pairs;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int sub = lane & 15;

  for (int64_t base = warp; base < units; base += kUnroll * nwarps) {
    typename Src::Raw raw[kUnroll];
    bool act[kUnroll];
    int64_t mm[kUnroll], gg[kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      const int64_t u = base + j * nwarps;
      const int64_t m = u / pairs;
      const int64_t g = 2 * (u - m * pairs) + half;
      mm[j] = m;
      gg[j] = g;
      act[j] = (u < units) && (g < G);
      if (act[j]) raw[j] = src.fetch(m, g * 128 + sub * 8);
    }
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      if (base + j * nwarps >= units) break;  // warp-uniform
      float v[8];
      if (act[j]) {
        src.values(raw[j], v);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
      }
      uint2 codes;
      const float sc = quant_half_warp(v, codes);
      if (act[j]) {
        *reinterpret_cast<uint2*>(q + mm[j] * ldq + gg[j] * 128 + sub * 8) = codes;
        if (sub == 0) s[gg[j] * lds + mm[j]] = sc;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// a3: RMSNorm + 1x128 quantization.
// Rows of up to kWarpRowChunks*256 elements: one warp per row (the row stays in
// registers, the sum of squares is a warp reduction), 8 rows per CTA.
// Longer rows: one CTA (256 threads) per row.
// Thread t of the row owns 8-element chunks t, t+T, ... (T = threads per row), so
// that each half-warp covers one 128-group.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float rstd_from_ss(double ss, int64_t H, float eps) {
  const double ms = __ddiv_rn(ss, static_cast<double>(H));
  const double rr = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, static_cast<double>(eps))));
  return __double2float_rn(rr);
}

// y = bf16(fl32(fl32(x r) g)) for one chunk, then the half-warp group quantization.
__device__ __forceinline__ void norm_quant_chunk(const uint4& xr, const uint16_t* gamma, int64_t c,
                                                 bool act, float r, uint8_t* qrow, float* s,
                                                 int64_t lds, int64_t m, int lane) {
  float v[8];
  if (act) {
    float xv[8], gv[8];
    unpack_bf16x8(xr, xv);
    unpack_bf16x8(ld_nc_v4(gamma + c * 8), gv);
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

constexpr int kWarpRowChunks = 24;  // warp-per-row path: H <= 24 * 256 = 6144

template <int kChunks>
__global__ void __launch_bounds__(256) rmsnorm_quant_warp_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ gamma, int64_t M, int64_t H,
    int64_t ldx, float eps, uint8_t* __restrict__ q, float* __restrict__ s, int64_t lds) {
  const int lane = threadIdx.x & 31;
  const int64_t nch = H >> 3;
  const int64_t wglobal = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t m = wglobal; m < M; m += nw) {
    const uint16_t* row = x + m * ldx;
    uint4 raw[kChunks];
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < kChunks; ++j) {
      const int64_t c = lane + 32 * j;
      if (c < nch) raw[j] = ld_nc_v4(row + c * 8);
    }
#pragma unroll
    for (int j = 0; j < kChunks; ++j) {
      const int64_t c = lane + 32 * j;
      if (c < nch) {
        float v[8];
        unpack_bf16x8(raw[j], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double d = static_cast<double>(v[i]);
          ss = __fma_rn(d, d, ss);  // the square is exact, so this is the fp64 sum
        }
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(kFull, ss, off));
    const float r = rstd_from_ss(ss, H, eps);
#pragma unroll
    for (int j = 0; j < kChunks; ++j) {
      if (32 * j >= nch) break;  // warp-uniform; nch is a multiple of 16
      const int64_t c = lane + 32 * j;
      norm_quant_chunk(raw[j], gamma, c, c < nch, r, q + m * H, s, lds, m, lane);
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
  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;
  const int64_t nch = H >> 3;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const uint16_t* row = x + m * ldx;
    uint4 raw[kNormMaxChunks];
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < kNormMaxChunks; ++j) {
      const int64_t c = tid + j * kNormThreads;
      if (c < nch) raw[j] = ld_nc_v4(row + c * 8);
    }
#pragma unroll
    for (int j = 0; j < kNormMaxChunks; ++j) {
      const int64_t c = tid + j * kNormThreads;
      if (c < nch) {
        float v[8];
        unpack_bf16x8(raw[j], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double d = static_cast<double>(v[i]);
          ss = __fma_rn(d, d, ss);
        }
      }
    }
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
      if (c0 >= nch) break;  // warp-uniform: nch is a multiple of 16
      const int64_t c = tid + j * kNormThreads;
      norm_quant_chunk(raw[j], gamma, c, c < nch, r, q + m * H, s, lds, m, lane);
    }
    __syncthreads();  // red / r_sh are reused by the next row
  }
}

// ---------------------------------------------------------------------------
// 128x128 tile kernels (a2, a6, a8). 256 threads.
// Row pass: thread t owns rows t/16 + 16j (j = 0..7) and the 8 columns
// 8*(t%16) .. +7, so each tile row is read by one half-warp as one contiguous run and
// each row is one 1x128 group.
// Column pass: the tile is staged in shared memory; thread t owns the column pair
// 2*(t%64), +1 and the 32 rows 32*(t/64) .. +31. A warp reads 32 consecutive column
// pairs of one row per load (no bank conflicts); each thread produces 2 x 32
// consecutive codes of the transposed output, stored as two 32-byte runs.
// ---------------------------------------------------------------------------
constexpr int kTP = 136;  // row pitch of a staged BF16 tile, in elements (272 bytes)

// Column pass over a staged BF16 tile Ts[128][kTP]. Column scales: computed per
// column (per_col) or the given block scale. Codes go to dst[(c)*ldd + r] for
// tile column c and tile row r; per-column scales to scol[c] (if not null).
__device__ __forceinline__ void tile_cols_bf16(const uint16_t* Ts, float* red, bool per_col,
                                               const GroupScale& blk, uint8_t* __restrict__ dst,
                                               int64_t ldd, float* __restrict__ scol) {
  const int tid = threadIdx.x;
  const int cp = tid & 63, rq = tid >> 6;
  uint32_t w[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) w[r] = *reinterpret_cast<const uint32_t*>(Ts + (32 * rq + r) * kTP + 2 * cp);
  GroupScale g0 = blk, g1 = blk;
  if (per_col) {
    float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      a0 = fmaxf(a0, fabsf(bf16_lo(w[r])));
      a1 = fmaxf(a1, fabsf(bf16_hi(w[r])));
    }
    red[rq * 128 + 2 * cp] = a0;
    red[rq * 128 + 2 * cp + 1] = a1;
    __syncthreads();
    a0 = fmaxf(fmaxf(red[2 * cp], red[128 + 2 * cp]), fmaxf(red[256 + 2 * cp], red[384 + 2 * cp]));
    a1 = fmaxf(fmaxf(red[2 * cp + 1], red[128 + 2 * cp + 1]),
               fmaxf(red[256 + 2 * cp + 1], red[384 + 2 * cp + 1]));
    g0 = group_scale(a0);
    g1 = group_scale(a1);
    if (rq == 0 && scol) *reinterpret_cast<float2*>(scol + 2 * cp) = make_float2(g0.s, g1.s);
  }
  uint32_t o0[8], o1[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float t0[4], t1[4];
    quotient2(bf16_lo(w[4 * k]), bf16_lo(w[4 * k + 1]), g0, t0[0], t0[1]);
    quotient2(bf16_lo(w[4 * k + 2]), bf16_lo(w[4 * k + 3]), g0, t0[2], t0[3]);
    quotient2(bf16_hi(w[4 * k]), bf16_hi(w[4 * k + 1]), g1, t1[0], t1[1]);
    quotient2(bf16_hi(w[4 * k + 2]), bf16_hi(w[4 * k + 3]), g1, t1[2], t1[3]);
    o0[k] = cvt_e4m3x4(t0[0], t0[1], t0[2], t0[3]);
    o1[k] = cvt_e4m3x4(t1[0], t1[1], t1[2], t1[3]);
  }
  uint4* d0 = reinterpret_cast<uint4*>(dst + (2 * cp) * ldd + 32 * rq);
  uint4* d1 = reinterpret_cast<uint4*>(dst + (2 * cp + 1) * ldd + 32 * rq);
  d0[0] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
  d0[1] = make_uint4(o0[4], o0[5], o0[6], o0[7]);
  d1[0] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
  d1[1] = make_uint4(o1[4], o1[5], o1[6], o1[7]);
}

// a2: 128x128 weight blocks. grid = (N/128) * (K/128).
__global__ void __launch_bounds__(256) quant_weight_kernel(const uint16_t* __restrict__ w,
                                                           int64_t N, int64_t K, int64_t ldw,
                                                           uint8_t* __restrict__ q,
                                                           float* __restrict__ s,
                                                           uint8_t* __restrict__ qT) {
  __shared__ float red[8];
  __shared__ __align__(16) uint16_t Ts[128 * kTP];
  const int64_t KB = K >> 7;
  const int64_t nb = blockIdx.x / KB, kb = blockIdx.x % KB;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int rr = tid >> 4, c8 = (tid & 15) * 8;
  const uint16_t* base = w + (nb * 128) * ldw + kb * 128 + c8;
  uint4 raw[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) raw[j] = ld_nc_v4(base + (rr + 16 * j) * ldw);
  float a = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float v[8];
    unpack_bf16x8(raw[j], v);
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    if (qT) *reinterpret_cast<uint4*>(Ts + (rr + 16 * j) * kTP + c8) = raw[j];
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, off));
  if (lane == 0) red[wid] = a;
  __syncthreads();
  float amax = red[0];
#pragma unroll
  for (int k = 1; k < 8; ++k) amax = fmaxf(amax, red[k]);
  const GroupScale g = group_scale(amax);
  if (tid == 0) s[nb * KB + kb] = g.s;
  uint8_t* qb = q + (nb * 128) * K + kb * 128 + c8;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float v[8];
    unpack_bf16x8(raw[j], v);
    *reinterpret_cast<uint2*>(qb + (rr + 16 * j) * K) = codes8(v, g);
  }
  if (qT) tile_cols_bf16(Ts, nullptr, false, g, qT + (kb * 128) * N + nb * 128, N, nullptr);
}

// a6: BF16 dY tile -> row-wise 1x128 codes (row pass) + column-wise 128x1 codes
// (column pass, transposed). grid = (M/128) * (N/128).
__global__ void __launch_bounds__(256) transpose_quant_bf16_kernel(
    const uint16_t* __restrict__ dy, int64_t M, int64_t N, int64_t lddy,
    uint8_t* __restrict__ q_row, float* __restrict__ s_row, int64_t lds_row,
    uint8_t* __restrict__ q_colT, float* __restrict__ s_col) {
  __shared__ float red[4 * 128];
  __shared__ __align__(16) uint16_t Ts[128 * kTP];
  const int64_t NB = N >> 7;
  const int64_t mb = blockIdx.x / NB, nb = blockIdx.x % NB;
  const int tid = threadIdx.x;
  const int rr = tid >> 4, c8 = (tid & 15) * 8;
  const uint16_t* base = dy + (mb * 128) * lddy + nb * 128 + c8;
  uint4 raw[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) raw[j] = ld_nc_v4(base + (rr + 16 * j) * lddy);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    *reinterpret_cast<uint4*>(Ts + (rr + 16 * j) * kTP + c8) = raw[j];
    if (q_row) {  // each tile row is one 1x128 group, held by a half-warp
      float v[8];
      unpack_bf16x8(raw[j], v);
      uint2 codes;
      const float sc = quant_half_warp(v, codes);
      const int64_t m = mb * 128 + rr + 16 * j;
      *reinterpret_cast<uint2*>(q_row + m * N + nb * 128 + c8) = codes;
      if ((tid & 15) == 0) s_row[nb * lds_row + m] = sc;
    }
  }
  __syncthreads();
  const GroupScale unused{1.0f, 1.0f, false};
  tile_cols_bf16(Ts, red, true, unused, q_colT + (nb * 128) * M + mb * 128, M,
                 s_col + mb * N + nb * 128);
}

// a8: saved FP8 activation tile (1x128 groups) -> xhat = fl32(s * dec(q)) ->
// 128x1 groups along M, stored transposed. grid = (M/128) * (K/128).
// The codes and row scales are staged in shared memory; the column pass decodes two
// codes per load. xhat is an arbitrary fp32 value here, so quotients use IEEE
// division.
constexpr int kQP = 144;  // row pitch of a staged code tile, in bytes

__global__ void __launch_bounds__(256) transpose_quant_fp8_kernel(
    const uint8_t* __restrict__ qin, const float* __restrict__ sin, int64_t M, int64_t K,
    int64_t lds, uint8_t* __restrict__ qT, float* __restrict__ sT) {
  __shared__ float red[4 * 128];
  __shared__ float rsc[128];
  __shared__ __align__(16) uint8_t Tq[128 * kQP];
  const int64_t KB = K >> 7;
  const int64_t mb = blockIdx.x / KB, kb = blockIdx.x % KB;
  const int tid = threadIdx.x;
  {
    const int rr = tid >> 3, c16 = (tid & 7) * 16;  // 32 rows x 8 chunks of 16 bytes per pass
    const uint8_t* base = qin + (mb * 128) * K + kb * 128 + c16;
    uint4 raw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) raw[j] = ld_nc_v4(base + (rr + 32 * j) * K);
    if (tid < 128) rsc[tid] = sin[kb * lds + mb * 128 + tid];
#pragma unroll
    for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4*>(Tq + (rr + 32 * j) * kQP + c16) = raw[j];
  }
  __syncthreads();
  const int cp = tid & 63, rq = tid >> 6;
  float x0[32], x1[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    const int row = 32 * rq + r;
    const uint16_t two = *reinterpret_cast<const uint16_t*>(Tq + row * kQP + 2 * cp);
    const float2 d = e4m3x2_to_f32(two);
    const float sr = rsc[row];
    x0[r] = __fmul_rn(sr, d.x);
    x1[r] = __fmul_rn(sr, d.y);
  }
  float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    a0 = fmaxf(a0, fabsf(x0[r]));
    a1 = fmaxf(a1, fabsf(x1[r]));
  }
  red[rq * 128 + 2 * cp] = a0;
  red[rq * 128 + 2 * cp + 1] = a1;
  __syncthreads();
  a0 = fmaxf(fmaxf(red[2 * cp], red[128 + 2 * cp]), fmaxf(red[256 + 2 * cp], red[384 + 2 * cp]));
  a1 = fmaxf(fmaxf(red[2 * cp + 1], red[128 + 2 * cp + 1]),
             fmaxf(red[256 + 2 * cp + 1], red[384 + 2 * cp + 1]));
  const float s0 = (a0 == 0.0f) ? 1.0f : __fdiv_rn(a0, 448.0f);
  const float s1 = (a1 == 0.0f) ? 1.0f : __fdiv_rn(a1, 448.0f);
  if (rq == 0) *reinterpret_cast<float2*>(sT + mb * K + kb * 128 + 2 * cp) = make_float2(s0, s1);
  uint32_t o0[8], o1[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    o0[k] = cvt_e4m3x4(__fdiv_rn(x0[4 * k], s0), __fdiv_rn(x0[4 * k + 1], s0),
                       __fdiv_rn(x0[4 * k + 2], s0), __fdiv_rn(x0[4 * k + 3], s0));
    o1[k] = cvt_e4m3x4(__fdiv_rn(x1[4 * k], s1), __fdiv_rn(x1[4 * k + 1], s1),
                       __fdiv_rn(x1[4 * k + 2], s1), __fdiv_rn(x1[4 * k + 3], s1));
  }
  uint8_t* dst = qT + (kb * 128) * M + mb * 128;
  uint4* d0 = reinterpret_cast<uint4*>(dst + (2 * cp) * M + 32 * rq);
  uint4* d1 = reinterpret_cast<uint4*>(dst + (2 * cp + 1) * M + 32 * rq);
  d0[0] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
  d0[1] = make_uint4(o0[4], o0[5], o0[6], o0[7]);
  d1[0] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
  d1[1] = make_uint4(o1[4], o1[5], o1[6], o1[7]);
}

int grid_for_units(int64_t warps_needed) {
  const int sms = sm100_sm_count();
  int64_t ctas = (warps_needed + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sms) * 8;  // 8 CTAs x 256 threads = 2048 per SM
  if (ctas > cap) ctas = cap;
  return static_cast<int>(ctas < 1 ? 1 : ctas);
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" fp8q_status fp8q_quant_act_1x128(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                            uint8_t* q, float* s, int64_t lds, void* stream) {
  if (!x || !q || !s) return FP8Q_ERR_NULL;
  if (M <= 0 || K <= 0 || K % 128 || ldx < K || lds < M || lds % 4) return FP8Q_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(q) || !aligned16(s) || ldx % 8) return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  const int64_t G = K / 128;
  const int64_t units = M * ((G + 1) / 2);
  rowgroup_quant_kernel<ActSrc, 4><<<grid_for_units((units + 3) / 4), 256, 0,
                                     static_cast<cudaStream_t>(stream)>>>(ActSrc{x, ldx}, M, G, q,
                                                                          K, s, lds);
  return launch_status("quant_act_1x128 launch");
}

extern "C" fp8q_status fp8q_swiglu_quant(const uint16_t* gu, int64_t M, int64_t I, int64_t ldgu,
                                         uint8_t* q, float* s, int64_t lds, void* stream) {
  if (!gu || !q || !s) return FP8Q_ERR_NULL;
  if (M <= 0 || I <= 0 || I % 128 || ldgu < 2 * I || lds < M || lds % 4) return FP8Q_ERR_SHAPE;
  if (!aligned16(gu) || !aligned16(q) || !aligned16(s) || ldgu % 8) return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  const int64_t G = I / 128;
  const int64_t units = M * ((G + 1) / 2);
  rowgroup_quant_kernel<SwigluSrc, 2><<<grid_for_units((units + 1) / 2), 256, 0,
                                        static_cast<cudaStream_t>(stream)>>>(
      SwigluSrc{gu, ldgu, I}, M, G, q, I, s, lds);
  return launch_status("swiglu_quant launch");
}

extern "C" fp8q_status fp8q_rmsnorm_quant(const uint16_t* x, const uint16_t* gamma, int64_t M,
                                          int64_t H, int64_t ldx, float eps, uint8_t* q, float* s,
                                          int64_t lds, void* stream) {
  if (!x || !gamma || !q || !s) return FP8Q_ERR_NULL;
  if (M <= 0 || H <= 0 || H % 128 || H > 8 * kNormMaxChunks * kNormThreads || ldx < H ||
      lds < M || lds % 4 || !(eps >= 0.0f))
    return FP8Q_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(q) || !aligned16(s) || ldx % 8)
    return FP8Q_ERR_ALIGN;
  const int sms = sm100_sm_count();
  if (!sms) return FP8Q_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (H <= 8 * 32 * kWarpRowChunks) {
    const int64_t ctas = (M + 7) / 8;
    const int64_t grid = ctas < static_cast<int64_t>(sms) * 8 ? ctas : static_cast<int64_t>(sms) * 8;
    if (H <= 8 * 32 * 16)
      rmsnorm_quant_warp_kernel<16><<<static_cast<int>(grid), 256, 0, st>>>(x, gamma, M, H, ldx,
                                                                            eps, q, s, lds);
    else
      rmsnorm_quant_warp_kernel<kWarpRowChunks><<<static_cast<int>(grid), 256, 0, st>>>(
          x, gamma, M, H, ldx, eps, q, s, lds);
  } else {
    const int64_t grid = M < static_cast<int64_t>(sms) * 64 ? M : static_cast<int64_t>(sms) * 64;
    rmsnorm_quant_cta_kernel<<<static_cast<int>(grid), kNormThreads, 0, st>>>(x, gamma, M, H, ldx,
                                                                              eps, q, s, lds);
  }
  return launch_status("rmsnorm_quant launch");
}

extern "C" fp8q_status fp8q_quant_weight_128x128(const uint16_t* w, int64_t N, int64_t K,
                                                 int64_t ldw, uint8_t* q, float* s, uint8_t* qT,
                                                 void* stream) {
  if (!w || !q || !s) return FP8Q_ERR_NULL;
  if (N <= 0 || K <= 0 || N % 128 || K % 128 || ldw < K) return FP8Q_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(q) || !aligned16(s) || (qT && !aligned16(qT)) || ldw % 8)
    return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  const int64_t blocks = (N / 128) * (K / 128);
  if (blocks > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  quant_weight_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                        static_cast<cudaStream_t>(stream)>>>(w, N, K, ldw, q, s, qT);
  return launch_status("quant_weight_128x128 launch");
}

extern "C" fp8q_status fp8q_transpose_quant_bf16(const uint16_t* dy, int64_t M, int64_t N,
                                                 int64_t lddy, uint8_t* q_row, float* s_row,
                                                 int64_t lds_row, uint8_t* q_colT, float* s_col,
                                                 void* stream) {
  if (!dy || !q_colT || !s_col || (q_row != nullptr) != (s_row != nullptr)) return FP8Q_ERR_NULL;
  if (M <= 0 || N <= 0 || M % 128 || N % 128 || lddy < N || (q_row && (lds_row < M || lds_row % 4)))
    return FP8Q_ERR_SHAPE;
  if (!aligned16(dy) || !aligned16(q_colT) || !aligned16(s_col) || lddy % 8 ||
      (q_row && (!aligned16(q_row) || !aligned16(s_row))))
    return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  const int64_t blocks = (M / 128) * (N / 128);
  if (blocks > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  transpose_quant_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                                static_cast<cudaStream_t>(stream)>>>(dy, M, N, lddy, q_row, s_row,
                                                                     lds_row, q_colT, s_col);
  return launch_status("transpose_quant_bf16 launch");
}

extern "C" fp8q_status fp8q_transpose_quant_fp8(const uint8_t* q, const float* s, int64_t M,
                                                int64_t K, int64_t lds, uint8_t* qT, float* sT,
                                                void* stream) {
  if (!q || !s || !qT || !sT) return FP8Q_ERR_NULL;
  if (M <= 0 || K <= 0 || M % 128 || K % 128 || lds < M) return FP8Q_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(s) || !aligned16(qT) || !aligned16(sT) || lds % 4)
    return FP8Q_ERR_ALIGN;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  const int64_t blocks = (M / 128) * (K / 128);
  if (blocks > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  transpose_quant_fp8_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                               static_cast<cudaStream_t>(stream)>>>(q, s, M, K, lds, qT, sT);
  return launch_status("transpose_quant_fp8 launch");
}
