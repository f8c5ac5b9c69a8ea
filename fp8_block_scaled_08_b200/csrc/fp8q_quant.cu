// Quantizer kernels of libfp8q (sm_100a): the 1x128 activation quantizer, the
// 128x128 weight quantizer, fused RMSNorm+quantize, fused SwiGLU+quantize, the
// dual (row 1x128 + transposed column 128x1) quantizer of BF16 gradients and the
// transposed 128x1 requantizer of saved FP8 activations.
//
// All of them are HBM-bound: BF16 is read with 16-byte loads that a warp issues
// as contiguous 512-byte runs, group maxima are taken with warp shuffles, and the
// codes come from the hardware E4M3 conversion (round to nearest even, saturate).
// Scale and quotient use IEEE division (div.rn) so that codes are a function of the
// inputs alone: s = amax/448 (s = 1 for an all-zero group), code = E4M3(x/s).
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

// ---------------------------------------------------------------------------
// One 1x128 group held by a half-warp: 16 lanes x 8 values.
// Returns the group scale; writes the 8 codes of this lane to `codes`.
// All 32 lanes must call it (the shuffles use the full mask).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float quant_half_warp(const float (&v)[8], uint2& codes) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, off));
  const float s = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 448.0f);
  float t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) t[i] = __fdiv_rn(v[i], s);
  codes.x = cvt_e4m3x4(t[0], t[1], t[2], t[3]);
  codes.y = cvt_e4m3x4(t[4], t[5], t[6], t[7]);
  return s;
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
// function of x.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float exp_cw(float x) {
  const float kLog2e = 0x1.715476p+0f;
  const float kLn2Hi = 0x1.62ep-1f;
  const float kLn2Lo = 0x1.0bfbe8p-15f;
  x = fminf(fmaxf(x, -80.0f), 88.0f);
  const float n = rintf(__fmul_rn(x, kLog2e));
  float r = __fmaf_rn(-n, kLn2Hi, x);
  r = __fmaf_rn(-n, kLn2Lo, r);
  float p = 0x1.a01a02p-13f;            // 1/7!
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);  // 1/6!
  p = __fmaf_rn(p, r, 0x1.111112p-7f);   // 1/5!
  p = __fmaf_rn(p, r, 0x1.555556p-5f);   // 1/4!
  p = __fmaf_rn(p, r, 0x1.555556p-3f);   // 1/3!
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const float two_n = __int_as_float((static_cast<int>(n) + 127) << 23);
  return __fmul_rn(p, two_n);
}

__device__ __forceinline__ float swiglu1(float g, float u) {
  const float e = exp_cw(-g);
  const float d = __fadd_rn(1.0f, e);
  const float silu = __fdiv_rn(g, d);
  return round_bf16(__fmul_rn(silu, u));
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
    for (int i = 0; i < 8; ++i) v[i] = swiglu1(g[i], u[i]);
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
// a3: RMSNorm + 1x128 quantization. One CTA (256 threads) per row; thread t owns
// 8-element chunks t, t+256, ... so that each half-warp covers one 128-group.
// ---------------------------------------------------------------------------
constexpr int kNormThreads = 256;
constexpr int kNormMaxChunks = 8;  // H <= 8 * 8 * 256 = 16384

__global__ void __launch_bounds__(kNormThreads) rmsnorm_quant_kernel(
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
          ss = __dadd_rn(ss, __dmul_rn(d, d));  // each square is exact in fp64
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
      const double ms = __ddiv_rn(tot, static_cast<double>(H));
      const double rr = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, static_cast<double>(eps))));
      r_sh = __double2float_rn(rr);
    }
    __syncthreads();
    const float r = r_sh;
#pragma unroll
    for (int j = 0; j < kNormMaxChunks; ++j) {
      const int64_t c0 = static_cast<int64_t>(j) * kNormThreads + (tid & ~31);
      if (c0 >= nch) break;  // warp-uniform: nch is a multiple of 16
      const int64_t c = tid + j * kNormThreads;
      const bool act = c < nch;
      float v[8];
      if (act) {
        float xv[8], gv[8];
        unpack_bf16x8(raw[j], xv);
        unpack_bf16x8(ld_nc_v4(gamma + c * 8), gv);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = round_bf16(__fmul_rn(__fmul_rn(xv[i], r), gv[i]));
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
      }
      uint2 codes;
      const float sc = quant_half_warp(v, codes);
      if (act) {
        *reinterpret_cast<uint2*>(q + m * H + c * 8) = codes;
        if ((tid & 15) == 0) s[(c >> 4) * lds + m] = sc;
      }
    }
    __syncthreads();  // red / r_sh are reused by the next row
  }
}

// ---------------------------------------------------------------------------
// 128x128 tile kernels (a2, a6, a8). 256 threads; thread t owns rows
// t/16 + 16j (j = 0..7) and the 8 columns 8*(t%16) .. +7 of the tile, so each
// row is read by one half-warp as a contiguous 256-byte (BF16) run. Codes that
// must be stored transposed go through a shared byte tile with an odd row pitch
// (129), which spreads a warp's byte stores over the banks.
// ---------------------------------------------------------------------------
constexpr int kTilePitch = 129;

// Column maxima over the 128 rows of the tile: v[j][i] is (row t/16+16j, col 8*(t%16)+i).
// Result: colmax[c] for c in 0..127 in shared memory.
__device__ __forceinline__ void tile_column_max(const float (&v)[8][8], float* colmax_part,
                                                float* colmax) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  float cm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(v[j][i]));
    a = fmaxf(a, __shfl_xor_sync(kFull, a, 16));
    cm[i] = a;
  }
  if (lane < 16) {
#pragma unroll
    for (int i = 0; i < 8; ++i) colmax_part[wid * 128 + lane * 8 + i] = cm[i];
  }
  __syncthreads();
  if (tid < 128) {
    float a = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) a = fmaxf(a, colmax_part[w * 128 + tid]);
    colmax[tid] = a;
  }
  __syncthreads();
}

// Quantize the tile by columns (scale sc[col]) into the transposed byte tile
// T[col][row], then store T's rows to dst[(col0 + c) * ldd + row0 .. +127].
__device__ __forceinline__ void tile_quant_cols_store_T(const float (&v)[8][8], const float* sc,
                                                        uint8_t* T, uint8_t* __restrict__ dst,
                                                        int64_t ldd) {
  const int tid = threadIdx.x;
  const int rr = tid >> 4, c8 = (tid & 15) * 8;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float s = sc[c8 + i];
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const uint32_t two = cvt_e4m3x2(__fdiv_rn(v[j][i], s), __fdiv_rn(v[j + 1][i], s));
      T[(c8 + i) * kTilePitch + rr + 16 * j] = static_cast<uint8_t>(two & 0xFF);
      T[(c8 + i) * kTilePitch + rr + 16 * (j + 1)] = static_cast<uint8_t>(two >> 8);
    }
  }
  __syncthreads();
  // 128 rows x 8 chunks of 16 bytes; 4 chunks per thread
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int idx = tid + k * 256;
    const int row = idx >> 3, ch = idx & 7;
    const uint8_t* src = T + row * kTilePitch + ch * 16;
    uint32_t w[4];
#pragma unroll
    for (int b = 0; b < 4; ++b)
      w[b] = static_cast<uint32_t>(src[4 * b]) | (static_cast<uint32_t>(src[4 * b + 1]) << 8) |
             (static_cast<uint32_t>(src[4 * b + 2]) << 16) |
             (static_cast<uint32_t>(src[4 * b + 3]) << 24);
    *reinterpret_cast<uint4*>(dst + row * ldd + ch * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// a2: 128x128 weight blocks. grid = (N/128) * (K/128).
__global__ void __launch_bounds__(256) quant_weight_kernel(const uint16_t* __restrict__ w,
                                                           int64_t N, int64_t K, int64_t ldw,
                                                           uint8_t* __restrict__ q,
                                                           float* __restrict__ s,
                                                           uint8_t* __restrict__ qT) {
  __shared__ float red[8];
  __shared__ __align__(16) uint8_t T[128 * kTilePitch];
  const int64_t KB = K >> 7;
  const int64_t nb = blockIdx.x / KB, kb = blockIdx.x % KB;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int rr = tid >> 4, c8 = (tid & 15) * 8;
  const uint16_t* base = w + (nb * 128) * ldw + kb * 128 + c8;
  uint4 raw[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) raw[j] = ld_nc_v4(base + (rr + 16 * j) * ldw);
  float v[8][8];
  float a = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    unpack_bf16x8(raw[j], v[j]);
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[j][i]));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, off));
  if (lane == 0) red[wid] = a;
  __syncthreads();
  float amax = red[0];
#pragma unroll
  for (int k = 1; k < 8; ++k) amax = fmaxf(amax, red[k]);
  const float sc = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
  if (tid == 0) s[nb * KB + kb] = sc;
  uint8_t* qb = q + (nb * 128) * K + kb * 128 + c8;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = __fdiv_rn(v[j][i], sc);
    uint2 codes;
    codes.x = cvt_e4m3x4(t[0], t[1], t[2], t[3]);
    codes.y = cvt_e4m3x4(t[4], t[5], t[6], t[7]);
    *reinterpret_cast<uint2*>(qb + (rr + 16 * j) * K) = codes;
    if (qT) {
      const uint8_t* cb = reinterpret_cast<const uint8_t*>(&codes);
#pragma unroll
      for (int i = 0; i < 8; ++i) T[(c8 + i) * kTilePitch + rr + 16 * j] = cb[i];
    }
  }
  if (qT) {
    __syncthreads();
    uint8_t* dst = qT + (kb * 128) * N + nb * 128;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = tid + k * 256;
      const int row = idx >> 3, ch = idx & 7;
      const uint8_t* src = T + row * kTilePitch + ch * 16;
      uint32_t wv[4];
#pragma unroll
      for (int b = 0; b < 4; ++b)
        wv[b] = static_cast<uint32_t>(src[4 * b]) | (static_cast<uint32_t>(src[4 * b + 1]) << 8) |
                (static_cast<uint32_t>(src[4 * b + 2]) << 16) |
                (static_cast<uint32_t>(src[4 * b + 3]) << 24);
      *reinterpret_cast<uint4*>(dst + row * N + ch * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
  }
}

// a6: BF16 dY tile -> row-wise 1x128 codes (direct) + column-wise 128x1 codes
// (transposed). grid = (M/128) * (N/128).
__global__ void __launch_bounds__(256) transpose_quant_bf16_kernel(
    const uint16_t* __restrict__ dy, int64_t M, int64_t N, int64_t lddy,
    uint8_t* __restrict__ q_row, float* __restrict__ s_row, int64_t lds_row,
    uint8_t* __restrict__ q_colT, float* __restrict__ s_col) {
  __shared__ float colmax_part[8 * 128];
  __shared__ float colsc[128];
  __shared__ __align__(16) uint8_t T[128 * kTilePitch];
  const int64_t NB = N >> 7;
  const int64_t mb = blockIdx.x / NB, nb = blockIdx.x % NB;
  const int tid = threadIdx.x;
  const int rr = tid >> 4, c8 = (tid & 15) * 8;
  const uint16_t* base = dy + (mb * 128) * lddy + nb * 128 + c8;
  uint4 raw[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) raw[j] = ld_nc_v4(base + (rr + 16 * j) * lddy);
  float v[8][8];
#pragma unroll
  for (int j = 0; j < 8; ++j) unpack_bf16x8(raw[j], v[j]);

  if (q_row) {  // row-wise: each tile row is one 1x128 group, held by a half-warp
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint2 codes;
      const float sc = quant_half_warp(v[j], codes);
      const int64_t m = mb * 128 + rr + 16 * j;
      *reinterpret_cast<uint2*>(q_row + m * N + nb * 128 + c8) = codes;
      if ((tid & 15) == 0) s_row[nb * lds_row + m] = sc;
    }
  }
  tile_column_max(v, colmax_part, colsc);
  if (tid < 128) {
    const float a = colsc[tid];
    const float sc = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 448.0f);
    colsc[tid] = sc;
    s_col[mb * N + nb * 128 + tid] = sc;
  }
  __syncthreads();
  tile_quant_cols_store_T(v, colsc, T, q_colT + (nb * 128) * M + mb * 128, M);
}

// a8: saved FP8 activation tile (1x128 groups) -> xhat = fl32(s * dec(q)) ->
// 128x1 groups along M, stored transposed. grid = (M/128) * (K/128).
__global__ void __launch_bounds__(256) transpose_quant_fp8_kernel(
    const uint8_t* __restrict__ qin, const float* __restrict__ sin, int64_t M, int64_t K,
    int64_t lds, uint8_t* __restrict__ qT, float* __restrict__ sT) {
  __shared__ float colmax_part[8 * 128];
  __shared__ float colsc[128];
  __shared__ __align__(16) uint8_t T[128 * kTilePitch];
  const int64_t KB = K >> 7;
  const int64_t mb = blockIdx.x / KB, kb = blockIdx.x % KB;
  const int tid = threadIdx.x;
  const int rr = tid >> 4, c8 = (tid & 15) * 8;
  const uint8_t* base = qin + (mb * 128) * K + kb * 128 + c8;
  uint2 raw[8];
  float rs[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    raw[j] = *reinterpret_cast<const uint2*>(base + (rr + 16 * j) * K);
    rs[j] = sin[kb * lds + mb * 128 + rr + 16 * j];
  }
  float v[8][8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t w[2] = {raw[j].x, raw[j].y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float2 lo = e4m3x2_to_f32(static_cast<uint16_t>(w[h] & 0xFFFF));
      const float2 hi = e4m3x2_to_f32(static_cast<uint16_t>(w[h] >> 16));
      v[j][4 * h + 0] = __fmul_rn(rs[j], lo.x);
      v[j][4 * h + 1] = __fmul_rn(rs[j], lo.y);
      v[j][4 * h + 2] = __fmul_rn(rs[j], hi.x);
      v[j][4 * h + 3] = __fmul_rn(rs[j], hi.y);
    }
  }
  tile_column_max(v, colmax_part, colsc);
  if (tid < 128) {
    const float a = colsc[tid];
    const float sc = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 448.0f);
    colsc[tid] = sc;
    sT[mb * K + kb * 128 + tid] = sc;
  }
  __syncthreads();
  tile_quant_cols_store_T(v, colsc, T, qT + (kb * 128) * M + mb * 128, M);
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
  rowgroup_quant_kernel<ActSrc, 2><<<grid_for_units((units + 1) / 2), 256, 0,
                                     static_cast<cudaStream_t>(stream)>>>(ActSrc{x, ldx}, M, G, q,
                                                                          K, s, lds);
  return launch_status();
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
  return launch_status();
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
  const int64_t grid = M < static_cast<int64_t>(sms) * 64 ? M : static_cast<int64_t>(sms) * 64;
  rmsnorm_quant_kernel<<<static_cast<int>(grid), kNormThreads, 0,
                         static_cast<cudaStream_t>(stream)>>>(x, gamma, M, H, ldx, eps, q, s, lds);
  return launch_status();
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
  return launch_status();
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
  return launch_status();
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
  return launch_status();
}
