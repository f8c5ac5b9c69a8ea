// Block-scaled FP8 GEMM for sm_100a (the forward, DGrad and WGrad of the linear
// layer):
//
//   out[i, j] = sum_r  sA(i, r) * sB(j, r) * sum_{l in slice r} qA[i, l] * qB[j, l]
//
// qA [M][K] and qB [N][K] are E4M3 codes, K-major; r runs over 128-wide K slices.
// sA(i, r) is a per-row fp32 scale (the 1x128 groups, stored [K/128][ldsa]);
// sB(j, r) is either one fp32 scale per 128x128 block of B (forward / DGrad) or
// one per column of B (WGrad, whose two operands are both grouped along the
// reduction dimension). "Resumen Técnico: Jet-RL", section "Esquema de
// Cuantización": 1x128 activations, 128x128 weights, FP8 DGrad/WGrad with 1x128
// and 128x1 grouping.
//
// Because the scales are arbitrary fp32 numbers, the tensor core cannot apply them
// (its block-scaled MMA only takes power-of-two or E4M3 scale formats). Each
// 128-wide slice is therefore multiplied on the tensor core into a fresh fp32 TMEM
// accumulator, and the CUDA cores "promote" it: acc += P_r * (sA * sB), in fp32,
// slice after slice in increasing r. That order is fixed, so a row of the output
// is the same whatever M is (the rollout and the training forward share numerics,
// "Arquitectura Central").
//
// Kernel structure (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warp 0      TMA producer: A/B tiles into a 4-stage shared-memory ring (128-byte
//               swizzle) and the scale vectors into an 8-slot ring.
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (kind::f8f6f4, 128x256x32, 4 per slice) into TMEM buffer r%2 and
//               commits to mbarriers that free the smem stage / publish the slice.
//   warps 2, 3  idle. Warpgroup 0 (warps 0-3) hands registers to the others.
//   warps 4..11 two warpgroups; warpgroup h promotes columns 128h..128h+127 of the
//               128x256 tile: tcgen05.ld, packed fp32 FMA into 128 registers per
//               thread, release the TMEM buffer; after the last slice they round to
//               BF16 and store the tile.
// Registers: the block launches with 168 per thread (168 x 384 = 64512); warpgroup
// 0 drops to 40 and the promotion warpgroups rise to 232 (40*128 + 232*256 = 64512).
// Every mbarrier wait is bounded (kWaitLimitNs): a wait that gives up records
// FP8Q_ERR_TIMEOUT in the device error word and the CTA winds down cleanly.
#include <algorithm>

#include "fp8q_device.cuh"
#include "fp8q_host.h"

namespace fp8q {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int kStages = 4;
constexpr int kScStages = 8;
constexpr int kThreads = 384;
constexpr uint32_t kRegsLaunch = 168;   // what ptxas allots under __launch_bounds__(384, 1)
constexpr uint32_t kRegsControl = 40;   // warpgroup 0 after the hand-over
constexpr uint32_t kRegsPromote = 232;  // warpgroups 1 and 2 after the hand-over
static_assert(kRegsControl * 128 + kRegsPromote * 256 <= kRegsLaunch * kThreads,
              "register hand-over exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;  // two 128x256 fp32 accumulators
constexpr uint32_t kABytes = BM * BK;
constexpr uint32_t kBBytes = BN * BK;
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kScABytes = BM * 4;
constexpr uint32_t kScBBytes = BN * 4;
constexpr uint32_t kScSlot = kScABytes + kScBBytes;

__host__ __device__ constexpr uint32_t kOffA(int s) { return s * kStageBytes; }
__host__ __device__ constexpr uint32_t kOffB(int s) { return s * kStageBytes + kABytes; }
__host__ __device__ constexpr uint32_t kOffScA(int i) { return kStages * kStageBytes + i * kScSlot; }
__host__ __device__ constexpr uint32_t kOffScB(int i) { return kOffScA(i) + kScABytes; }
constexpr uint32_t kOffBars = kStages * kStageBytes + kScStages * kScSlot;
constexpr uint32_t kNumBars = 2 * kStages + 4 + 2 * kScStages + 1;
constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr size_t kSmemBytes = kSmemUsed + 1024;  // slack to align the base to 1024
static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");

struct GemmParams {
  int32_t M, N, K;
  int32_t mblocks, nblocks, kblocks;
  int32_t n_fastest;
  const float* sb;  // per-block B scales: sb[(j/128)*sb_sj + r*sb_sr]
  int64_t sb_sj, sb_sr;
  uint16_t* y;
  int64_t ldy;
  unsigned* err;
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void tile_coords(int t, const GemmParams& p, int& mb, int& nb) {
  if (p.n_fastest) {
    nb = t % p.nblocks;
    mb = t / p.nblocks;
  } else {
    mb = t % p.mblocks;
    nb = t / p.mblocks;
  }
}

// Wait used while winding down after a give-up: ignores the abort flag, still bounded.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

template <bool kColScaleB>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* sfull = tempty + 2;
  uint64_t* sempty = sfull + kScStages;
  uint64_t* done = sempty + kScStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 8);  // the 8 promotion warps
    }
    for (int i = 0; i < kScStages; ++i) {
      mbar_init(sfull + i, 1);
      mbar_init(sempty + i, 8);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmSA);
    if (kColScaleB) prefetch_tensormap(&tmSB);
  }
  if (warp == 1) tmem_alloc<kTmemCols>(tmem_slot);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.err, p.wait_limit_ns};
  const int num_tiles = p.mblocks * p.nblocks;

  if (warp < 4) {
   // Each role's code sits inside the branch of its register budget, so that the
   // compiler allocates it under that budget.
   regs_decrease<kRegsControl>();
   if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, sci = 0, scph = 0;
      // bit s of issued/par: stage s has a load in flight or done, and its phase parity
      uint32_t issued = 0, par = 0, sc_issued = 0, sc_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(full + stage, kStageBytes);
          tma_load_2d(smem + kOffA(stage), &tmA, kb * BK, mb * BM, full + stage);
          tma_load_2d(smem + kOffB(stage), &tmB, kb * BK, nb * BN, full + stage);
          issued |= 1u << stage;
          par = (par & ~(1u << stage)) | (phase << stage);
          if (!mbar_wait(sempty + sci, scph ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(sfull + sci, kScABytes + (kColScaleB ? kScBBytes : 0u));
          tma_load_2d(smem + kOffScA(sci), &tmSA, mb * BM, kb, sfull + sci);
          if (kColScaleB) tma_load_2d(smem + kOffScB(sci), &tmSB, nb * BN, kb, sfull + sci);
          sc_issued |= 1u << sci;
          sc_par = (sc_par & ~(1u << sci)) | (scph << sci);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
          if (++sci == kScStages) { sci = 0; scph ^= 1; }
        }
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        for (int s = 0; s < kStages; ++s)
          if ((issued >> s) & 1u) mbar_wait_drain(full + s, (par >> s) & 1u, p.wait_limit_ns);
        for (int i = 0; i < kScStages; ++i)
          if ((sc_issued >> i) & 1u) mbar_wait_drain(sfull + i, (sc_par >> i) & 1u, p.wait_limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_e4m3_f32(BM, BN);
      uint32_t stage = 0, phase = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        for (int kb = 0; kb < p.kblocks; ++kb) {
          const uint32_t buf = it & 1u, tph = (it >> 1) & 1u;
          if (!mbar_wait(tempty + buf, tph ^ 1u, ctl)) { ok = false; break; }
          if (!mbar_wait(full + stage, phase, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + kOffA(stage));
          const uint32_t b0 = smem_u32(smem + kOffB(stage));
          const uint32_t d = tmem_base + buf * BN;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_f8f6f4(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k), idesc,
                       k > 0 ? 1u : 0u);
          mma_commit(empty + stage);
          mma_commit(tfull + buf);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
          ++it;
        }
      }
      // wait for every MMA this thread issued (they read smem and write TMEM)
      mma_commit(done);
      mbar_wait_drain(done, 0, p.wait_limit_ns);
    }
    __syncwarp();
   }
  } else {
    regs_increase<kRegsPromote>();
    // ------------------------------------------------------------ promotion + epilogue
    const int wq = warp & 3;           // TMEM lane quarter this warp may access
    const int half = (warp - 4) >> 2;  // column half of the 256-wide tile
    const int row = wq * 32 + lane;
    uint32_t it = 0, sci = 0, scph = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int ncol0 = nb * BN + half * BM;
      const bool col_ok = ncol0 < p.N;
      const float* sbp = kColScaleB ? nullptr : p.sb + static_cast<int64_t>(ncol0 / 128) * p.sb_sj;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
      for (int kb = 0; kb < p.kblocks; ++kb) {
        float sbv = 0.0f;
        if (!kColScaleB && col_ok) sbv = __ldg(sbp + kb * p.sb_sr);
        if (!mbar_wait_warp(sfull + sci, scph, ctl)) { ok = false; break; }
        const float sa = reinterpret_cast<const float*>(smem + kOffScA(sci))[row];
        const uint32_t buf = it & 1u, tph = (it >> 1) & 1u;
        if (!mbar_wait_warp(tfull + buf, tph, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t taddr =
            tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + buf * BN + half * BM;
        if (!kColScaleB) {
          const float s = __fmul_rn(sa, sbv);
#pragma unroll
          for (int c = 0; c < 2; ++c) {  // two 64-column halves, two loads in flight
            uint32_t r[64];
            tmem_ld32(taddr + c * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            tmem_ld32(taddr + c * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 64; i += 2)
              fma2(acc[c * 64 + i], acc[c * 64 + i + 1], __uint_as_float(r[i]),
                   __uint_as_float(r[i + 1]), s, s);
          }
        } else {
          const float* scb = reinterpret_cast<const float*>(smem + kOffScB(sci)) + half * BM;
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // four 32-column quarters, one load in flight
            uint32_t r[32];
            tmem_ld32(taddr + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 sb2 = *reinterpret_cast<const float2*>(scb + c * 32 + i);
              float s0, s1;
              mul2(s0, s1, sa, sa, sb2.x, sb2.y);
              fma2(acc[c * 32 + i], acc[c * 32 + i + 1], __uint_as_float(r[i]),
                   __uint_as_float(r[i + 1]), s0, s1);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(tempty + buf);
          mbar_arrive(sempty + sci);
        }
        ++it;
        if (++sci == kScStages) { sci = 0; scph ^= 1; }
      }
      if (!ok) break;
      const int64_t m = static_cast<int64_t>(mb) * BM + row;
      if (m < p.M && col_ok) {
        uint4* dst = reinterpret_cast<uint4*>(p.y + m * p.ldy + ncol0);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          uint4 v;
          v.x = pack_bf16x2(acc[8 * c + 0], acc[8 * c + 1]);
          v.y = pack_bf16x2(acc[8 * c + 2], acc[8 * c + 3]);
          v.z = pack_bf16x2(acc[8 * c + 4], acc[8 * c + 5]);
          v.w = pack_bf16x2(acc[8 * c + 6], acc[8 * c + 7]);
          dst[c] = v;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc<kTmemCols>(tmem_base);
  }
}

template <bool kCol>
bool ensure_smem_attr() {
  static int done_for_device[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (done_for_device[dev]) return true;
  const cudaError_t e = cudaFuncSetAttribute(
      gemm_kernel<kCol>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(gemm max dynamic smem)", e);
    cudaGetLastError();
    return false;
  }
  // The register hand-over inside the kernel waits until the block's launch allocation
  // covers the new budgets; refuse to launch a build whose allocation would not.
  cudaFuncAttributes attr;
  const cudaError_t ea = cudaFuncGetAttributes(&attr, gemm_kernel<kCol>);
  if (ea != cudaSuccess) {
    set_last_error("cudaFuncGetAttributes(gemm)", ea);
    cudaGetLastError();
    return false;
  }
  if (static_cast<uint32_t>(attr.numRegs) * kThreads < kRegsControl * 128 + kRegsPromote * 256 ||
      attr.maxThreadsPerBlock < kThreads) {
    set_last_error("gemm register budget check", cudaErrorLaunchOutOfResources);
    return false;
  }
  done_for_device[dev] = 1;
  return true;
}

// out [Mg][Ng] = A [Mg][Kg] x B [Ng][Kg]^T with the scales described above.
template <bool kCol>
fp8q_status launch_gemm(const uint8_t* A, const uint8_t* B, int64_t Mg, int64_t Ng, int64_t Kg,
                        const float* sa, int64_t ldsa, const float* sb, int64_t sb_sj,
                        int64_t sb_sr, const float* sbcol, uint16_t* y, int64_t ldy,
                        cudaStream_t stream) {
  const int sms = sm100_sm_count();
  if (!sms) return FP8Q_ERR_UNSUPPORTED;
  if (Mg > 0x7FFFFFFF || Ng > 0x7FFFFFFF || Kg > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  CUtensorMap tmA, tmB, tmSA, tmSB;
  bool ok = encode_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, Kg, Mg, Kg, BK, BM,
                           CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, Kg, Ng, Kg, BK, BN,
                           CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_tmap_2d(&tmSA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sa, Mg, Kg / BK, ldsa * 4, BM,
                           1, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (ok && kCol)
    ok = encode_tmap_2d(&tmSB, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sbcol, Ng, Kg / BK, Ng * 4, BN, 1,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    tmSB = tmSA;
  if (!ok) return FP8Q_ERR_UNSUPPORTED;
  if (!ensure_smem_attr<kCol>()) return FP8Q_ERR_CUDA;

  GemmParams p;
  p.M = static_cast<int32_t>(Mg);
  p.N = static_cast<int32_t>(Ng);
  p.K = static_cast<int32_t>(Kg);
  p.mblocks = static_cast<int32_t>((Mg + BM - 1) / BM);
  p.nblocks = static_cast<int32_t>((Ng + BN - 1) / BN);
  p.kblocks = static_cast<int32_t>(Kg / BK);
  p.n_fastest = Ng <= Mg ? 1 : 0;
  p.sb = sb;
  p.sb_sj = sb_sj;
  p.sb_sr = sb_sr;
  p.y = y;
  p.ldy = ldy;
  p.err = device_error_word();
  p.wait_limit_ns = kWaitLimitNs;
  if (!p.err) return FP8Q_ERR_CUDA;
  const int64_t tiles = static_cast<int64_t>(p.mblocks) * p.nblocks;
  if (tiles > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const int grid = static_cast<int>(std::min<int64_t>(tiles, sms));
  gemm_kernel<kCol><<<grid, kThreads, kSmemBytes, stream>>>(tmA, tmB, tmSA, tmSB, p);
  return launch_status("gemm_kernel launch");
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" fp8q_status fp8q_linear_fwd(const uint8_t* qa, const float* sa, int64_t ldsa,
                                       const uint8_t* qw, const float* sw, int64_t M, int64_t N,
                                       int64_t K, uint16_t* y, int64_t ldy, void* stream) {
  if (!qa || !sa || !qw || !sw || !y) return FP8Q_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || N % 128 || K % 128 || ldsa < M || ldy < N)
    return FP8Q_ERR_SHAPE;
  if (!aligned16(qa) || !aligned16(sa) || !aligned16(qw) || !aligned16(sw) || !aligned16(y) ||
      ldsa % 4 || ldy % 8)
    return FP8Q_ERR_ALIGN;
  // B = W [N][K]; block scale of (n, slice r) = sw[(n/128)*(K/128) + r]
  return launch_gemm<false>(qa, qw, M, N, K, sa, ldsa, sw, K / 128, 1, nullptr, y, ldy,
                            static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_linear_dgrad(const uint8_t* qdy, const float* sdy, int64_t ldsdy,
                                         const uint8_t* qwT, const float* sw, int64_t M,
                                         int64_t N, int64_t K, uint16_t* dx, int64_t lddx,
                                         void* stream) {
  if (!qdy || !sdy || !qwT || !sw || !dx) return FP8Q_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || N % 128 || K % 128 || ldsdy < M || lddx < K)
    return FP8Q_ERR_SHAPE;
  if (!aligned16(qdy) || !aligned16(sdy) || !aligned16(qwT) || !aligned16(sw) ||
      !aligned16(dx) || ldsdy % 4 || lddx % 8)
    return FP8Q_ERR_ALIGN;
  // GEMM rows = M, columns = K, reduction = N. B = W^T [K][N];
  // block scale of (k, slice r over n) = sw[r*(K/128) + k/128]
  return launch_gemm<false>(qdy, qwT, M, K, N, sdy, ldsdy, sw, 1, K / 128, nullptr, dx, lddx,
                            static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_linear_wgrad(const uint8_t* qdyT, const float* sdy_c,
                                         const uint8_t* qxT, const float* sx_c, int64_t M,
                                         int64_t N, int64_t K, uint16_t* dw, int64_t lddw,
                                         void* stream) {
  if (!qdyT || !sdy_c || !qxT || !sx_c || !dw) return FP8Q_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || M % 128 || N % 128 || K % 128 || lddw < K)
    return FP8Q_ERR_SHAPE;
  if (!aligned16(qdyT) || !aligned16(sdy_c) || !aligned16(qxT) || !aligned16(sx_c) ||
      !aligned16(dw) || lddw % 8)
    return FP8Q_ERR_ALIGN;
  // GEMM rows = N, columns = K, reduction = M (tokens).
  // Row scale of (n, slice r) = sdy_c[r*N + n]  (a [M/128][N] array: ldsa = N)
  // Column scale of (k, slice r) = sx_c[r*K + k]
  return launch_gemm<true>(qdyT, qxT, N, K, M, sdy_c, N, nullptr, 0, 0, sx_c, dw, lddw,
                           static_cast<cudaStream_t>(stream));
}
