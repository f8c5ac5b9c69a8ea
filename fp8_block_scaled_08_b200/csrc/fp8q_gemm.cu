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
// Kernel structure. CTAs run in pairs (a cluster of 2 on neighbouring SMs) that share
// one 256x256 output tile: each CTA loads its own 128 rows of A and its own 128 rows
// of B (no multicast), and the leader CTA issues tcgen05.mma.cta_group::2 (M = 256,
// N = 256, K = 32; 4 per slice) that reads both CTAs' shared memory and writes
// 128 x 256 fp32 into each CTA's TMEM. Per 128-wide slice each SM therefore moves
// 32 KB in (TMA) and 32 KB out (tensor-core reads) of shared memory instead of 48 + 48
// KB with single-CTA 128x256 tiles, which keeps shared-memory bandwidth below the
// tensor core's demand. 384 threads per CTA:
//   warp 0      TMA producer: its A/B halves into a 4-stage ring (128-byte swizzle),
//               completing on the leader's barrier; the row scales (and WGrad's column
//               scales) into a small ring of slots, 8 slices per slot for the
//               block-scaled kernels, so their promotion waits for scales once per 8
//               slices (a barrier wait costs ~100-200 cycles even when it is already
//               complete: measured).
//   warp 1      allocates 512 TMEM columns (both CTAs); in the leader, one thread
//               issues the pair MMAs into TMEM buffer r%2 and commits to barriers in
//               both CTAs that free the smem stage / publish the slice. For the
//               block-scaled B (forward, DGrad) one thread of warp 2 issues every other
//               slice, so two threads share the issuing.
//   warps 2, 3  otherwise idle. Warpgroup 0 (warps 0-3) hands registers to the others.
//   warps 4..11 two warpgroups; warpgroup h promotes columns 128h..128h+127 of this
//               CTA's 128 x 256 part: tcgen05.ld, packed fp32 FMA into 128 registers
//               per thread, release the TMEM buffer (every thread arrives; the peer's on the
//               leader's barrier); after the last slice they round to BF16, stage the
//               rows in shared memory (128-byte swizzle) and store them with TMA (the
//               fp32-accumulate WGrad stages fp32 boxes and adds them into its output
//               with TMA reduce-add instead).
// Registers: the block launches with 168 per thread (168 x 384 = 64512); warpgroup
// 0 drops to 56 and the promotion warpgroups rise to 224 (56*128 + 224*256 = 64512),
// 40 and 232 for the column-scaled WGrad.
// Every mbarrier wait is bounded (kWaitLimitNs): a wait that gives up records
// FP8Q_ERR_TIMEOUT in the device error word and both CTAs wind down.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "fp8q_device.cuh"
#include "fp8q_host.h"

namespace fp8q {
namespace {

constexpr int BM = 128;        // rows of the tile per CTA (the pair covers 256)
constexpr int BN = 256;        // columns of the tile (each CTA loads 128 rows of B)
constexpr int BK = 128;        // one scale slice
constexpr int kPairM = 2 * BM;
constexpr int kStages = 4;
// Scales: the row scales (and the column-scaled WGrad's column scales) of sc_batch
// consecutive slices arrive together in one of sc_slots slots. The block-scaled kernels
// take 8 slices per barrier wait (measured 13-19 % faster than one); the WGrad measured
// ~7 % slower that way than with one slice per slot and 8 slots.
template <bool kCol>
__host__ __device__ constexpr int sc_batch() { return kCol ? 1 : 8; }
template <bool kCol>
__host__ __device__ constexpr int sc_slots() { return kCol ? 8 : 2; }
constexpr int kScSlotsMax = 8;
constexpr int kThreads = 384;
// Leader threads issuing MMAs, taking alternate slices (warps 1 and 2): one thread needs
// about 90 cycles per MMA plus ~100-200 per barrier wait (measured), close to the 512
// cycles of tensor work per slice. The column-scaled WGrad measured ~2 % slower with two.
template <bool kColScaleB>
__host__ __device__ constexpr int issuers() { return kColScaleB ? 1 : 2; }
static_assert(kStages % 2 == 0, "each ring stage is always used by the same issuer");
constexpr uint32_t kRegsLaunch = 168;   // what ptxas allots under __launch_bounds__(384, 1)
// Warpgroup 0 after the hand-over: with two MMA issuers 40 registers made the compiler
// spill in the issue loop, so the block-scaled kernels give it 56.
template <bool kCol>
__host__ __device__ constexpr uint32_t regs_control() { return kCol ? 40 : 56; }
// Warpgroups 1 and 2 after the hand-over.
template <bool kCol>
__host__ __device__ constexpr uint32_t regs_promote() { return kCol ? 232 : 224; }
static_assert(regs_control<true>() * 128 + regs_promote<true>() * 256 <= kRegsLaunch * kThreads &&
                  regs_control<false>() * 128 + regs_promote<false>() * 256 <= kRegsLaunch * kThreads,
              "register hand-over exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;  // two 128x256 fp32 accumulators
constexpr uint32_t kABytes = BM * BK;
constexpr uint32_t kBBytes = (BN / 2) * BK;
constexpr uint32_t kStageBytes = kABytes + kBBytes;  // per CTA
template <bool kCol>  // [sc_batch][BM] row scales
__host__ __device__ constexpr uint32_t sc_a_bytes() { return BM * 4 * sc_batch<kCol>(); }
template <bool kCol>  // [sc_batch][BN] column scales (WGrad)
__host__ __device__ constexpr uint32_t sc_b_bytes() { return kCol ? BN * 4 * sc_batch<kCol>() : 0; }
constexpr uint32_t kScRegion = 24576;  // scale slots of either variant
static_assert(sc_slots<true>() * (sc_a_bytes<true>() + sc_b_bytes<true>()) <= kScRegion &&
                  sc_slots<false>() * (sc_a_bytes<false>() + sc_b_bytes<false>()) <= kScRegion &&
                  sc_slots<true>() <= kScSlotsMax && sc_slots<false>() <= kScSlotsMax,
              "scale slots exceed their region");
constexpr uint32_t kStageOutBytes = 32 * 64 * 2;  // one 32-row x 64-column BF16 box

__host__ __device__ constexpr uint32_t kOffA(int s) { return s * kStageBytes; }
__host__ __device__ constexpr uint32_t kOffB(int s) { return s * kStageBytes + kABytes; }
template <bool kCol>
__host__ __device__ constexpr uint32_t off_sc_a(int i) {
  return kStages * kStageBytes + i * (sc_a_bytes<kCol>() + sc_b_bytes<kCol>());
}
template <bool kCol>
__host__ __device__ constexpr uint32_t off_sc_b(int i) { return off_sc_a<kCol>(i) + sc_a_bytes<kCol>(); }
constexpr uint32_t kOffOut = kStages * kStageBytes + kScRegion;  // 8 warps x 2 boxes
__host__ __device__ constexpr uint32_t kOffOutBox(int w, int j) {
  return kOffOut + (2 * w + j) * kStageOutBytes;
}
constexpr uint32_t kOffBars = kOffOut + 16 * kStageOutBytes;
constexpr uint32_t kNumBars = 2 * kStages + 4 + 2 * kScSlotsMax + 1;
constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr size_t kSmemBytes = kSmemUsed + 1024;  // slack to align the base to 1024
static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");
static_assert(kOffOut % 1024 == 0, "TMA store boxes need 1024-byte alignment");

struct GemmParams {
  int32_t M, N, K;
  int32_t mblocks, nblocks, kblocks;
  int32_t group;  // panels per raster group (column panels; row panels with `swap`)
  int32_t swap;
  const float* sb;  // per-block B scales: sb[(j/128)*sb_sj + r*sb_sr]
  int64_t sb_sj, sb_sr;
  uint16_t* y;
  int64_t ldy;
  unsigned* err;
  uint64_t wait_limit_ns;
};

// Tile order. Within a group of `group` consecutive column panels (row panels with
// `swap`) the tiles walk that group fastest and the other dimension's panels slower.
// The host picks one of two orders from the operand sizes:
//  - the smaller operand fits in half of L2: one group spans all of its panels, so they
//    stay in L2 while each panel of the larger operand streams through once;
//  - otherwise groups of 8 column panels, so that the 74 tiles of one wave of CTA pairs
//    cover about 9 row panels x 8 column panels (17 distinct operand panels). Every wave
//    re-reads its panels from DRAM (the K loop restarts), so the distinct panels per wave
//    set the traffic (measured 17 % less DRAM traffic for the down-projection forward
//    and 10 % less for the gate/up DGrad than a walk over all 16 column panels).
__device__ __forceinline__ void tile_coords(int t, const GemmParams& p, int& mb, int& nb) {
  const int slow = p.swap ? p.nblocks : p.mblocks;
  const int fast = p.swap ? p.mblocks : p.nblocks;
  const int span = p.group * slow;
  const int g = t / span;
  const int w = t - g * span;
  const int width = min(p.group, fast - g * p.group);
  const int x = g * p.group + w % width;
  const int y = w / width;
  mb = p.swap ? x : y;
  nb = p.swap ? y : x;
}

// Wait used while winding down after a give-up: ignores the abort flag, still bounded.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

// kAccF32: instead of storing BF16, add the fp32 accumulator into an fp32 output
// (out += A x B^T) by TMA reduce-add of 32 x 32 boxes.
template <bool kColScaleB, bool kAccF32 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint64_t* full = bars;              // leader: both CTAs' A/B bytes of a stage
  uint64_t* empty = full + kStages;   // both: stage consumed by the pair MMAs
  uint64_t* tfull = empty + kStages;  // both: slice accumulator in TMEM buffer b ready
  uint64_t* tempty = tfull + 2;       // leader: both CTAs' promotion done with buffer b
  uint64_t* sfull = tempty + 2;       // local scale batches
  uint64_t* sempty = sfull + kScSlotsMax;
  uint64_t* done = sempty + kScSlotsMax;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    // A TMEM buffer is released by every thread of both promotion warpgroups of each
    // CTA (every thread arrives, with no warp-level gather first: measured 5-6 % faster
    // for all three GEMMs than one arrival per warp after a __syncwarp).
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 2 * 256);
    }
    for (int i = 0; i < sc_slots<kColScaleB>(); ++i) {
      mbar_init(sfull + i, 1);
      mbar_init(sempty + i, 256);
    }
    mbar_init(done, issuers<kColScaleB>());
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmSA);
    prefetch_tensormap(&tmY);
    if (kColScaleB) prefetch_tensormap(&tmSB);
  }
  if (warp == 1) tmem_alloc_pair<kTmemCols>(tmem_slot);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.err, p.wait_limit_ns};
  const int num_tiles = p.mblocks * p.nblocks;

  if (warp < 4) {
   // Each role's code sits inside the branch of its register budget, so that the
   // compiler allocates it under that budget.
   regs_decrease<regs_control<kColScaleB>()>();
   if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, sci = 0, scph = 0;
      // bit s of issued/par: stage s has a load in flight or done, and its phase parity
      uint32_t issued = 0, par = 0, sc_issued = 0, sc_par = 0;
      bool ok = true;
      for (int t = pair; ok && t < num_tiles; t += npairs) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        const int row0 = mb * kPairM + static_cast<int>(rank) * BM;
        const int brow0 = nb * BN + static_cast<int>(rank) * (BN / 2);
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1, ctl)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(full + stage, 2 * kStageBytes);
          const uint32_t leader_full = cluster_addr(full + stage, 0);
          tma_load_2d_pair(smem + kOffA(stage), &tmA, kb * BK, row0, leader_full);
          tma_load_2d_pair(smem + kOffB(stage), &tmB, kb * BK, brow0, leader_full);
          issued |= 1u << stage;
          par = (par & ~(1u << stage)) | (phase << stage);
          if (kb % sc_batch<kColScaleB>() == 0) {  // the scales of slices kb .. kb + batch - 1
            if (!mbar_wait(sempty + sci, scph ^ 1, ctl)) { ok = false; break; }
            mbar_arrive_expect_tx(sfull + sci, sc_a_bytes<kColScaleB>() + sc_b_bytes<kColScaleB>());
            tma_load_2d(smem + off_sc_a<kColScaleB>(sci), &tmSA, row0, kb, sfull + sci);
            if (kColScaleB) tma_load_2d(smem + off_sc_b<kColScaleB>(sci), &tmSB, nb * BN, kb, sfull + sci);
            sc_issued |= 1u << sci;
            sc_par = (sc_par & ~(1u << sci)) | (scph << sci);
            if (++sci == sc_slots<kColScaleB>()) { sci = 0; scph ^= 1; }
          }
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        if (rank == 0)
          for (int s = 0; s < kStages; ++s)
            if ((issued >> s) & 1u) mbar_wait_drain(full + s, (par >> s) & 1u, p.wait_limit_ns);
        for (int i = 0; i < sc_slots<kColScaleB>(); ++i)
          if ((sc_issued >> i) & 1u) mbar_wait_drain(sfull + i, (sc_par >> i) & 1u, p.wait_limit_ns);
      }
    }
    __syncwarp();
   } else if (warp <= issuers<kColScaleB>()) {
    // ------------------------------------------------------------ MMA issuers (leader)
    // With two issuers, issuer i = warp - 1 takes the slices that use TMEM buffer i (slice
    // parity); each slice is 4 MMAs of N = 256 into its buffer and one commit.
    if (lane == 0 && rank == 0) {
      const uint32_t issuer = static_cast<uint32_t>(warp - 1);
      const uint32_t idesc = idesc_e4m3_f32(kPairM, BN);
      uint32_t stage = 0, phase = 0, it = 0;
      bool ok = true;
      for (int t = pair; ok && t < num_tiles; t += npairs) {
        for (int kb = 0; ok && kb < p.kblocks; ++kb) {
          const uint32_t buf = it & 1u, tph = (it >> 1) & 1u;
          if (issuers<kColScaleB>() == 2 && buf != issuer) {  // the other issuer's slice
            if (++stage == kStages) { stage = 0; phase ^= 1; }
            ++it;
            continue;
          }
          if (!mbar_wait(full + stage, phase, ctl)) { ok = false; break; }
          const uint32_t a0 = smem_u32(smem + kOffA(stage));
          const uint32_t b0 = smem_u32(smem + kOffB(stage));
          if (!mbar_wait(tempty + buf, tph ^ 1u, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem_base + buf * BN;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_f8f6f4_pair(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k),
                            idesc, k > 0 ? 1u : 0u);
          mma_commit_pair_multicast(tfull + buf, 0x3);
          mma_commit_pair_multicast(empty + stage, 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
          ++it;
        }
      }
      // wait for every MMA issued by both issuers (they read both CTAs' smem and write
      // both TMEMs); `done` completes after each issuer's commit
      mma_commit_pair_multicast(done, 0x1);
      mbar_wait_drain(done, 0, p.wait_limit_ns);
    }
    __syncwarp();
   }
  } else {
    regs_increase<regs_promote<kColScaleB>()>();
    // ------------------------------------------------------------ promotion + epilogue
    // Warpgroup `half` owns TMEM columns [128*half, +128) of each slice buffer, which are
    // tile columns 128*half + [0,128) (a pair MMA of width 256 takes its first 128
    // columns from the leader's B rows and the next 128 from the peer's): one 128-wide
    // block of B, so one block scale per slice when B is block-scaled.
    const int wq = warp & 3;           // TMEM lane quarter this warp may access
    const int half = (warp - 4) >> 2;  // TMEM half-buffer of this warpgroup
    const int row = wq * 32 + lane;
    const uint32_t tempty_leader0 = cluster_addr(tempty, 0);
    uint8_t* out0 = smem + kOffOutBox(warp - 4, 0);
    uint8_t* out1 = smem + kOffOutBox(warp - 4, 1);
    uint32_t it = 0, sci = 0, scph = 0;
    bool ok = true, stored = false;
    for (int t = pair; ok && t < num_tiles; t += npairs) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int row0 = mb * kPairM + static_cast<int>(rank) * BM;
      const int col_lo = nb * BN + 128 * half;  // tile columns of acc[0..63]
      const int col_hi = col_lo + 64;           // of acc[64..127]
      // a ragged N (a multiple of 16) ends inside a box: the tensor store clips it
      const bool lo_ok = col_lo < p.N;
      const bool hi_ok = col_hi < p.N;
      const float* sbp = kColScaleB ? nullptr : p.sb + static_cast<int64_t>(col_lo / 128) * p.sb_sj;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
      // block scales of B, 32 slices at a time: lane l holds slice 32*(kb/32) + l; the
      // next 32 are fetched 16 slices ahead (a global load per slice, even prefetched one
      // slice ahead, measured ~10 % slower)
      auto sb_fetch = [&](int kk) -> float {
        return (!kColScaleB && lo_ok && kk < p.kblocks) ? __ldg(sbp + static_cast<int64_t>(kk) * p.sb_sr)
                                                        : 0.0f;
      };
      float sbv = sb_fetch(lane), sbx = 0.0f;
      for (int kb = 0; kb < p.kblocks; ++kb) {
        const int j = kb % sc_batch<kColScaleB>();  // slice within its scale batch
        if (!kColScaleB) {
          if ((kb & 31) == 16) sbx = sb_fetch(kb + 16 + lane);
          if ((kb & 31) == 0 && kb > 0) sbv = sbx;
        }
        const float sb = kColScaleB ? 0.0f : __shfl_sync(0xFFFFFFFFu, sbv, kb & 31);
        if (j == 0 && !mbar_wait_warp(sfull + sci, scph, ctl)) { ok = false; break; }
        const float* sa_slot = reinterpret_cast<const float*>(smem + off_sc_a<kColScaleB>(sci)) + j * BM;
        const float* scb = reinterpret_cast<const float*>(smem + off_sc_b<kColScaleB>(sci)) + j * BN;
        const uint32_t buf = it & 1u, tph = (it >> 1) & 1u;
        // block-scaled B: one scale product per slice; column-scaled B: the row scales of
        // this thread's four rows (lanes 8e + lane/4 of the warp's quarter, the 16x256b
        // layout below). Both are read before the wait, not after it on the critical path
        // (measured ~16 % faster for the column-scaled WGrad).
        float s_h = kColScaleB ? 0.0f : __fmul_rn(sa_slot[row], sb);
        float sa4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (kColScaleB) {
#pragma unroll
          for (int e = 0; e < 4; ++e) sa4[e] = sa_slot[wq * 32 + 8 * e + (lane >> 2)];
        }
        asm volatile("" : "+f"(s_h), "+f"(sa4[0]), "+f"(sa4[1]), "+f"(sa4[2]), "+f"(sa4[3]));
        if (!mbar_wait_warp(tfull + buf, tph, ctl)) { ok = false; break; }
        tc_fence_after();
        if constexpr (!kColScaleB) {
          const uint32_t taddr =
              tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + buf * BN + half * (BN / 2);
#pragma unroll
          for (int c = 0; c < 2; ++c) {  // acc columns [64c, 64c + 64), two loads in flight
            uint32_t r[64];
            tmem_ld32(taddr + c * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            tmem_ld32(taddr + c * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 64; i += 2)
              fma2(acc[c * 64 + i], acc[c * 64 + i + 1], __uint_as_float(r[i]),
                   __uint_as_float(r[i + 1]), s_h, s_h);
          }
        } else {
          // Column-scaled B: every element needs its own column's scale. With one row per
          // thread (the 32x32b shape) each thread would hold all 128 column scales of its
          // columns in registers every slice, and filling them from shared memory took
          // 70 % of the shared-memory pipe (measured): that bound the kernel. In the
          // 16x256b shape a thread holds 4 rows x 32 columns, so it needs a quarter of the
          // column scales. acc[((2b + cc) * 8 + k) * 4 + 2hi + {0,1}] is row
          // 16b + 8hi + lane/4 of the warp's quarter, columns 64cc + 8k + 2(lane%4) + {0,1}
          // of the warpgroup's 128.
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            float2 sb2[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              sb2[k] = *reinterpret_cast<const float2*>(scb + 128 * half + 64 * cc + 8 * k + 2 * (lane & 3));
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              uint32_t r[32];
              tmem_ld_16x256b_x8(tmem_base + (static_cast<uint32_t>(wq * 32 + 16 * b) << 16) + buf * BN +
                                     half * (BN / 2) + 64 * cc,
                                 r);
              tmem_wait_ld();
              if (cc == 1 && b == 1) {
                // the buffer goes back before the last FMAs (measured ~6 % faster here,
                // ~7 % slower for the block-scaled kernels)
                tc_fence_before();
                if (rank == 0) mbar_arrive(tempty + buf);
                else mbar_arrive_cluster(tempty_leader0 + buf * 8);
              }
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                float* a = acc + ((2 * b + cc) * 8 + k) * 4;
                float s0, s1, s2, s3;
                mul2(s0, s1, sa4[2 * b], sa4[2 * b], sb2[k].x, sb2[k].y);
                mul2(s2, s3, sa4[2 * b + 1], sa4[2 * b + 1], sb2[k].x, sb2[k].y);
                fma2(a[0], a[1], __uint_as_float(r[4 * k]), __uint_as_float(r[4 * k + 1]), s0, s1);
                fma2(a[2], a[3], __uint_as_float(r[4 * k + 2]), __uint_as_float(r[4 * k + 3]), s2, s3);
              }
            }
          }
        }
        // hand the TMEM buffer back: every thread arrives once its own TMEM loads are
        // complete; the scale batch likewise after its last slice
        if (!kColScaleB) {
          tc_fence_before();
          if (rank == 0) mbar_arrive(tempty + buf);
          else mbar_arrive_cluster(tempty_leader0 + buf * 8);
        }
        if (j == sc_batch<kColScaleB>() - 1 || kb == p.kblocks - 1) {
          mbar_arrive(sempty + sci);
          if (++sci == sc_slots<kColScaleB>()) { sci = 0; scph ^= 1; }
        }
        ++it;
      }
      if (!ok) break;
      // epilogue: BF16 rows into this warp's two swizzled 32 x 64 boxes, then TMA stores
      // (fp32 accumulate: four 32 x 32 boxes, two at a time, added by TMA reduce)
      const int wrow0 = row0 + wq * 32;
      if (wrow0 < p.M && lo_ok) {
        if constexpr (kAccF32) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {  // tile columns col_lo (hh = 0) / col_hi, 64 each
            if (stored) {  // the previous boxes must have been read
              if (lane == 0) tma_store_wait_read();
              __syncwarp();
            }
            if constexpr (kColScaleB) {  // the 16x256b layout (see the promotion)
#pragma unroll
              for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
#pragma unroll
                  for (int k = 0; k < 8; ++k) {
                    const int rr = 16 * b + 8 * hi + (lane >> 2);
                    const float* a = acc + ((2 * b + hh) * 8 + k) * 4 + 2 * hi;
                    const int chunk = 2 * (k & 3) + ((lane & 3) >> 1);
                    uint8_t* box = (k >> 2) ? out1 : out0;
                    *reinterpret_cast<uint2*>(box + rr * 128 + ((chunk ^ (rr & 7)) << 4) + 8 * (lane & 1)) =
                        make_uint2(__float_as_uint(a[0]), __float_as_uint(a[1]));
                  }
            } else {
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                uint8_t* box = j ? out1 : out0;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const float* a = acc + hh * 64 + j * 32 + c * 4;
                  *reinterpret_cast<uint4*>(box + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                      make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                                 __float_as_uint(a[3]));
                }
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && (hh == 0 || hi_ok)) {
              const int cb = hh ? col_hi : col_lo;
              tma_reduce_add_2d(&tmY, out0, cb, wrow0);
              if (cb + 32 < p.N) tma_reduce_add_2d(&tmY, out1, cb + 32, wrow0);  // ragged N
              tma_store_commit();
            }
            stored = true;
          }
        } else {
          if (stored) {  // the previous tile's stores must have read the boxes
            if (lane == 0) tma_store_wait_read();
            __syncwarp();
          }
          if constexpr (kColScaleB) {  // the 16x256b layout (see the promotion)
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
              for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
#pragma unroll
                  for (int k = 0; k < 8; ++k) {
                    const int rr = 16 * b + 8 * hi + (lane >> 2);
                    const float* a = acc + ((2 * b + cc) * 8 + k) * 4 + 2 * hi;
                    uint8_t* box = cc ? out1 : out0;
                    *reinterpret_cast<uint32_t*>(box + rr * 128 + ((k ^ (rr & 7)) << 4) + 4 * (lane & 3)) =
                        pack_bf16x2(a[0], a[1]);
                  }
          } else {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              uint8_t* box = j ? out1 : out0;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const float* a = acc + j * 64 + c * 8;
                uint4 v;
                v.x = pack_bf16x2(a[0], a[1]);
                v.y = pack_bf16x2(a[2], a[3]);
                v.z = pack_bf16x2(a[4], a[5]);
                v.w = pack_bf16x2(a[6], a[7]);
                *reinterpret_cast<uint4*>(box + lane * 128 + ((c ^ (lane & 7)) << 4)) = v;
              }
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, out0, col_lo, wrow0);
            if (hi_ok) tma_store_2d(&tmY, out1, col_hi, wrow0);
            tma_store_commit();
          }
          stored = true;
        }
      }
    }
    if (stored && lane == 0) tma_store_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair<kTmemCols>(tmem_base);
  }
}

// Per device and kernel variant: opt in to the shared memory, check the register
// budget of the hand-over, and find how many CTA pairs can be resident at once (pairs
// are placed within one GPC, so this can be below half the SM count). Returns that
// number, or 0 on failure (the reason is in fp8q_last_error_message).
template <bool kCol, bool kAcc = false>
int kernel_setup() {
  // written once per device under the lock; host threads may launch concurrently
  static std::atomic<int> pairs_for_device[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (const int known = pairs_for_device[dev].load(std::memory_order_acquire)) return known;
  std::lock_guard<std::mutex> lock(mu);
  if (const int known = pairs_for_device[dev].load(std::memory_order_relaxed)) return known;
  const cudaError_t e = cudaFuncSetAttribute(
      gemm_kernel<kCol, kAcc>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(gemm max dynamic smem)", e);
    cudaGetLastError();
    return 0;
  }
  // The register hand-over inside the kernel waits until the block's launch allocation
  // covers the new budgets; refuse to launch a build whose allocation would not.
  cudaFuncAttributes attr;
  const cudaError_t ea = cudaFuncGetAttributes(&attr, gemm_kernel<kCol, kAcc>);
  if (ea != cudaSuccess) {
    set_last_error("cudaFuncGetAttributes(gemm)", ea);
    cudaGetLastError();
    return 0;
  }
  if (static_cast<uint32_t>(attr.numRegs) * kThreads <
          regs_control<kCol>() * 128 + regs_promote<kCol>() * 256 ||
      attr.maxThreadsPerBlock < kThreads) {
    set_last_error("gemm register budget check", cudaErrorLaunchOutOfResources);
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 74, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int clusters = 0;
  const cudaError_t eo =
      cudaOccupancyMaxActiveClusters(&clusters, gemm_kernel<kCol, kAcc>, &cfg);
  if (eo != cudaSuccess || clusters <= 0) {
    set_last_error("cudaOccupancyMaxActiveClusters(gemm)", eo != cudaSuccess ? eo : cudaErrorInvalidConfiguration);
    cudaGetLastError();
    return 0;
  }
  pairs_for_device[dev].store(clusters, std::memory_order_release);
  return clusters;
}

// out [Mg][Ng] = A [Mg][Kg] x B [Ng][Kg]^T with the scales described above; out is BF16
// (y: uint16_t) or, with kAcc, an fp32 array the product is added to (y: float).
template <bool kCol, bool kAcc = false>
fp8q_status launch_gemm(const uint8_t* A, const uint8_t* B, int64_t Mg, int64_t Ng, int64_t Kg,
                        const float* sa, int64_t ldsa, const float* sb, int64_t sb_sj,
                        int64_t sb_sr, const float* sbcol, void* y, int64_t ldy,
                        cudaStream_t stream) {
  const int sms = sm100_sm_count();
  if (!sms) return FP8Q_ERR_UNSUPPORTED;
  if (Mg > 0x7FFFFFFF || Ng > 0x7FFFFFFF || Kg > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  // 128-wide K slices; a partial last slice (Kg not a multiple of 128) is zero-filled
  // by the tensor copies, which adds nothing to any dot product
  const int64_t kslices = (Kg + BK - 1) / BK;
  CUtensorMap tmA, tmB, tmSA, tmSB, tmY;
  bool ok = encode_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, Kg, Mg, Kg, BK, BM,
                           CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, Kg, Ng, Kg, BK, BN / 2,
                           CU_TENSOR_MAP_SWIZZLE_128B) &&
            (kAcc ? encode_tmap_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, y, Ng, Mg, ldy * 4, 32,
                                   32, CU_TENSOR_MAP_SWIZZLE_128B)
                  : encode_tmap_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, Ng, Mg, ldy * 2, 64,
                                   32, CU_TENSOR_MAP_SWIZZLE_128B)) &&
            encode_tmap_2d(&tmSA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sa, Mg, kslices, ldsa * 4, BM,
                           sc_batch<kCol>(), CU_TENSOR_MAP_SWIZZLE_NONE);
  // (scale batches past the last slice read the copies' zero fill)
  if (ok && kCol)
    ok = encode_tmap_2d(&tmSB, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sbcol, Ng, kslices, Ng * 4, BN,
                        sc_batch<kCol>(), CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    tmSB = tmSA;
  if (!ok) return FP8Q_ERR_UNSUPPORTED;
  const int max_pairs = kernel_setup<kCol, kAcc>();
  if (max_pairs <= 0) return FP8Q_ERR_CUDA;

  GemmParams p;
  p.M = static_cast<int32_t>(Mg);
  p.N = static_cast<int32_t>(Ng);
  p.K = static_cast<int32_t>(Kg);
  p.mblocks = static_cast<int32_t>((Mg + kPairM - 1) / kPairM);
  p.nblocks = static_cast<int32_t>((Ng + BN - 1) / BN);
  p.kblocks = static_cast<int32_t>(kslices);
  {
    const double a_bytes = static_cast<double>(Mg) * Kg, b_bytes = static_cast<double>(Ng) * Kg;
    if (std::min(a_bytes, b_bytes) <= 48e6) {  // the smaller operand stays in L2
      p.swap = b_bytes <= a_bytes ? 0 : 1;
      p.group = p.swap ? p.mblocks : p.nblocks;
    } else {
      p.swap = 0;
      p.group = std::min<int32_t>(8, p.nblocks);
    }
  }
  p.sb = sb;
  p.sb_sj = sb_sj;
  p.sb_sr = sb_sr;
  p.y = static_cast<uint16_t*>(y);
  p.ldy = ldy;
  p.err = device_error_word();
  p.wait_limit_ns = kWaitLimitNs;
  if (!p.err) return FP8Q_ERR_CUDA;
  const int64_t tiles = static_cast<int64_t>(p.mblocks) * p.nblocks;
  if (tiles > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const int grid = 2 * static_cast<int>(std::min<int64_t>(tiles, max_pairs));
  gemm_kernel<kCol, kAcc><<<grid, kThreads, kSmemBytes, stream>>>(tmA, tmB, tmSA, tmSB,
                                                                           tmY, p);
  return launch_status("gemm_kernel launch");
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" fp8q_status fp8q_linear_fwd(const uint8_t* qa, const float* sa, int64_t ldsa,
                                       const uint8_t* qw, const float* sw, int64_t M, int64_t N,
                                       int64_t K, uint16_t* y, int64_t ldy, void* stream) {
  if (!qa || !sa || !qw || !sw || !y) return FP8Q_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || N % 16 || K % 16 || ldsa < M || ldy < N)
    return FP8Q_ERR_SHAPE;
  if (!aligned16(qa) || !aligned16(sa) || !aligned16(qw) || !aligned16(sw) || !aligned16(y) ||
      ldsa % 4 || ldy % 8)
    return FP8Q_ERR_ALIGN;
  // B = W [N][K]; block scale of (n, slice r) = sw[(n/128)*KB + r], KB = ceil(K/128).
  // The skinny kernel reads whole 128-wide slices and strips: ragged shapes take the
  // pair kernel at any M (the same arithmetic in the same order).
  const int64_t KB = (K + 127) / 128;
  if (M <= kSkinnyMaxM && K % 128 == 0 && N % 128 == 0)
    return launch_skinny_gemm(qa, qw, M, N, K, sa, ldsa, sw, KB, 1, y, ldy,
                              static_cast<cudaStream_t>(stream));
  return launch_gemm<false>(qa, qw, M, N, K, sa, ldsa, sw, KB, 1, nullptr, y, ldy,
                            static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_linear_dgrad(const uint8_t* qdy, const float* sdy, int64_t ldsdy,
                                         const uint8_t* qwT, const float* sw, int64_t M,
                                         int64_t N, int64_t K, uint16_t* dx, int64_t lddx,
                                         void* stream) {
  if (!qdy || !sdy || !qwT || !sw || !dx) return FP8Q_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || N % 16 || K % 16 || ldsdy < M || lddx < K)
    return FP8Q_ERR_SHAPE;
  if (!aligned16(qdy) || !aligned16(sdy) || !aligned16(qwT) || !aligned16(sw) ||
      !aligned16(dx) || ldsdy % 4 || lddx % 8)
    return FP8Q_ERR_ALIGN;
  // GEMM rows = M, columns = K, reduction = N. B = W^T [K][N];
  // block scale of (k, slice r over n) = sw[r*KB + k/128], KB = ceil(K/128)
  const int64_t KB = (K + 127) / 128;
  if (M <= kSkinnyMaxM && K % 128 == 0 && N % 128 == 0)
    return launch_skinny_gemm(qdy, qwT, M, K, N, sdy, ldsdy, sw, 1, KB, dx, lddx,
                              static_cast<cudaStream_t>(stream));
  return launch_gemm<false>(qdy, qwT, M, K, N, sdy, ldsdy, sw, 1, KB, nullptr, dx, lddx,
                            static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_linear_wgrad(const uint8_t* qdyT, const float* sdy_c,
                                         const uint8_t* qxT, const float* sx_c, int64_t M,
                                         int64_t N, int64_t K, uint16_t* dw, int64_t lddw,
                                         void* stream) {
  if (!qdyT || !sdy_c || !qxT || !sx_c || !dw) return FP8Q_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || M % 16 || N % 16 || K % 16 || lddw < K)
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

extern "C" fp8q_status fp8q_linear_wgrad_acc_f32(const uint8_t* qdyT, const float* sdy_c,
                                                 const uint8_t* qxT, const float* sx_c, int64_t M,
                                                 int64_t N, int64_t K, float* dw, int64_t lddw,
                                                 void* stream) {
  if (!qdyT || !sdy_c || !qxT || !sx_c || !dw) return FP8Q_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || M % 16 || N % 16 || K % 16 || lddw < K)
    return FP8Q_ERR_SHAPE;
  if (!aligned16(qdyT) || !aligned16(sdy_c) || !aligned16(qxT) || !aligned16(sx_c) ||
      !aligned16(dw) || lddw % 4)
    return FP8Q_ERR_ALIGN;
  // as fp8q_linear_wgrad, with dw += the fp32 accumulator instead of dw = bf16(it)
  return launch_gemm<true, true>(qdyT, qxT, N, K, M, sdy_c, N, nullptr, 0, 0, sx_c, dw,
                                        lddw, static_cast<cudaStream_t>(stream));
}
