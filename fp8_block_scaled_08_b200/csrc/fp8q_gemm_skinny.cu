// Skinny-M block-scaled FP8 GEMM for sm_100a: the forward (and DGrad) of the linear
// layer when the token batch is small (decode, M <= 256).
//
//   out[i, j] = sum_r  sA(i, r) * sB(j / 128, r) * sum_{l in slice r} qA[i, l] * qB[j, l]
//
// with the same operands, scales and promotion order as the large-tile kernel
// ("Resumen Técnico: Jet-RL", section "Esquema de Cuantización": 1x128 activation
// groups, 128x128 weight blocks). At these sizes the layer is bound by reading the
// FP8 weights (about 2M flops per weight byte, far below the tensor-core ridge), so the
// design goal is many SMs streaming weights at once with enough bytes in flight:
//
//  * Each CTA owns a narrow strip of kBN (16, 32 or 64) weight rows and at most 128
//    token rows, over the whole K. Strips are independent: no split-K, so every output
//    element is promoted slice after slice in increasing r, exactly as in the
//    large-tile kernel (acc = fma(P_r, sA*sB, acc) from +0), and a row of the output has
//    the same bits whatever M is ("Arquitectura Central": the rollout graph is a
//    subgraph of the training graph).
//  * tcgen05.mma.cta_group::1, M = 128 (token rows; rows past the batch are left as
//    whatever the shared-memory tile holds and their accumulator lanes are never read),
//    N = kBN, K = 32, four per 128-wide slice, into one of up to 8 TMEM accumulator
//    buffers, so the tensor core runs ahead of the promotion by several slices.
//  * A TMA ring of "super-stages" of G consecutive K-slices, about 96 KB of shared
//    memory so that two CTAs fit on an SM. One 3D tensor copy per operand brings G
//    slices at once (dimensions: 128 bytes of a slice, rows, slice index; the slice
//    stride is 128 bytes), so each row of the strip is read as one G*128-byte run: with
//    one 128-byte piece per row and slice, the weight stream is scattered over DRAM
//    pages and ran below a third of the HBM bandwidth. The row scales of a super-stage
//    arrive by TMA in a ring of their own (released by the promotion warps, since they
//    outlive the stage), and the strip's KB block scales are read into shared memory
//    once, so the promotion loop never waits on a global load.
//  * 224 threads: warp 0 TMA producer; warps 1 and 2 issue the MMAs, alternating
//    slices (warp 1 also allocates TMEM); warps 3-6 promotion (warp w reads TMEM lanes
//    32*(w%4) .. +31; only the quarters that hold token rows work). One issuing thread
//    needs ~70 cycles per MMA instruction and ~700 per slice in all (measured), which
//    with narrow strips would cap the weight stream at N*128 bytes per 700 cycles; each
//    slice is an independent 4-MMA group into its own TMEM buffer, so two threads can
//    issue alternate slices. Promotion adds each slice into kBN fp32 registers per
//    thread; the epilogue rounds to BF16 and stores each token row's kBN outputs.
// Every mbarrier wait is bounded; a wait that gives up records FP8Q_ERR_TIMEOUT in the
// device error word and the CTA winds down.
#include <algorithm>
#include <cstdio>
#include <atomic>
#include <mutex>

#include "fp8q_device.cuh"
#include "fp8q_host.h"

namespace fp8q {
namespace {

constexpr int kSkIssuers = 2;                      // MMA-issuing warps
constexpr int kSkThreads = 32 * (1 + kSkIssuers + 4);
constexpr int kSkBK = 128;
constexpr int kSkMaxStages = 8;
constexpr int kSkMaxG = 8;
constexpr uint32_t kSkSmemTarget = 96 * 1024;
constexpr uint32_t kSkATileRead = 128 * kSkBK;  // the MMA reads 128 rows of A
constexpr int kSkScRing = 8;                     // row-scale slots (one per super-stage)

struct SkinnyParams {
  int32_t M, N, kblocks;
  int32_t mtiles;
  int32_t stages;             // super-stages in the ring
  int32_t G;                  // K-slices per super-stage
  uint32_t a_slice, b_slice;  // bytes of one slice of A / B (1024-aligned)
  uint32_t a_rows;            // token rows per A box
  uint32_t off_b;             // start of the B ring
  uint32_t off_sa;            // row-scale ring: kSkScRing slots of sa_slot bytes
  uint32_t sa_slot;           // G * a_rows * 4 rounded up to 128 (TMA destination alignment)
  uint32_t off_sb;            // block scales of the strip: kblocks fp32
  uint32_t off_bars;
  const float* sa;
  int64_t ldsa;
  const float* sb;
  int64_t sb_sj, sb_sr;
  uint16_t* y;
  int64_t ldy;
  int32_t splits;         // CTAs per output strip along K (split variant)
  float* ws_partials;     // [strip][kb][M][kBN] raw slice products (split variant)
  unsigned* ws_counters;  // [strip] finished CTAs (split variant; zero between calls)
  unsigned* err;
  uint64_t wait_limit_ns;
};

template <int kBN>
struct SkinnyShape {
  static constexpr int kBufs = (kBN * 8 <= 256) ? 8 : 256 / kBN;  // accumulator buffers
  static constexpr uint32_t kTmemCols = kBufs * kBN < 32 ? 32 : kBufs * kBN;
  static_assert(kBN % 16 == 0 && kBN >= 16 && kBN <= 64, "N of a cta_group::1 M=128 MMA");
  static_assert((kTmemCols & (kTmemCols - 1)) == 0, "TMEM allocations are powers of two");
};

__device__ __forceinline__ void sk_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

template <int kBN>
__device__ __forceinline__ void sk_tmem_load(uint32_t taddr, uint32_t (&r)[kBN]) {
  if constexpr (kBN == 16) {
    tmem_ld16(taddr, r);
  } else {
#pragma unroll
    for (int c = 0; c < kBN / 32; ++c)
      tmem_ld32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
  }
  tmem_wait_ld();
}

template <int kBN, bool kSplit>
__global__ void __launch_bounds__(kSkThreads) skinny_gemm_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const __grid_constant__ CUtensorMap tmSA, const SkinnyParams p) {
  using Shape = SkinnyShape<kBN>;
  constexpr int kBufs = Shape::kBufs;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int last_flag;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int S = p.stages, G = p.G, KB = p.kblocks;
  const uint32_t a_stage = G * p.a_slice, b_stage = G * p.b_slice;
  uint8_t* a_ring = smem;
  uint8_t* b_ring = smem + p.off_b;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  uint64_t* empty = full + kSkMaxStages;
  uint64_t* tfull = empty + kSkMaxStages;
  uint64_t* tempty = tfull + kBufs;
  uint64_t* sfull = tempty + kBufs;
  uint64_t* sempty = sfull + kSkScRing;
  uint64_t* done = sempty + kSkScRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sb_s = reinterpret_cast<float*>(smem + p.off_sb);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA -> (output strip, part of K); the CTAs of one strip are adjacent
  const int tile = kSplit ? static_cast<int>(blockIdx.x) / p.splits : static_cast<int>(blockIdx.x);
  const int part = kSplit ? static_cast<int>(blockIdx.x) % p.splits : 0;
  const int mt = tile % p.mtiles;
  const int nt = tile / p.mtiles;
  const int m0 = mt * 128;
  const int n0 = nt * kBN;
  const int rows = min(128, p.M - m0);       // token rows of this tile
  const int quarters = (rows + 31) >> 5;     // TMEM lane quarters that hold them
  const int kb_begin = kSplit ? (part * KB) / p.splits : 0;
  const int nsl = (kSplit ? ((part + 1) * KB) / p.splits : KB) - kb_begin;  // slices here
  const int nst = (nsl + G - 1) / G;         // super-stages

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kSkIssuers);  // each issuer commits once per super-stage
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, quarters);
    }
    for (int i = 0; i < kSkScRing; ++i) {
      mbar_init(sfull + i, 1);
      mbar_init(sempty + i, quarters);
    }
    mbar_init(done, kSkIssuers);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (!kSplit) prefetch_tensormap(&tmSA);
  }
  if (warp == 1) tmem_alloc<Shape::kTmemCols>(tmem_slot);
  if (!kSplit) {  // block scales of this strip, one per slice
    const float* sbp = p.sb + static_cast<int64_t>(n0 / 128) * p.sb_sj;
    for (int kb = threadIdx.x; kb < KB; kb += kSkThreads)
      sb_s[kb] = __ldg(sbp + static_cast<int64_t>(kb) * p.sb_sr);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.err, p.wait_limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // slices past K (the last super-stage may be partial) read as zeros, and the
      // transaction count is the full box either way
      const uint32_t stage_tx = G * (p.a_rows * kSkBK + kBN * kSkBK);
      int issued = 0, sc_issued = 0;
      bool ok = true;
      for (int st = 0; st < nst; ++st) {
        const int s = st % S;
        const int z = kb_begin + st * G;
        if (!mbar_wait(empty + s, (static_cast<uint32_t>(st / S) & 1u) ^ 1u, ctl)) { ok = false; break; }
        mbar_arrive_expect_tx(full + s, stage_tx);
        tma_load_3d(a_ring + s * a_stage, &tmA, 0, m0, z, full + s);
        tma_load_3d(b_ring + s * b_stage, &tmB, 0, n0, z, full + s);
        issued = st + 1;
        if (kSplit) continue;  // raw products: no scales here
        const int si = st % kSkScRing;
        if (!mbar_wait(sempty + si, (static_cast<uint32_t>(st / kSkScRing) & 1u) ^ 1u, ctl)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(sfull + si, G * p.a_rows * 4u);
        tma_load_2d(smem + p.off_sa + si * p.sa_slot, &tmSA, m0, z, sfull + si);
        sc_issued = st + 1;
      }
      if (!ok) {  // let the copies still in flight land before the CTA exits
        for (int st = max(0, issued - S); st < issued; ++st)
          sk_wait_drain(full + st % S, static_cast<uint32_t>(st / S) & 1u, p.wait_limit_ns);
        for (int st = max(0, sc_issued - kSkScRing); st < sc_issued; ++st)
          sk_wait_drain(sfull + st % kSkScRing, static_cast<uint32_t>(st / kSkScRing) & 1u,
                        p.wait_limit_ns);
      }
    }
    __syncwarp();
  } else if (warp <= kSkIssuers) {
    // ------------------------------------------------------------ MMA issuers
    // issuer i = warp - 1 takes the slices i, i + kSkIssuers, ... of this CTA
    if (lane == 0) {
      const int issuer = warp - 1;
      const uint32_t idesc = idesc_e4m3_f32(128, kBN);
      bool ok = true;
      for (int st = 0; ok && st < nst; ++st) {
        const int s = st % S;
        if (!mbar_wait(full + s, static_cast<uint32_t>(st / S) & 1u, ctl)) { ok = false; break; }
        for (int j = 0; j < G; ++j) {
          const int i = st * G + j;  // slice number within this CTA
          if (i >= nsl) break;
          if (i % kSkIssuers != issuer) continue;
          const int buf = i % kBufs;
          const uint32_t tph = static_cast<uint32_t>(i / kBufs) & 1u;
          if (!mbar_wait(tempty + buf, tph ^ 1u, ctl)) { ok = false; break; }
          tc_fence_after();
          mma_f8f6f4_slice(tmem_base + buf * kBN,
                           smem_desc_k_sw128(smem_u32(a_ring + s * a_stage + j * p.a_slice)),
                           smem_desc_k_sw128(smem_u32(b_ring + s * b_stage + j * p.b_slice)), idesc);
          mma_commit(tfull + buf);
        }
        // this issuer's reads of the super-stage are done when its MMAs are
        if (ok) mma_commit(empty + s);
      }
      // every MMA this thread issued has finished reading shared memory and writing TMEM
      mma_commit(done);
      sk_wait_drain(done, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ promotion + epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    if (q < quarters) {
      const int row = q * 32 + lane;
      const int m = m0 + row;
      const bool row_ok = m < p.M;
      const int srow = row < static_cast<int>(p.a_rows) ? row : 0;
      float acc[kBN];
#pragma unroll
      for (int c = 0; c < kBN; ++c) acc[c] = 0.0f;
      bool ok = true;
      for (int i = 0; i < nsl; ++i) {
        float s = 0.0f;
        if (!kSplit) {
          const int st = i / G, j = i - st * G;
          const int si = st % kSkScRing;
          if (j == 0 &&
              !mbar_wait_warp(sfull + si, static_cast<uint32_t>(st / kSkScRing) & 1u, ctl)) {
            ok = false;
            break;
          }
          const float sa =
              reinterpret_cast<const float*>(smem + p.off_sa + si * p.sa_slot)[j * p.a_rows + srow];
          s = __fmul_rn(sa, sb_s[i]);
          if (j == G - 1 || i == nsl - 1) {  // last use of this super-stage's scales
            __syncwarp();
            if (lane == 0) mbar_arrive(sempty + si);
          }
        }
        const int buf = i % kBufs;
        const uint32_t tph = static_cast<uint32_t>(i / kBufs) & 1u;
        if (!mbar_wait_warp(tfull + buf, tph, ctl)) { ok = false; break; }
        tc_fence_after();
        uint32_t r[kBN];
        sk_tmem_load<kBN>(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kBN, r);
        if (kSplit) {
          if (row_ok) {  // raw products of slice kb_begin + i, row m: kBN fp32
            uint4* dst = reinterpret_cast<uint4*>(
                p.ws_partials + ((static_cast<int64_t>(tile) * KB + kb_begin + i) * p.M + m) * kBN);
#pragma unroll
            for (int c = 0; c < kBN / 4; ++c)
              dst[c] = make_uint4(r[4 * c], r[4 * c + 1], r[4 * c + 2], r[4 * c + 3]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < kBN; c += 2)
            fma2(acc[c], acc[c + 1], __uint_as_float(r[c]), __uint_as_float(r[c + 1]), s, s);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty + buf);
      }
      if (!kSplit && ok && row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(p.y + static_cast<int64_t>(m) * p.ldy + n0);
#pragma unroll
        for (int c = 0; c < kBN / 8; ++c) {
          const float* a = acc + 8 * c;
          dst[c] = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                              pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<Shape::kTmemCols>(tmem_base);
  }
  if (kSplit) {
    // Every thread of this CTA has written its partials (barrier above). The CTA that
    // completes the strip's count promotes all its slices in order and resets the count.
    if (threadIdx.x == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(p.ws_counters + tile, 1u);
      last_flag = (prev == static_cast<unsigned>(p.splits - 1)) ? 1 : 0;
      if (last_flag) atomicExch(p.ws_counters + tile, 0u);
    }
    __syncthreads();
    if (last_flag) {
      __threadfence();
      // scale products sa * sb of every (slice, row) of the strip, in the shared memory
      // the stages no longer use (the launch checks it fits: KB * M floats)
      float* sc = reinterpret_cast<float*>(smem);
      const float* sbp = p.sb + static_cast<int64_t>(n0 / 128) * p.sb_sj;
      for (int idx = threadIdx.x; idx < KB * rows; idx += kSkThreads) {
        const int kb = idx / rows, mr = idx - kb * rows;
        sc[idx] = __fmul_rn(__ldg(p.sa + static_cast<int64_t>(kb) * p.ldsa + m0 + mr),
                            __ldg(sbp + static_cast<int64_t>(kb) * p.sb_sr));
      }
      __syncthreads();
      // each output: the partials of all slices in increasing kb, 16 loads in flight
      constexpr int kBatch = 16;
      const int64_t pstride = static_cast<int64_t>(p.M) * kBN;
      for (int idx = threadIdx.x; idx < rows * kBN; idx += kSkThreads) {
        const int mr = idx / kBN, c = idx % kBN;
        const float* pp = p.ws_partials + (static_cast<int64_t>(tile) * KB * p.M + m0 + mr) * kBN + c;
        float acc = 0.0f;
        for (int kb0 = 0; kb0 < KB; kb0 += kBatch) {
          float part[kBatch];
#pragma unroll
          for (int j = 0; j < kBatch; ++j)
            part[j] = (kb0 + j < KB) ? __ldcg(pp + (kb0 + j) * pstride) : 0.0f;
#pragma unroll
          for (int j = 0; j < kBatch; ++j)
            if (kb0 + j < KB) acc = __fmaf_rn(part[j], sc[(kb0 + j) * rows + mr], acc);
        }
        p.y[static_cast<int64_t>(m0 + mr) * p.ldy + n0 + c] =
            static_cast<uint16_t>(pack_bf16x2(acc, 0.0f) & 0xFFFFu);
      }
    }
  }
}

// Per device and kernel variant: opt in to the shared memory the launch asks for.
// Per device and kernel variant: the dynamic shared memory opted in so far (host threads
// launching on different streams may get here at once: reads are atomic, updates locked).
template <int kBN, bool kSplit>
bool skinny_setup(size_t smem_bytes) {
  static std::atomic<size_t> opted[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (opted[dev].load(std::memory_order_acquire) >= smem_bytes) return true;
  std::lock_guard<std::mutex> lock(mu);
  if (opted[dev].load(std::memory_order_relaxed) >= smem_bytes) return true;
  const cudaError_t e = cudaFuncSetAttribute(skinny_gemm_kernel<kBN, kSplit>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem_bytes));
  if (e != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(skinny_gemm)", e);
    cudaGetLastError();
    return false;
  }
  opted[dev].store(smem_bytes, std::memory_order_release);
  return true;
}

template <int kBN, bool kSplit>
fp8q_status launch_skinny(const uint8_t* A, int64_t Mg, const float* sa, int64_t ldsa,
                          const uint8_t* B, int64_t Ng, int64_t Kg, SkinnyParams p,
                          cudaStream_t stream) {
  using Shape = SkinnyShape<kBN>;
  p.b_slice = kBN * kSkBK;  // 16 rows x 128 B = 2 KB: a multiple of the 1024-byte atom
  const uint32_t per_slice = p.a_slice + p.b_slice;
  // G slices per super-stage: up to 8 and at least two super-stages in the ring; when K
  // is split, G divides each CTA's share (the splits divide the slice count), so no
  // copy reaches into the next CTA's slices
  p.G = static_cast<int32_t>(std::clamp<uint32_t>(kSkSmemTarget / 2 / per_slice, 1u,
                                                  static_cast<uint32_t>(kSkMaxG)));
  if (kSplit) {
    const int32_t share = p.kblocks / p.splits;
    while (share % p.G) --p.G;
  }
  p.stages = static_cast<int32_t>(std::clamp<uint32_t>(kSkSmemTarget / (p.G * per_slice), 2u,
                                                       static_cast<uint32_t>(kSkMaxStages)));
  const uint32_t a_stage = p.G * p.a_slice, b_stage = p.G * p.b_slice;
  p.off_b = p.stages * a_stage;
  uint32_t data = p.off_b + p.stages * b_stage;
  // the MMA reads 128 rows from the last A slice: keep that inside the allocation
  data = std::max<uint32_t>(data, (p.stages - 1) * a_stage + (p.G - 1) * p.a_slice + kSkATileRead);
  // every TMA destination in shared memory starts on a 128-byte boundary
  p.sa_slot = (p.G * p.a_rows * 4u + 127u) & ~127u;
  p.off_sa = (data + 127u) & ~127u;
  p.off_sb = p.off_sa + kSkScRing * p.sa_slot;
  p.off_bars = (p.off_sb + static_cast<uint32_t>(p.kblocks) * 4u + 7u) & ~7u;
  if (p.a_slice % 1024u || p.b_slice % 1024u || p.off_b % 1024u || p.off_sa % 128u ||
      p.sa_slot % 128u)
    return FP8Q_ERR_UNSUPPORTED;
  if (kSplit) {  // the last CTA's scale table reuses the stage memory: make it fit
    const uint64_t table = static_cast<uint64_t>(p.kblocks) * static_cast<uint64_t>(Mg) * 4u;
    if (table > p.off_sa) {
      if (table > 200u * 1024u) return FP8Q_ERR_UNSUPPORTED;
      p.off_sa = static_cast<uint32_t>((table + 127u) & ~127ull);
      p.off_sb = p.off_sa + kSkScRing * p.sa_slot;
      p.off_bars = (p.off_sb + static_cast<uint32_t>(p.kblocks) * 4u + 7u) & ~7u;
    }
  }
  const uint32_t bars = (2 * kSkMaxStages + 2 * Shape::kBufs + 2 * kSkScRing + 1) * 8 + 16;
  const size_t smem = p.off_bars + bars + 1024;
  if (smem > 232448) return FP8Q_ERR_UNSUPPORTED;
  // A and W as (128 bytes of a slice, rows, slice index): one copy brings G slices of
  // a row block; the row-scale box covers the same G slices
  CUtensorMap tmA, tmB, tmSA;
  const uint64_t kslices = static_cast<uint64_t>(Kg / kSkBK);
  const uint64_t strides[2] = {static_cast<uint64_t>(Kg), static_cast<uint64_t>(kSkBK)};
  const uint64_t dims_a[3] = {static_cast<uint64_t>(kSkBK), static_cast<uint64_t>(Mg), kslices};
  const uint64_t dims_b[3] = {static_cast<uint64_t>(kSkBK), static_cast<uint64_t>(Ng), kslices};
  const uint32_t box_a[3] = {static_cast<uint32_t>(kSkBK), p.a_rows, static_cast<uint32_t>(p.G)};
  const uint32_t box_b[3] = {static_cast<uint32_t>(kSkBK), static_cast<uint32_t>(kBN),
                             static_cast<uint32_t>(p.G)};
  if (!encode_tmap_3d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, dims_a, strides, box_a,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_3d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, dims_b, strides, box_b,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tmSA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sa, Mg, kslices, ldsa * 4, p.a_rows,
                      static_cast<uint32_t>(p.G), CU_TENSOR_MAP_SWIZZLE_NONE))
    return FP8Q_ERR_UNSUPPORTED;
  if (!skinny_setup<kBN, kSplit>(smem)) return FP8Q_ERR_CUDA;
  const int64_t grid = static_cast<int64_t>(p.mtiles) * (Ng / kBN) * (kSplit ? p.splits : 1);
  if (grid > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  skinny_gemm_kernel<kBN, kSplit><<<static_cast<unsigned>(grid), kSkThreads, smem, stream>>>(
      tmA, tmB, tmSA, p);
  return launch_status("skinny_gemm_kernel launch");
}

}  // namespace

fp8q_status launch_skinny_gemm(const uint8_t* A, const uint8_t* B, int64_t Mg, int64_t Ng,
                               int64_t Kg, const float* sa, int64_t ldsa, const float* sb,
                               int64_t sb_sj, int64_t sb_sr, uint16_t* y, int64_t ldy,
                               cudaStream_t stream) {
  const int sms = sm100_sm_count();
  if (!sms) return FP8Q_ERR_UNSUPPORTED;
  if (Mg <= 0 || Mg > kSkinnyMaxM || Ng % 128 || Kg % 128 || Ng > 0x7FFFFFFF ||
      Kg > 0x7FFFFFFF)
    return FP8Q_ERR_SHAPE;
  SkinnyParams p;
  p.M = static_cast<int32_t>(Mg);
  p.N = static_cast<int32_t>(Ng);
  p.kblocks = static_cast<int32_t>(Kg / kSkBK);
  p.mtiles = static_cast<int32_t>((Mg + 127) / 128);
  // A box: the token rows (a multiple of 8, at most 128); rows past M read as zeros
  p.a_rows = static_cast<uint32_t>(std::min<int64_t>(128, (Mg + 7) / 8 * 8));
  p.a_slice = p.a_rows * kSkBK;  // a multiple of 1024 since a_rows is a multiple of 8
  p.sa = sa;
  p.ldsa = ldsa;
  p.splits = 1;
  p.ws_partials = nullptr;
  p.ws_counters = nullptr;
  p.sb = sb;
  p.sb_sj = sb_sj;
  p.sb_sr = sb_sr;
  p.y = y;
  p.ldy = ldy;
  p.err = device_error_word();
  p.wait_limit_ns = kWaitLimitNs;
  if (!p.err) return FP8Q_ERR_CUDA;
  // Strip width: the widest strip that still gives every SM at least one CTA (wider
  // strips re-read the token rows from L2 fewer times); 16 if none does.
  const int64_t mt = p.mtiles;
  if (mt * (Ng / 64) >= sms) return launch_skinny<64, false>(A, Mg, sa, ldsa, B, Ng, Kg, p, stream);
  if (mt * (Ng / 32) >= sms) return launch_skinny<32, false>(A, Mg, sa, ldsa, B, Ng, Kg, p, stream);
  return launch_skinny<16, false>(A, Mg, sa, ldsa, B, Ng, Kg, p, stream);
}

// Split variant: 64-column strips, K divided over `splits` CTAs per strip so that the
// grid covers about two CTAs per SM.
constexpr int kSplitBN = 64;

int64_t splitk_counter_bytes(int64_t N) { return (4 * (N / kSplitBN) + 255) / 256 * 256; }

int64_t splitk_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return splitk_counter_bytes(N) + N * (K / kSkBK) * M * 4;
}

fp8q_status launch_skinny_gemm_splitk(const uint8_t* A, const uint8_t* B, int64_t Mg, int64_t Ng,
                                      int64_t Kg, const float* sa, int64_t ldsa, const float* sb,
                                      int64_t sb_sj, int64_t sb_sr, uint16_t* y, int64_t ldy,
                                      void* workspace, int64_t workspace_bytes,
                                      cudaStream_t stream) {
  const int sms = sm100_sm_count();
  if (!sms) return FP8Q_ERR_UNSUPPORTED;
  if (Mg <= 0 || Mg > 128 || Ng % 128 || Kg % 128 || Ng > 0x7FFFFFFF || Kg > 0x7FFFFFFF)
    return FP8Q_ERR_SHAPE;
  const int64_t strips = Ng / kSplitBN;
  const int64_t kblocks = Kg / kSkBK;
  // the smallest divisor of the slice count that gives about two CTAs per SM
  const int64_t target = (2 * sms + strips - 1) / strips;
  int64_t splits = 1;
  if (target > 1) {
    splits = kblocks;
    for (int64_t d = target; d < kblocks; ++d)
      if (kblocks % d == 0) { splits = d; break; }
  }
  if (splits <= 1)  // the strips alone fill the GPU
    return launch_skinny_gemm(A, B, Mg, Ng, Kg, sa, ldsa, sb, sb_sj, sb_sr, y, ldy, stream);
  if (!workspace || !aligned16(workspace)) return workspace ? FP8Q_ERR_ALIGN : FP8Q_ERR_NULL;
  if (workspace_bytes < splitk_workspace_bytes(Mg, Ng, Kg)) return FP8Q_ERR_SHAPE;
  SkinnyParams p;
  p.M = static_cast<int32_t>(Mg);
  p.N = static_cast<int32_t>(Ng);
  p.kblocks = static_cast<int32_t>(kblocks);
  p.mtiles = 1;
  p.a_rows = static_cast<uint32_t>((Mg + 7) / 8 * 8);
  p.a_slice = p.a_rows * kSkBK;
  p.sa = sa;
  p.ldsa = ldsa;
  p.sb = sb;
  p.sb_sj = sb_sj;
  p.sb_sr = sb_sr;
  p.y = y;
  p.ldy = ldy;
  p.splits = static_cast<int32_t>(splits);
  p.ws_counters = static_cast<unsigned*>(workspace);
  p.ws_partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                           splitk_counter_bytes(Ng));
  p.err = device_error_word();
  p.wait_limit_ns = kWaitLimitNs;
  if (!p.err) return FP8Q_ERR_CUDA;
  return launch_skinny<kSplitBN, true>(A, Mg, sa, ldsa, B, Ng, Kg, p, stream);
}

// The split launch with the counters and the partial products at given addresses
// (counters zero on entry; left zero).
fp8q_status launch_skinny_gemm_splitk_into(const uint8_t* A, const uint8_t* B, int64_t Mg,
                                           int64_t Ng, int64_t Kg, const float* sa, int64_t ldsa,
                                           const float* sb, int64_t sb_sj, int64_t sb_sr,
                                           uint16_t* y, int64_t ldy, unsigned* counters,
                                           float* partials, cudaStream_t stream) {
  const int sms = sm100_sm_count();
  if (!sms) return FP8Q_ERR_UNSUPPORTED;
  if (Mg <= 0 || Mg > 128 || Ng % 128 || Kg % 128 || Ng > 0x7FFFFFFF || Kg > 0x7FFFFFFF)
    return FP8Q_ERR_SHAPE;
  const int64_t strips = Ng / kSplitBN;
  const int64_t kblocks = Kg / kSkBK;
  const int64_t target = (2 * sms + strips - 1) / strips;
  int64_t splits = 1;
  if (target > 1) {
    splits = kblocks;
    for (int64_t d = target; d < kblocks; ++d)
      if (kblocks % d == 0) { splits = d; break; }
  }
  if (splits <= 1)  // the strips alone fill the GPU
    return launch_skinny_gemm(A, B, Mg, Ng, Kg, sa, ldsa, sb, sb_sj, sb_sr, y, ldy, stream);
  SkinnyParams p;
  p.M = static_cast<int32_t>(Mg);
  p.N = static_cast<int32_t>(Ng);
  p.kblocks = static_cast<int32_t>(kblocks);
  p.mtiles = 1;
  p.a_rows = static_cast<uint32_t>((Mg + 7) / 8 * 8);
  p.a_slice = p.a_rows * kSkBK;
  p.sa = sa;
  p.ldsa = ldsa;
  p.sb = sb;
  p.sb_sj = sb_sj;
  p.sb_sr = sb_sr;
  p.y = y;
  p.ldy = ldy;
  p.splits = static_cast<int32_t>(splits);
  p.ws_counters = counters;
  p.ws_partials = partials;
  p.err = device_error_word();
  p.wait_limit_ns = kWaitLimitNs;
  if (!p.err) return FP8Q_ERR_CUDA;
  return launch_skinny<kSplitBN, true>(A, Mg, sa, ldsa, B, Ng, Kg, p, stream);
}

}  // namespace fp8q

using namespace fp8q;

extern "C" int64_t fp8q_linear_fwd_splitk_workspace(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || M > 128 || N <= 0 || K <= 0 || N % 128 || K % 128) return 0;
  return splitk_workspace_bytes(M, N, K);
}

extern "C" int64_t fp8q_linear_fwd_splitk_counter_bytes(int64_t M, int64_t N) {
  if (M <= 0 || M > 128 || N <= 0 || N % 128) return 0;
  return splitk_counter_bytes(N);
}

extern "C" fp8q_status fp8q_linear_fwd_splitk(const uint8_t* qa, const float* sa, int64_t ldsa,
                                              const uint8_t* qw, const float* sw, int64_t M,
                                              int64_t N, int64_t K, uint16_t* y, int64_t ldy,
                                              void* workspace, int64_t workspace_bytes,
                                              void* stream) {
  if (!qa || !sa || !qw || !sw || !y) return FP8Q_ERR_NULL;
  if (M <= 0 || M > 128 || N <= 0 || K <= 0 || N % 128 || K % 128 || ldsa < M || ldy < N)
    return FP8Q_ERR_SHAPE;
  if (!aligned16(qa) || !aligned16(sa) || !aligned16(qw) || !aligned16(sw) || !aligned16(y) ||
      ldsa % 4 || ldy % 8)
    return FP8Q_ERR_ALIGN;
  // B = W [N][K]; block scale of (n, slice r) = sw[(n/128)*(K/128) + r]
  return launch_skinny_gemm_splitk(qa, qw, M, N, K, sa, ldsa, sw, K / 128, 1, y, ldy, workspace,
                                   workspace_bytes, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Split-K forward without a caller workspace: the scratch is one static device array
// per device, laid out as a fixed counter area followed by the partial products (fixed
// so that the counters never sit where an earlier call of another shape wrote
// partials). The array is zero when the module loads, the counter area is cleared once
// more per device before its first use, and every completed call leaves the counters
// at zero. All calls on a device share the one array, so calls must not overlap.
// ---------------------------------------------------------------------------
namespace fp8q {
namespace {

constexpr int64_t kNoAllocBytes = 64ll << 20;
constexpr int64_t kNoAllocCounterBytes = 64ll << 10;
static __device__ __align__(256) uint8_t g_noalloc_workspace[kNoAllocBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_address[64] = {nullptr};
bool g_noalloc_cleared[64] = {false};

// The array's address on the current device (looked up once per device, with that
// device current) with its counter area cleared; nullptr on failure (message recorded).
void* noalloc_workspace(cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    set_last_error("cudaGetDevice (static split-K workspace)",
                   e != cudaSuccess ? e : cudaErrorInvalidDevice);
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_address[dev]) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_noalloc_workspace);
    if (e != cudaSuccess || !addr) {
      set_last_error("cudaGetSymbolAddress (static split-K workspace)",
                     e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_address[dev] = addr;
  }
  if (!g_noalloc_cleared[dev]) {
    e = cudaMemsetAsync(g_noalloc_address[dev], 0, kNoAllocCounterBytes, stream);
    if (e != cudaSuccess) {
      set_last_error("cudaMemsetAsync (static split-K workspace counters)", e);
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_cleared[dev] = true;
  }
  return g_noalloc_address[dev];
}

}  // namespace
}  // namespace fp8q

extern "C" fp8q_status fp8q_linear_fwd_splitk_noalloc(const uint8_t* qa, const float* sa,
                                                      int64_t ldsa, const uint8_t* qw,
                                                      const float* sw, int64_t M, int64_t N,
                                                      int64_t K, uint16_t* y, int64_t ldy,
                                                      void* stream) {
  if (!qa || !sa || !qw || !sw || !y) return FP8Q_ERR_NULL;
  if (M <= 0 || M > 128 || N <= 0 || K <= 0 || N % 128 || K % 128 || ldsa < M || ldy < N)
    return FP8Q_ERR_SHAPE;
  if (!aligned16(qa) || !aligned16(sa) || !aligned16(qw) || !aligned16(sw) || !aligned16(y) ||
      ldsa % 4 || ldy % 8)
    return FP8Q_ERR_ALIGN;
  const int64_t counters = 4 * (N / kSplitBN);
  const int64_t partials = N * (K / kSkBK) * M * 4;
  if (counters > kNoAllocCounterBytes || partials > kNoAllocBytes - kNoAllocCounterBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "fp8q_linear_fwd_splitk_noalloc: M=%lld N=%lld K=%lld needs %lld bytes of "
             "partials; the static workspace holds %lld",
             static_cast<long long>(M), static_cast<long long>(N), static_cast<long long>(K),
             static_cast<long long>(partials),
             static_cast<long long>(kNoAllocBytes - kNoAllocCounterBytes));
    set_last_error_text(msg);
    return FP8Q_ERR_SHAPE;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(noalloc_workspace(st));
  if (!ws) return FP8Q_ERR_CUDA;
  // B = W [N][K]; block scale of (n, slice r) = sw[(n/128)*(K/128) + r]
  return launch_skinny_gemm_splitk_into(qa, qw, M, N, K, sa, ldsa, sw, K / 128, 1, y, ldy,
                                        reinterpret_cast<unsigned*>(ws),
                                        reinterpret_cast<float*>(ws + kNoAllocCounterBytes), st);
}
