// Host-side helpers shared by the libfp8q translation units: argument checks,
// device queries, TMA descriptor encoding and the device error word.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fp8q.h"

namespace fp8q {

// Address of the device error word on the current device (set up once per device).
unsigned* device_error_word();

// Streaming multiprocessor count of the current device; 0 if it is not sm_100.
int sm100_sm_count();

// 2D tiled tensor map (no multicast, no interleave). `inner`/`outer` are the tensor's
// extents in elements, `row_bytes` the byte stride between rows. Returns false if
// the driver entry point is missing or the encoding is rejected.
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                    uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                    uint32_t box_outer, CUtensorMapSwizzle swizzle);

// 3D tiled tensor map with explicit byte strides for dimensions 1 and 2 (dimension 0
// is contiguous); the strides need not increase with the dimension.
bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                    const uint64_t (&dims)[3], const uint64_t (&strides_bytes)[2],
                    const uint32_t (&box)[3], CUtensorMapSwizzle swizzle);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Remembers the text of a failure for fp8q_last_error_message (thread-local).
void set_last_error(const char* where, cudaError_t e);
void set_last_error_text(const char* text);

inline fp8q_status launch_status(const char* where = "launch") {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return FP8Q_OK;
  set_last_error(where, e);
  return FP8Q_ERR_CUDA;
}

// Bounded waits inside the kernels give up after this long (nanoseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Token batches up to this many rows take the skinny-M GEMM (forward and DGrad).
constexpr int64_t kSkinnyMaxM = 256;

// out [Mg][Ng] = A [Mg][Kg] x B [Ng][Kg]^T with per-row A scales sa[r*ldsa + i] and
// per-128x128-block B scales sb[(j/128)*sb_sj + r*sb_sr], for Mg <= kSkinnyMaxM.
// Same arithmetic, in the same order, as the large-tile kernel.
fp8q_status launch_skinny_gemm(const uint8_t* A, const uint8_t* B, int64_t Mg, int64_t Ng,
                               int64_t Kg, const float* sa, int64_t ldsa, const float* sb,
                               int64_t sb_sj, int64_t sb_sr, uint16_t* y, int64_t ldy,
                               cudaStream_t stream);

}  // namespace fp8q
