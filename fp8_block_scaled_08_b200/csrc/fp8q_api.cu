// libfp8q: library-wide entry points (status strings, version, the device error
// word, the failure-path probe) and the host helpers the kernels' launchers share
// (device query, TMA descriptor encoding through the driver entry point).
#include <cudaTypedefs.h>
#include <stdio.h>
#include <mutex>

#include "fp8q_device.cuh"
#include "fp8q_host.h"

namespace fp8q {

// Set by kernels when a bounded wait gives up (bit kErrTimeout).
__device__ unsigned g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int checked = 0;
  int sm_count = 0;  // 0 if the device is not sm_100
  unsigned* err = nullptr;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

DeviceInfo* current_info() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceInfo* d = &g_dev[dev];
  if (d->checked) return d;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!d->checked) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    d->sm_count = (major == 10 && minor == 0) ? sms : 0;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess) d->err = static_cast<unsigned*>(p);
    cudaGetLastError();
    d->checked = 1;
  }
  return d;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

// One CTA waits on an mbarrier that nothing completes, with the GEMM's bounded wait.
__global__ void debug_wait_kernel(unsigned* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const WaitCtl ctl{&abort_flag, err, limit_ns};
  mbar_wait_warp(&bar, 0, ctl);  // phase 0 never completes: gives up after limit_ns
  __syncthreads();
}

}  // namespace

namespace {
thread_local char g_last_error[256] = "";
}

void set_last_error(const char* where, cudaError_t e) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorString(e),
           cudaGetErrorName(e));
}

void set_last_error_text(const char* text) { snprintf(g_last_error, sizeof(g_last_error), "%s", text); }

unsigned* device_error_word() {
  DeviceInfo* d = current_info();
  return d ? d->err : nullptr;
}

int sm100_sm_count() {
  DeviceInfo* d = current_info();
  return d ? d->sm_count : 0;
}

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                    uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                    uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) {
    set_last_error("cuTensorMapEncodeTiled entry point", cudaErrorNotSupported);
    return false;
  }
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed: CUresult %d",
             static_cast<int>(r));
    return false;
  }
  return true;
}

bool encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                    const uint64_t (&dims)[3], const uint64_t (&strides_bytes)[2],
                    const uint32_t (&box)[3], CUtensorMapSwizzle swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) {
    set_last_error("cuTensorMapEncodeTiled entry point", cudaErrorNotSupported);
    return false;
  }
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {strides_bytes[0], strides_bytes[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, dtype, 3, const_cast<void*>(base), d, st, bx, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (3D) failed: CUresult %d",
             static_cast<int>(r));
    return false;
  }
  return true;
}

}  // namespace fp8q

using namespace fp8q;

extern "C" const char* fp8q_status_string(fp8q_status status) {
  switch (status) {
    case FP8Q_OK: return "FP8Q_OK";
    case FP8Q_ERR_NULL: return "FP8Q_ERR_NULL: a required pointer is NULL";
    case FP8Q_ERR_SHAPE: return "FP8Q_ERR_SHAPE: size or leading dimension not allowed";
    case FP8Q_ERR_ALIGN: return "FP8Q_ERR_ALIGN: pointer or row stride not 16-byte aligned";
    case FP8Q_ERR_CUDA: return "FP8Q_ERR_CUDA: CUDA launch or runtime error";
    case FP8Q_ERR_TIMEOUT: return "FP8Q_ERR_TIMEOUT: a kernel gave up a bounded wait";
    case FP8Q_ERR_UNSUPPORTED: return "FP8Q_ERR_UNSUPPORTED: needs an sm_100 device";
    default: return "FP8Q_ERR_UNKNOWN";
  }
}

extern "C" int fp8q_version(void) { return 10000; }

extern "C" const char* fp8q_last_error_message(void) { return g_last_error; }

extern "C" fp8q_status fp8q_device_error(void* stream, int clear) {
  unsigned* w = device_error_word();
  if (!w) return FP8Q_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FP8Q_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return FP8Q_ERR_CUDA;
  if (clear && v) {
    const unsigned zero = 0;
    if (cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return FP8Q_ERR_CUDA;
  }
  return (v & kErrTimeout) ? FP8Q_ERR_TIMEOUT : FP8Q_OK;
}

extern "C" fp8q_status fp8q_last_device_error(void* stream) {
  return fp8q_device_error(stream, 0);
}

extern "C" fp8q_status fp8q_debug_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns <= 0 || limit_ns > 10000000000ll) return FP8Q_ERR_SHAPE;
  if (!sm100_sm_count()) return FP8Q_ERR_UNSUPPORTED;
  unsigned* w = device_error_word();
  if (!w) return FP8Q_ERR_CUDA;
  debug_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(w, static_cast<uint64_t>(limit_ns));
  return launch_status();
}
