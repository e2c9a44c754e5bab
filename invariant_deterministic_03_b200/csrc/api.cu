// api.cu -- library-wide host plumbing: thread-local error text, the device
// status word, device checks and TMA descriptor encoding.
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "host.h"

namespace bi {

// One status word per device (a __device__ variable exists once per device
// context). Kernels OR error bits into it; bi_device_status reads it.
__device__ int32_t g_status_word;

static thread_local char t_err[512] = "";

bi_status fail(bi_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
  return st;
}

bi_status cuda_fail(cudaError_t e, const char* where) {
  cudaGetLastError();  // clear a non-sticky error so the caller's next CUDA call is not blamed
  return fail(BI_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

namespace {
constexpr int kMaxDev = 64;
std::mutex g_mu;
int g_sm100[kMaxDev];        // 0 unknown, 1 yes, -1 no
int32_t* g_status_ptr[kMaxDev];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
}  // namespace

bi_status require_sm100() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDev) return fail(BI_ERR_UNSUPPORTED, "device id %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sm100[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    g_sm100[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (g_sm100[dev] < 0) return fail(BI_ERR_UNSUPPORTED, "device %d is not sm_100 (B200)", dev);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    g_status_ptr[dev] = static_cast<int32_t*>(p);
  }
  return BI_OK;
}

int32_t* status_word() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < kMaxDev) ? g_status_ptr[dev] : nullptr;
}

bi_status encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, void* base,
                      const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                      CUtensorMapSwizzle swizzle) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return fail(BI_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled unavailable");
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(map, dtype, rank, base, reinterpret_cast<const cuuint64_t*>(dims),
                        reinterpret_cast<const cuuint64_t*>(strides_bytes),
                        reinterpret_cast<const cuuint32_t*>(box), elem_strides,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BI_ERR_ALIGN, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return BI_OK;
}

// Self-check of the wait bound: thread 0 waits on an mbarrier that nothing
// ever arrives on, through the same bounded wait every kernel uses, with a
// short limit; it gives up, records BI_DEV_WAIT_TIMEOUT and raises the CTA's
// abort flag, which releases the other threads' waits on the same barrier.
__global__ void wait_bound_check_kernel(long long limit, int32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* ab = &abort_flag;
  if (threadIdx.x == 0) {
    mbar_wait(&bar, 0, status, ab, limit);
  } else {
    mbar_wait(&bar, 0, status, ab, 2 * limit + 1000000);
  }
}

}  // namespace bi

extern "C" bi_status bi_check_wait_bound(int64_t limit_cycles, void* stream) {
  if (limit_cycles < 1000 || limit_cycles > bi::kWaitLimitCycles)
    return bi::fail(BI_ERR_INVALID_ARG, "check_wait_bound: limit %lld outside [1000, 2^32] cycles",
                    (long long)limit_cycles);
  bi_status st = bi::require_sm100();
  if (st != BI_OK) return st;
  bi::wait_bound_check_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles,
                                                                              bi::status_word());
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return bi::cuda_fail(e, "check_wait_bound launch");
  return BI_OK;
}

extern "C" const char* bi_last_error(void) { return bi::t_err; }

extern "C" bi_status bi_device_status(int32_t* status, int32_t clear, void* stream) {
  if (!status) return bi::fail(BI_ERR_INVALID_ARG, "bi_device_status: status is null");
  bi_status st = bi::require_sm100();
  if (st != BI_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return bi::cuda_fail(e, "bi_device_status: stream sync");
  int32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, bi::g_status_word, sizeof(v));
  if (e != cudaSuccess) return bi::cuda_fail(e, "bi_device_status: read");
  if (clear) {
    int32_t z = 0;
    e = cudaMemcpyToSymbol(bi::g_status_word, &z, sizeof(z));
    if (e != cudaSuccess) return bi::cuda_fail(e, "bi_device_status: clear");
  }
  *status = v;
  if (v) return bi::fail(BI_ERR_DEVICE_CHECK, "device status word 0x%x", v);
  return BI_OK;
}
