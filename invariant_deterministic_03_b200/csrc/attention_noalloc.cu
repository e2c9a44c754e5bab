// attention_noalloc.cu -- decode attention for callers that cannot allocate
// device memory.
//
// bi_attn_decode needs a caller-owned workspace for the per-split partial
// results. Some callers cannot provide one: a host application that hands all
// device memory to its own pool at start-up and forbids any later cudaMalloc,
// or a latency-critical loop where cudaMalloc's implicit device-wide
// synchronisation is not acceptable. bi_attn_decode_noalloc serves them with
// a fixed scratch array that lives in this file as a static __device__
// variable: it is part of the library's device image, so every GPU that loads
// libbi holds it (BI_ATTN_NOALLOC_SCRATCH_BYTES) until the process exits, and
// nothing is allocated per call.
//
// The array's name means nothing to host code (there it is a host-side
// stand-in, not a device address), so the device address is looked up with
// cudaGetSymbolAddress, with the device current, once per device and CUDA
// context, and cached; the cache is keyed by the current context, so a
// context that was destroyed and re-created (cudaDeviceReset, a released
// primary context) gets a fresh lookup instead of a stale address. The
// lookup happens on the first call in each context, which should therefore
// come before any stream capture.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "host.h"

namespace bi {
namespace noalloc {

static __device__ __align__(256) uint8_t g_attn_scratch[BI_ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
static std::mutex g_mu;
static CUcontext g_ctx[kMaxDev];        // context the cached address belongs to
static void* g_scratch_ptr[kMaxDev];
static PFN_cuCtxGetCurrent_v4000 g_get_ctx = nullptr;

// Device address of the scratch array in the current device's current
// context (looked up once per device and context, with that device current).
static bi_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "attn_decode_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDev) return fail(BI_ERR_UNSUPPORTED, "attn_decode_noalloc: device id %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_get_ctx) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
      return fail(BI_ERR_UNSUPPORTED, "attn_decode_noalloc: cuCtxGetCurrent unavailable");
    g_get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  }
  CUcontext ctx = nullptr;
  if (g_get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  if (!ctx || !g_scratch_ptr[dev] || g_ctx[dev] != ctx) {
    // the lookup also makes the device's primary context current when no
    // context is yet (the runtime initialises it on first use)
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "attn_decode_noalloc: cudaGetSymbolAddress");
    if (g_get_ctx(&ctx) != CUDA_SUCCESS || !ctx)
      return fail(BI_ERR_CUDA, "attn_decode_noalloc: no current CUDA context");
    g_scratch_ptr[dev] = p;
    g_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return BI_OK;
}

}  // namespace noalloc
}  // namespace bi

using namespace bi;

extern "C" bi_status bi_attn_decode_noalloc(const void* q, int64_t ldq, const void* k_cache,
                                            const void* v_cache, const int32_t* block_table,
                                            const int32_t* seq_lens, int32_t B,
                                            const bi_attn_shape* shape, void* out, int64_t ldo,
                                            void* stream) {
  if (B < 0) return fail(BI_ERR_INVALID_ARG, "attn_decode_noalloc: negative B");
  size_t need = 0;
  bi_status st = bi_attn_workspace_size(shape, B, &need);
  if (st != BI_OK) return st;
  if (need > (size_t)BI_ATTN_NOALLOC_SCRATCH_BYTES)
    return fail(BI_ERR_WORKSPACE,
                "attn_decode_noalloc: %d sequences x %d q heads x ceil(max_kv_len/%d) splits need "
                "%zu scratch bytes, above the fixed maximum of %zu",
                B, shape->num_q_heads, BI_ATTN_SPLIT, need, (size_t)BI_ATTN_NOALLOC_SCRATCH_BYTES);
  if (B == 0) return BI_OK;
  void* scratch = nullptr;
  if ((st = noalloc::scratch_address(&scratch)) != BI_OK) return st;
  // No part of the scratch has to start at zero: the merge pass reads only
  // partials that the split pass of the same call has written.
  return bi_attn_decode(q, ldq, k_cache, v_cache, block_table, seq_lens, B, shape, out, ldo,
                        scratch, (size_t)BI_ATTN_NOALLOC_SCRATCH_BYTES, stream);
}
