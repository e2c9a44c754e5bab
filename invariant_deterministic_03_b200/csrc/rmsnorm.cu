// rmsnorm.cu -- batch-invariant RMSNorm, one CTA per row.
//
// "Defeating Nondeterminism in LLM Inference", section "Batch-invariant
// RMSNorm": assign each batch element (row) to one core so that no row's
// reduction is ever split; the reduction strategy may depend on the reduced
// length D, never on the number of rows. Small batches simply leave SMs idle.
//
// Fixed order of the sum of squares of row i (depends on D only):
//   1. thread t adds x^2 of its chunks c = t, t + T, t + 2T, ... (8 elements
//      each, left to right) with fmaf, T = threads per CTA (a function of D);
//   2. warp shuffle-down tree, offsets 16, 8, 4, 2, 1 (lane 0 ends with the
//      warp sum);
//   3. thread 0 adds the warp sums in warp order and forms
//      r = 1 / sqrtf(ss / D + eps);
//   4. every element: y = bf16((x * r) * gamma), round to nearest even.
#include "common.cuh"
#include "host.h"

namespace bi {

template <typename Tin>
struct Row8;  // 8 consecutive input elements as fp32

template <>
struct Row8<bf16> {
  static __device__ __forceinline__ void load(const bf16* p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
};

template <>
struct Row8<f16> {
  static __device__ __forceinline__ void load(const f16* p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = E16<f16>::lo(w[i]);
      v[2 * i + 1] = E16<f16>::hi(w[i]);
    }
  }
};

template <>
struct Row8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
    float4 a = *reinterpret_cast<const float4*>(p);
    float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

// CPT = chunks per thread (compile-time so the row stays in registers).
// SPLIT: write the fp32 result as a bf16 pair (y = bf16(v), y_lo = bf16(v - y))
// for the fp32-activation path; otherwise y = r16(v), r16 the rounding to
// the 16-bit output type ET (bf16, or fp16 for the FP16 variant; gamma has
// the same type). R_ONLY: write only the row's scale r to r_out[row] (the
// same reduction, for a GEMM that applies the norm to its A operand).
template <typename Tin, int CPT, bool SPLIT, typename ET, bool R_ONLY = false>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const Tin* __restrict__ x,
                                                      const ET* __restrict__ gamma,
                                                      ET* __restrict__ y, ET* __restrict__ y_lo,
                                                      int D, float eps, float* __restrict__ r_out = nullptr) {
  __shared__ float warp_sum[32];
  __shared__ float row_scale;
  const int T = blockDim.x;
  const int t = threadIdx.x;
  const int nchunks = D >> 3;
  const size_t row = blockIdx.x;
  const Tin* xr = x + row * (size_t)D;
  ET* yr = y + row * (size_t)D;

  float v[CPT][8];
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    int c = t + i * T;
    if (c < nchunks) {
      Row8<Tin>::load(xr + c * 8, v[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(v[i][e], v[i][e], ss);
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ss += __shfl_down_sync(0xffffffffu, ss, off);
  const int warp = t >> 5, lane = t & 31;
  if (lane == 0) warp_sum[warp] = ss;
  __syncthreads();
  if (t == 0) {
    float total = 0.0f;
    const int nw = T >> 5;
    for (int w = 0; w < nw; ++w) total = total + warp_sum[w];
    row_scale = 1.0f / sqrtf(total / (float)D + eps);
    if (R_ONLY) r_out[row] = row_scale;
  }
  if (R_ONLY) return;
  __syncthreads();
  const float r = row_scale;
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    int c = t + i * T;
    if (c < nchunks) {
      float g[8];
      Row8<ET>::load(gamma + c * 8, g);
      uint4 o, olo;
      uint32_t* op = reinterpret_cast<uint32_t*>(&o);
      uint32_t* olp = reinterpret_cast<uint32_t*>(&olo);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = __fmul_rn(__fmul_rn(v[i][2 * e], r), g[2 * e]);
        const float b = __fmul_rn(__fmul_rn(v[i][2 * e + 1], r), g[2 * e + 1]);
        op[e] = E16<ET>::pack2(a, b);
        if (SPLIT) {
          const __nv_bfloat162 hb = *reinterpret_cast<const __nv_bfloat162*>(&op[e]);
          const float2 hf = __bfloat1622float2(hb);
          olp[e] = pack_bf16x2(__fsub_rn(a, hf.x), __fsub_rn(b, hf.y));
        }
      }
      *reinterpret_cast<uint4*>(yr + c * 8) = o;
      if (SPLIT) *reinterpret_cast<uint4*>(y_lo + row * (size_t)D + c * 8) = olo;
    }
  }
}

// Threads per CTA and chunks per thread as a function of D alone.
static void rms_geometry(int64_t D, int* threads, int* cpt) {
  int64_t nchunks = D / 8;
  int64_t T = ((nchunks + 31) / 32) * 32;
  if (T > 256) T = 256;
  int64_t c = (nchunks + T - 1) / T;
  int p = 1;
  while (p < c) p <<= 1;
  *threads = (int)T;
  *cpt = p;
}

template <typename Tin, bool SPLIT = false, typename ET = bf16>
static bi_status launch_rms(const Tin* x, const ET* g, ET* y, int64_t M, int64_t D, float eps,
                            cudaStream_t s, ET* y_lo = nullptr) {
  int T, cpt;
  rms_geometry(D, &T, &cpt);
  dim3 grid((unsigned)M), block(T);
  switch (cpt) {
    case 1: rmsnorm_kernel<Tin, 1, SPLIT, ET><<<grid, block, 0, s>>>(x, g, y, y_lo, (int)D, eps); break;
    case 2: rmsnorm_kernel<Tin, 2, SPLIT, ET><<<grid, block, 0, s>>>(x, g, y, y_lo, (int)D, eps); break;
    case 4: rmsnorm_kernel<Tin, 4, SPLIT, ET><<<grid, block, 0, s>>>(x, g, y, y_lo, (int)D, eps); break;
    case 8: rmsnorm_kernel<Tin, 8, SPLIT, ET><<<grid, block, 0, s>>>(x, g, y, y_lo, (int)D, eps); break;
    case 16: rmsnorm_kernel<Tin, 16, SPLIT, ET><<<grid, block, 0, s>>>(x, g, y, y_lo, (int)D, eps); break;
    default: return fail(BI_ERR_SHAPE, "rmsnorm: D=%lld unsupported", (long long)D);
  }
  BI_CHECK_LAUNCH("rmsnorm launch");
  return BI_OK;
}

static bi_status check_rms(const void* x, const void* gamma, const void* y, int64_t M, int64_t D,
                           float eps) {
  if (!x || !gamma || !y) return fail(BI_ERR_INVALID_ARG, "rmsnorm: null pointer");
  if (M < 0 || D <= 0) return fail(BI_ERR_INVALID_ARG, "rmsnorm: bad sizes M=%lld D=%lld", (long long)M, (long long)D);
  if (D % 8 != 0 || D > 32768) return fail(BI_ERR_SHAPE, "rmsnorm: D=%lld must be a multiple of 8 and <= 32768", (long long)D);
  if (M > 0x7fffffffll) return fail(BI_ERR_SHAPE, "rmsnorm: M=%lld too large", (long long)M);
  if (!(eps >= 0.0f)) return fail(BI_ERR_INVALID_ARG, "rmsnorm: eps must be >= 0");
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(y)) return fail(BI_ERR_ALIGN, "rmsnorm: pointers must be 16-byte aligned");
  return BI_OK;
}

// The row scales r_i = 1 / sqrt(sum_j x_ij^2 / D + eps) of fp32 rows, by the
// reduction bi_rmsnorm_f32in uses (same geometry, same order), into r[M].
bi_status rmsnorm_scales_f32(const float* x, int64_t M, int64_t D, float eps, float* r, cudaStream_t s) {
  if (!x || !r) return fail(BI_ERR_INVALID_ARG, "rmsnorm scales: null pointer");
  if (M < 0 || D <= 0 || D % 8 != 0 || D > 32768 || M > 0x7fffffffll)
    return fail(BI_ERR_SHAPE, "rmsnorm scales: bad sizes M=%lld D=%lld", (long long)M, (long long)D);
  if (!(eps >= 0.0f)) return fail(BI_ERR_INVALID_ARG, "rmsnorm scales: eps must be >= 0");
  if (!aligned16(x)) return fail(BI_ERR_ALIGN, "rmsnorm scales: x must be 16-byte aligned");
  if (M == 0) return BI_OK;
  int T, cpt;
  rms_geometry(D, &T, &cpt);
  dim3 grid((unsigned)M), block(T);
  switch (cpt) {
    case 1: rmsnorm_kernel<float, 1, false, bf16, true><<<grid, block, 0, s>>>(x, nullptr, nullptr, nullptr, (int)D, eps, r); break;
    case 2: rmsnorm_kernel<float, 2, false, bf16, true><<<grid, block, 0, s>>>(x, nullptr, nullptr, nullptr, (int)D, eps, r); break;
    case 4: rmsnorm_kernel<float, 4, false, bf16, true><<<grid, block, 0, s>>>(x, nullptr, nullptr, nullptr, (int)D, eps, r); break;
    case 8: rmsnorm_kernel<float, 8, false, bf16, true><<<grid, block, 0, s>>>(x, nullptr, nullptr, nullptr, (int)D, eps, r); break;
    case 16: rmsnorm_kernel<float, 16, false, bf16, true><<<grid, block, 0, s>>>(x, nullptr, nullptr, nullptr, (int)D, eps, r); break;
    default: return fail(BI_ERR_SHAPE, "rmsnorm scales: D=%lld unsupported", (long long)D);
  }
  BI_CHECK_LAUNCH("rmsnorm scales launch");
  return BI_OK;
}

// fp32 rows (the residual stream) to fp16 rows: the FP16 precision mode of
// the forward.
bi_status rmsnorm_f32in_f16(const float* x, const void* gamma, void* y, int64_t M, int64_t D, float eps,
                            cudaStream_t s) {
  bi_status st = check_rms(x, gamma, y, M, D, eps);
  if (st != BI_OK || M == 0) return st;
  if ((st = require_sm100()) != BI_OK) return st;
  return launch_rms<float, false, f16>(x, static_cast<const f16*>(gamma), static_cast<f16*>(y), M, D, eps, s);
}

}  // namespace bi

using namespace bi;

extern "C" bi_status bi_rmsnorm(const void* x, const void* gamma, void* y, int64_t M, int64_t D,
                                float eps, void* stream) {
  bi_status st = check_rms(x, gamma, y, M, D, eps);
  if (st != BI_OK || M == 0) return st;
  if ((st = require_sm100()) != BI_OK) return st;
  return launch_rms<bf16>(static_cast<const bf16*>(x), static_cast<const bf16*>(gamma),
                          static_cast<bf16*>(y), M, D, eps, static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_rmsnorm_f32in(const float* x, const void* gamma, void* y, int64_t M,
                                      int64_t D, float eps, void* stream) {
  bi_status st = check_rms(x, gamma, y, M, D, eps);
  if (st != BI_OK || M == 0) return st;
  if ((st = require_sm100()) != BI_OK) return st;
  return launch_rms<float>(x, static_cast<const bf16*>(gamma), static_cast<bf16*>(y), M, D, eps,
                           static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_rmsnorm_split(const float* x, const void* gamma, void* y_hi, void* y_lo,
                                      int64_t M, int64_t D, float eps, void* stream) {
  bi_status st = check_rms(x, gamma, y_hi, M, D, eps);
  if (st != BI_OK) return st;
  if (!y_lo || !aligned16(y_lo)) return fail(BI_ERR_ALIGN, "rmsnorm_split: y_lo null or misaligned");
  if (M == 0) return BI_OK;
  if ((st = require_sm100()) != BI_OK) return st;
  return launch_rms<float, true>(x, static_cast<const bf16*>(gamma), static_cast<bf16*>(y_hi), M, D,
                                 eps, static_cast<cudaStream_t>(stream), static_cast<bf16*>(y_lo));
}
