// pointwise.cu -- the element-wise steps of the decoder and the KV-cache write.
//
// "Defeating Nondeterminism in LLM Inference", section "How do we make
// kernels batch-invariant?": pointwise operations are batch-invariant as long
// as every element goes through the same code (the page's counter-example is
// a CPU kernel that vectorises part of an array and not the rest). Each kernel
// here has one code path per element: no vector/scalar tail split depends on
// the batch, and every element's arithmetic is written out with explicit
// rounding intrinsics.
//
// The cache write follows section "Batch-invariant attention": the KV cache
// and page table are updated before attention runs, so attention always reads
// keys from one layout.
#include "common.cuh"
#include "host.h"

namespace bi {
namespace pw {

// ---- KV append: one warp per (token, kv head). Each (page, kv head) block
// of 16 keys x 128 d is stored in the tensor core's canonical no-swizzle
// K-major order, so attention copies it into shared memory as one piece:
//   keys:   element (slot o, d) at (o/8)*1024 + (d/8)*64 + (o%8)*8 + d%8
//   values: element (d, slot o) at (d/8)*128 + (o/8)*64 + (d%8)*8 + o%8
// (element offsets inside the block; 8 x 8 core matrices of 128 bytes).
// The copy moves 16-bit elements as bits, so it serves bf16 and fp16 caches.
__global__ void kv_append_kernel(const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
                                 int64_t ld_new, const int32_t* __restrict__ slots, int64_t n_tok,
                                 int Hkv, int num_pages, uint16_t* __restrict__ kc,
                                 uint16_t* __restrict__ vc, int32_t* status) {
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= n_tok * Hkv) return;
  const int64_t t = wid / Hkv;
  const int g = (int)(wid % Hkv);
  const int32_t slot = slots[t];
  if (slot < 0) return;  // padding token
  if (slot >= num_pages * BI_PAGE_SIZE) {
    if (lane == 0) set_status(status, BI_DEV_BAD_SLOT);
    return;
  }
  const int page = slot / BI_PAGE_SIZE, o = slot % BI_PAGE_SIZE;
  const uint16_t* ksrc = k_new + t * ld_new + (int64_t)g * BI_HEAD_DIM;
  const uint16_t* vsrc = v_new + t * ld_new + (int64_t)g * BI_HEAD_DIM;
  const size_t blk = ((size_t)page * Hkv + g) * (BI_PAGE_SIZE * BI_HEAD_DIM);
  const int d0 = lane * 4;  // this lane's 4 consecutive d values (one core-matrix row half)
  const uint2 kv = reinterpret_cast<const uint2*>(ksrc)[lane];
  *reinterpret_cast<uint2*>(kc + blk + (o >> 3) * 1024 + (d0 >> 3) * 64 + (o & 7) * 8 + (d0 & 7)) = kv;
  uint16_t* vdst = vc + blk + (o >> 3) * 64 + (o & 7);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int d = d0 + i;
    vdst[(d >> 3) * 128 + (d & 7) * 8] = vsrc[d];
  }
}

// ---- embedding gather into the fp32 residual stream (16-bit table, exact)
template <typename ET>
__global__ void embed_kernel(const int32_t* __restrict__ tokens, const ET* __restrict__ table,
                             int64_t vocab, int D, float* __restrict__ out, int32_t* status) {
  const int64_t t = blockIdx.x;
  const int32_t id = tokens[t];
  const bool ok = id >= 0 && id < vocab;
  if (!ok && threadIdx.x == 0) set_status(status, BI_DEV_BAD_TOKEN);
  for (int c = threadIdx.x; c < D / 8; c += blockDim.x) {
    float v[8];
    if (ok) {
      const uint4 u = reinterpret_cast<const uint4*>(table + (size_t)id * D)[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = E16<ET>::lo(w[i]);
        v[2 * i + 1] = E16<ET>::hi(w[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.0f;
    }
    float4* o = reinterpret_cast<float4*>(out + t * (size_t)D + c * 8);
    o[0] = make_float4(v[0], v[1], v[2], v[3]);
    o[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// ---- RoPE table: cos/sin of pos * theta^(-2i/128) in fp64, stored as fp32
__global__ void rope_table_kernel(float* __restrict__ cs, int max_pos, double theta) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)max_pos * 64) return;
  const int pos = (int)(idx / 64), i = (int)(idx % 64);
  const double inv_freq = pow(theta, -2.0 * (double)i / (double)BI_HEAD_DIM);
  const double a = (double)pos * inv_freq;
  cs[idx * 2] = (float)cos(a);
  cs[idx * 2 + 1] = (float)sin(a);
}

// ---- RoPE in place: one thread per (token, head, pair i < 64)
// grid (token, head-pair block): each thread rotates 8 consecutive pairs
// (i, i + 64), i = i0 .. i0+7, of one head with 16-byte accesses (rows
// 16-byte aligned), or one pair (VEC == 1)
template <int VEC, typename ET>
__global__ void rope_kernel(ET* __restrict__ x, int64_t ldx, int n_heads,
                            const int32_t* __restrict__ pos, const float* __restrict__ cs,
                            int max_pos, int32_t* status) {
  constexpr int PER_HEAD = 64 / VEC;
  const int64_t t = blockIdx.x;
  const int k = blockIdx.y * blockDim.x + threadIdx.x;
  if (k >= n_heads * PER_HEAD) return;
  const int h = k / PER_HEAD, i0 = (k % PER_HEAD) * VEC;
  const int p = pos[t];
  if (p < 0 || p >= max_pos) {
    if (k == 0) set_status(status, BI_DEV_BAD_TOKEN);
    return;
  }
  ET* row = x + t * ldx + (int64_t)h * BI_HEAD_DIM;
  const float* csp = cs + ((size_t)p * 64 + i0) * 2;
  float a[VEC], b[VEC], c[VEC], sn[VEC];
  if constexpr (VEC == 8) {
    const uint4 av = *reinterpret_cast<const uint4*>(row + i0), bv = *reinterpret_cast<const uint4*>(row + i0 + 64);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      a[j] = E16<ET>::to_f32(reinterpret_cast<const ET*>(&av)[j]);
      b[j] = E16<ET>::to_f32(reinterpret_cast<const ET*>(&bv)[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 q = reinterpret_cast<const float4*>(csp)[j];
      c[2 * j] = q.x;
      sn[2 * j] = q.y;
      c[2 * j + 1] = q.z;
      sn[2 * j + 1] = q.w;
    }
  } else {
    a[0] = E16<ET>::to_f32(row[i0]);
    b[0] = E16<ET>::to_f32(row[i0 + 64]);
    c[0] = csp[0];
    sn[0] = csp[1];
  }
  float ra[VEC], rb[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) {
    rope_rotate(a[j], b[j], c[j], sn[j], ra[j], rb[j]);
  }
  if constexpr (VEC == 8) {
    using E = E16<ET>;
    *reinterpret_cast<uint4*>(row + i0) = make_uint4(E::pack2(ra[0], ra[1]), E::pack2(ra[2], ra[3]),
                                                     E::pack2(ra[4], ra[5]), E::pack2(ra[6], ra[7]));
    *reinterpret_cast<uint4*>(row + i0 + 64) = make_uint4(E::pack2(rb[0], rb[1]), E::pack2(rb[2], rb[3]),
                                                          E::pack2(rb[4], rb[5]), E::pack2(rb[6], rb[7]));
  } else {
    row[i0] = E16<ET>::from_f32(ra[0]);
    row[i0 + 64] = E16<ET>::from_f32(rb[0]);
  }
}

// ---- SwiGLU: out = bf16(silu(g) * u), silu(g) = g / (1 + exp(-g))
// grid (token, feature block); VEC features per thread: 8 with 16-byte
// vector access (F % 8 == 0, aligned rows), else 1
template <int VEC>
__global__ void swiglu_kernel(const bf16* __restrict__ gu, int64_t F, bf16* __restrict__ out) {
  const int64_t t = blockIdx.x;
  const int64_t f = ((int64_t)blockIdx.y * blockDim.x + threadIdx.x) * VEC;
  if (f >= F) return;
  const bf16* g = gu + t * 2 * F + f;
  const bf16* u = g + F;
  bf16* o = out + t * F + f;
  if constexpr (VEC == 8) {
    const uint4 gv = *reinterpret_cast<const uint4*>(g), uv = *reinterpret_cast<const uint4*>(u);
    const bf16* ge = reinterpret_cast<const bf16*>(&gv);
    const bf16* ue = reinterpret_cast<const bf16*>(&uv);
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = swiglu_f32(__bfloat162float(ge[k]), __bfloat162float(ue[k]));
    *reinterpret_cast<uint4*>(o) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                              pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  } else {
    o[0] = __float2bfloat16_rn(swiglu_f32(__bfloat162float(g[0]), __bfloat162float(u[0])));
  }
}

// ---- residual add into the fp32 stream
__global__ void residual_kernel(float* __restrict__ x, const bf16* __restrict__ d, int64_t n) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n) return;
  x[idx] = __fadd_rn(x[idx], __bfloat162float(d[idx]));
}

// ---- argmax per row, lowest index on ties; NaN counts as the largest value
__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
  const bool na = a != a, nb = b != b;
  if (na || nb) return na && (!nb || ia < ib);
  if (a != b) return a > b;
  return ia < ib;
}

__global__ void argmax_kernel(const float* __restrict__ logits, int64_t V, int64_t ld,
                              int32_t* __restrict__ idx_out) {
  __shared__ float sv[32];
  __shared__ int si[32];
  const float* row = logits + (size_t)blockIdx.x * ld;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int64_t j = threadIdx.x; j < V; j += blockDim.x) {
    const float v = row[j];
    if (better(v, (int)j, bv, bi)) { bv = v; bi = (int)j; }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const float ov = __shfl_down_sync(0xffffffffu, bv, off);
    const int oi = __shfl_down_sync(0xffffffffu, bi, off);
    if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) { sv[w] = bv; si[w] = bi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k)
      if (better(sv[k], si[k], bv, bi)) { bv = sv[k]; bi = si[k]; }
    idx_out[blockIdx.x] = bi == 0x7fffffff ? 0 : bi;
  }
}

}  // namespace pw

bi_status launch_kv_append(const uint16_t* k, const uint16_t* v, int64_t ld_new, const int32_t* slots,
                           int64_t n_tok, uint16_t* kc, uint16_t* vc, int Hkv, int num_pages,
                           cudaStream_t s) {
  const int64_t warps = n_tok * Hkv;
  const int64_t blocks = (warps + 7) / 8;
  pw::kv_append_kernel<<<(unsigned)blocks, 256, 0, s>>>(k, v, ld_new, slots, n_tok, Hkv, num_pages,
                                                        kc, vc, status_word());
  BI_CHECK_LAUNCH("kv_append launch");
  return BI_OK;
}

template <typename ET>
bi_status launch_embed(const int32_t* tok, int64_t n_tok, const ET* table, int64_t vocab,
                       int64_t D, float* out, cudaStream_t s) {
  pw::embed_kernel<ET><<<(unsigned)n_tok, 128, 0, s>>>(tok, table, vocab, (int)D, out, status_word());
  BI_CHECK_LAUNCH("embed launch");
  return BI_OK;
}
template bi_status launch_embed<bf16>(const int32_t*, int64_t, const bf16*, int64_t, int64_t, float*, cudaStream_t);
template bi_status launch_embed<f16>(const int32_t*, int64_t, const f16*, int64_t, int64_t, float*, cudaStream_t);

template <typename ET>
bi_status launch_rope(ET* x, int64_t ldx, int n_heads, const int32_t* pos, int64_t n_tok,
                      const float* cs, int max_pos, cudaStream_t s) {
  if (n_tok == 0) return BI_OK;
  const bool vec = ldx % 8 == 0 && aligned16(x);
  const int64_t per_tok = (int64_t)n_heads * (vec ? 8 : 64);
  const dim3 grid((unsigned)n_tok, (unsigned)((per_tok + 255) / 256));
  if (n_tok > 0x7fffffff || grid.y > 65535) return fail(BI_ERR_SHAPE, "rope: size out of range");
  if (vec) pw::rope_kernel<8, ET><<<grid, 256, 0, s>>>(x, ldx, n_heads, pos, cs, max_pos, status_word());
  else pw::rope_kernel<1, ET><<<grid, 256, 0, s>>>(x, ldx, n_heads, pos, cs, max_pos, status_word());
  BI_CHECK_LAUNCH("rope launch");
  return BI_OK;
}
template bi_status launch_rope<bf16>(bf16*, int64_t, int, const int32_t*, int64_t, const float*, int, cudaStream_t);
template bi_status launch_rope<f16>(f16*, int64_t, int, const int32_t*, int64_t, const float*, int, cudaStream_t);

bi_status launch_swiglu(const bf16* gu, int64_t n_tok, int64_t F, bf16* out, cudaStream_t s) {
  const bool vec = F % 8 == 0 && aligned16(gu) && aligned16(out);
  const int64_t per_tok = vec ? F / 8 : F;
  const dim3 grid((unsigned)n_tok, (unsigned)((per_tok + 255) / 256));
  if (n_tok > 0x7fffffff || grid.y > 65535) return fail(BI_ERR_SHAPE, "swiglu: size out of range");
  if (vec) pw::swiglu_kernel<8><<<grid, 256, 0, s>>>(gu, F, out);
  else pw::swiglu_kernel<1><<<grid, 256, 0, s>>>(gu, F, out);
  BI_CHECK_LAUNCH("swiglu launch");
  return BI_OK;
}

bi_status launch_residual(float* x, const bf16* d, int64_t n, cudaStream_t s) {
  pw::residual_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(x, d, n);
  BI_CHECK_LAUNCH("residual launch");
  return BI_OK;
}

bi_status launch_argmax(const float* logits, int64_t rows, int64_t V, int64_t ld, int32_t* idx,
                        cudaStream_t s) {
  pw::argmax_kernel<<<(unsigned)rows, 256, 0, s>>>(logits, V, ld, idx);
  BI_CHECK_LAUNCH("argmax launch");
  return BI_OK;
}

}  // namespace bi

using namespace bi;

static bi_status check_kv(const bi_kv_layout* kv) {
  if (!kv) return fail(BI_ERR_INVALID_ARG, "kv layout is null");
  if (kv->head_dim != BI_HEAD_DIM || kv->page_size != BI_PAGE_SIZE)
    return fail(BI_ERR_SHAPE, "kv layout: head_dim must be 128 and page_size 16");
  if (kv->num_pages <= 0 || kv->num_kv_heads <= 0) return fail(BI_ERR_SHAPE, "kv layout: sizes must be positive");
  if ((int64_t)kv->num_pages * BI_PAGE_SIZE > 0x7fffffffll) return fail(BI_ERR_SHAPE, "kv layout: too many pages");
  return BI_OK;
}

extern "C" bi_status bi_kv_append(const void* k_new, const void* v_new, int64_t ld_new,
                                  const int32_t* slot_mapping, int64_t n_tok, void* k_cache,
                                  void* v_cache, const bi_kv_layout* kv, void* stream) {
  bi_status st = check_kv(kv);
  if (st != BI_OK) return st;
  if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache) return fail(BI_ERR_INVALID_ARG, "kv_append: null pointer");
  if (n_tok < 0) return fail(BI_ERR_INVALID_ARG, "kv_append: negative n_tok");
  if (ld_new < (int64_t)kv->num_kv_heads * BI_HEAD_DIM) return fail(BI_ERR_SHAPE, "kv_append: ld_new smaller than num_kv_heads*128");
  if (ld_new % 8 || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(BI_ERR_ALIGN, "kv_append: rows must be 16-byte aligned");
  if (n_tok == 0) return BI_OK;
  if ((st = require_sm100()) != BI_OK) return st;
  return launch_kv_append(static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new), ld_new,
                          slot_mapping, n_tok, static_cast<uint16_t*>(k_cache),
                          static_cast<uint16_t*>(v_cache), kv->num_kv_heads, kv->num_pages,
                          static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_embed(const int32_t* tokens, int64_t n_tok, const void* table,
                              int64_t vocab, int64_t D, float* out, void* stream) {
  if (!tokens || !table || !out) return fail(BI_ERR_INVALID_ARG, "embed: null pointer");
  if (n_tok < 0 || vocab <= 0 || D <= 0) return fail(BI_ERR_INVALID_ARG, "embed: bad sizes");
  if (D % 8 || !aligned16(table) || !aligned16(out)) return fail(BI_ERR_ALIGN, "embed: D % 8 and 16-byte alignment required");
  if (n_tok > 0x7fffffffll) return fail(BI_ERR_SHAPE, "embed: too many tokens");
  if (n_tok == 0) return BI_OK;
  bi_status st = require_sm100();
  if (st != BI_OK) return st;
  return launch_embed<bf16>(tokens, n_tok, static_cast<const bf16*>(table), vocab, D, out,
                      static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_rope_table(float* cos_sin, int32_t max_pos, double theta, void* stream) {
  if (!cos_sin || max_pos <= 0 || !(theta > 1.0)) return fail(BI_ERR_INVALID_ARG, "rope_table: bad arguments");
  bi_status st = require_sm100();
  if (st != BI_OK) return st;
  const int64_t n = (int64_t)max_pos * 64;
  pw::rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      cos_sin, max_pos, theta);
  BI_CHECK_LAUNCH("rope_table launch");
  return BI_OK;
}

extern "C" bi_status bi_rope(void* x, int64_t ldx, int32_t n_heads, const int32_t* positions,
                             int64_t n_tok, const float* cos_sin, int32_t max_pos, void* stream) {
  if (!x || !positions || !cos_sin) return fail(BI_ERR_INVALID_ARG, "rope: null pointer");
  if (n_tok < 0 || n_heads <= 0 || max_pos <= 0) return fail(BI_ERR_INVALID_ARG, "rope: bad sizes");
  if (ldx < (int64_t)n_heads * BI_HEAD_DIM) return fail(BI_ERR_SHAPE, "rope: ldx smaller than n_heads*128");
  if (n_tok == 0) return BI_OK;
  bi_status st = require_sm100();
  if (st != BI_OK) return st;
  return launch_rope<bf16>(static_cast<bf16*>(x), ldx, n_heads, positions, n_tok, cos_sin, max_pos,
                     static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_swiglu(const void* gu, int64_t n_tok, int64_t F, void* out, void* stream) {
  if (!gu || !out) return fail(BI_ERR_INVALID_ARG, "swiglu: null pointer");
  if (n_tok < 0 || F <= 0) return fail(BI_ERR_INVALID_ARG, "swiglu: bad sizes");
  if (n_tok == 0) return BI_OK;
  bi_status st = require_sm100();
  if (st != BI_OK) return st;
  return launch_swiglu(static_cast<const bf16*>(gu), n_tok, F, static_cast<bf16*>(out),
                       static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_residual_add(float* x, const void* d, int64_t n_tok, int64_t D,
                                     void* stream) {
  if (!x || !d) return fail(BI_ERR_INVALID_ARG, "residual_add: null pointer");
  if (n_tok < 0 || D <= 0) return fail(BI_ERR_INVALID_ARG, "residual_add: bad sizes");
  if (n_tok == 0) return BI_OK;
  bi_status st = require_sm100();
  if (st != BI_OK) return st;
  return launch_residual(x, static_cast<const bf16*>(d), n_tok * D,
                         static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_argmax(const float* logits, int64_t rows, int64_t V, int64_t ld,
                               int32_t* idx, void* stream) {
  if (!logits || !idx) return fail(BI_ERR_INVALID_ARG, "argmax: null pointer");
  if (rows < 0 || V <= 0 || ld < V) return fail(BI_ERR_INVALID_ARG, "argmax: bad sizes");
  if (V > 0x7fffffffll || rows > 0x7fffffffll) return fail(BI_ERR_SHAPE, "argmax: too large");
  if (rows == 0) return BI_OK;
  bi_status st = require_sm100();
  if (st != BI_OK) return st;
  return launch_argmax(logits, rows, V, ld, idx, static_cast<cudaStream_t>(stream));
}
