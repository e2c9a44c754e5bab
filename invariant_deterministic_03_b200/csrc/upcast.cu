// upcast.cu -- the fp32-activation ("upcast") variants of the decoder steps.
//
// The cross-vendor logit-mismatch paper (arXiv 2610.05458, abstract) traces
// logit differences to accumulation order and reports that upcasting to FP32
// reduces them (at about 3x the runtime), and that keeping only the MLP in
// BF16 keeps most of the gain (about 1.3x). These kernels give the decoder an
// fp32 activation path with the same batch-invariance rules as the bf16 one:
//
//  * an fp32 activation x that feeds a GEMM is carried as a bf16 pair
//    (hi = bf16(x), lo = bf16(x - hi)): hi + lo keeps ~16 significant bits,
//    and bi_gemm_x2 multiplies both terms by the same bf16 weight tile;
//  * RoPE, SwiGLU and the residual stream stay fp32;
//  * attention reads an fp32 KV cache; one warp per (query, q head, split)
//    computes scores and the weighted value sum in fp32 with a fixed order
//    (lane partial sums over d, then a shuffle-down tree, keys in order), and
//    the same fixed-size-split merge as the bf16 path.
#include "common.cuh"
#include "host.h"

namespace bi {
namespace up {

constexpr int HD = BI_HEAD_DIM;
constexpr int PAGE = BI_PAGE_SIZE;
constexpr int SPLIT = BI_ATTN_SPLIT;

__device__ __forceinline__ void split2(float y, bf16& hi, bf16& lo) {
  hi = __float2bfloat16_rn(y);
  lo = __float2bfloat16_rn(__fsub_rn(y, __bfloat162float(hi)));  // y - hi is exact in fp32
}

// ---- elementwise fp32 -> (hi, lo)
__global__ void split_kernel(const float* __restrict__ x, int64_t n, bf16* __restrict__ hi,
                             bf16* __restrict__ lo) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) split2(x[i], hi[i], lo[i]);
}

// ---- SwiGLU in fp32 on fp32 gate/up rows, output as a (hi, lo) pair
__global__ void swiglu_split_kernel(const float* __restrict__ gu, int64_t n_tok, int64_t F,
                                    bf16* __restrict__ hi, bf16* __restrict__ lo) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_tok * F) return;
  const int64_t t = idx / F, i = idx % F;
  const float g = gu[t * 2 * F + i];
  const float u = gu[t * 2 * F + F + i];
  const float silu = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
  split2(__fmul_rn(silu, u), hi[idx], lo[idx]);
}

// ---- RoPE in place on fp32 rows
__global__ void rope_f32_kernel(float* __restrict__ x, int64_t ldx, int n_heads,
                                const int32_t* __restrict__ pos, int64_t n_tok,
                                const float* __restrict__ cs, int max_pos, int32_t* status) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_tok * n_heads * 64) return;
  const int i = (int)(idx % 64);
  const int64_t th = idx / 64;
  const int h = (int)(th % n_heads);
  const int64_t t = th / n_heads;
  const int p = pos[t];
  float* row = x + t * ldx + (int64_t)h * HD;
  if (p < 0 || p >= max_pos) {
    if (i == 0) set_status(status, BI_DEV_BAD_TOKEN);
    return;
  }
  const float c = cs[((size_t)p * 64 + i) * 2], s = cs[((size_t)p * 64 + i) * 2 + 1];
  const float a = row[i], b = row[i + 64];
  row[i] = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
  row[i + 64] = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
}

// ---- fp32 KV cache append: both caches [num_pages][Hkv][16][128] fp32
__global__ void kv_append_f32_kernel(const float* __restrict__ k, const float* __restrict__ v,
                                     int64_t ld, const int32_t* __restrict__ slots, int64_t n_tok,
                                     int Hkv, int num_pages, float* __restrict__ kc,
                                     float* __restrict__ vc, int32_t* status) {
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= n_tok * Hkv) return;
  const int64_t t = wid / Hkv;
  const int g = (int)(wid % Hkv);
  const int32_t slot = slots[t];
  if (slot < 0) return;
  if (slot >= num_pages * PAGE) {
    if (lane == 0) set_status(status, BI_DEV_BAD_SLOT);
    return;
  }
  const size_t row = ((size_t)(slot / PAGE) * Hkv + g) * PAGE + slot % PAGE;
  reinterpret_cast<float4*>(kc + row * HD)[lane] = reinterpret_cast<const float4*>(k + t * ld + (size_t)g * HD)[lane];
  reinterpret_cast<float4*>(vc + row * HD)[lane] = reinterpret_cast<const float4*>(v + t * ld + (size_t)g * HD)[lane];
}

// ---- fp32 attention, split part. grid (n_split, n_tok, Hkv), G warps per CTA
// (warp w = q head g*G + w). Lane owns d = 4*lane .. 4*lane+3.
struct AttnParams {
  const float* q;
  int64_t ldq;
  const int32_t* cu_q;  // null: decode
  const float* kc;
  const float* vc;
  const int32_t* block_table;
  const int32_t* seq_lens;
  float* ws_o;
  float* ws_ml;
  int32_t B, Hq, Hkv, G, n_tok, num_pages, max_pages, max_kv_len, n_split_max;
  float scale_log2;
  int32_t* status;
};

__device__ __forceinline__ bool token_seq(const int32_t* cu_q, int B, int tok, int n_tok, int& b,
                                          int& nb, int& qidx) {
  if (!cu_q) {
    b = tok;
    nb = 1;
    qidx = 0;
    return true;
  }
  int lo = 0, hi = B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu_q[mid] <= tok) lo = mid; else hi = mid;
  }
  b = lo;
  nb = cu_q[b + 1] - cu_q[b];
  qidx = tok - cu_q[b];
  return cu_q[b] >= 0 && cu_q[b + 1] <= n_tok && qidx >= 0 && qidx < nb;
}

__global__ void attn_f32_split_kernel(const AttnParams p) {
  extern __shared__ float s_scores[];  // [G][SPLIT]
  const int s = blockIdx.x, tok = blockIdx.y, g = blockIdx.z;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, nb, qidx;
  if (!token_seq(p.cu_q, p.B, tok, p.n_tok, b, nb, qidx)) return;
  const int L = p.seq_lens[b];
  if (L < nb || L > p.max_kv_len) {
    if (threadIdx.x == 0 && s == 0 && g == 0) set_status(p.status, BI_DEV_BAD_SEQLEN);
    return;
  }
  const int pos = L - nb + qidx;
  const int k0 = s * SPLIT;
  if (k0 > pos) return;
  const int k1 = min((s + 1) * SPLIT, pos + 1);
  const int h = g * p.G + w;
  const float4 q4 = reinterpret_cast<const float4*>(p.q + (size_t)tok * p.ldq + (size_t)h * HD)[lane];
  float* sc = s_scores + w * SPLIT;
  float m = -INFINITY;
  for (int j = k0; j < k1; ++j) {
    const int pidx = j / PAGE;
    const int32_t pid = pidx < p.max_pages ? p.block_table[(size_t)b * p.max_pages + pidx] : -1;
    float dot = 0.0f;
    if (pid >= 0 && pid < p.num_pages) {
      const float4 k4 = reinterpret_cast<const float4*>(
          p.kc + (((size_t)pid * p.Hkv + g) * PAGE + j % PAGE) * HD)[lane];
      dot = __fmaf_rn(q4.x, k4.x, dot);
      dot = __fmaf_rn(q4.y, k4.y, dot);
      dot = __fmaf_rn(q4.z, k4.z, dot);
      dot = __fmaf_rn(q4.w, k4.w, dot);
    } else if (lane == 0) {
      set_status(p.status, BI_DEV_BAD_PAGE);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) dot = __fadd_rn(dot, __shfl_down_sync(0xffffffffu, dot, off));
    dot = __shfl_sync(0xffffffffu, dot, 0);  // lane 0's sum for every lane
    const float sv = __fmul_rn(dot, p.scale_log2);
    if (lane == 0) sc[j - k0] = sv;
    m = fmaxf(m, sv);
  }
  __syncwarp();
  float l = 0.0f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = k0; j < k1; ++j) {
    const float pj = exp2f(__fsub_rn(sc[j - k0], m));
    l = __fadd_rn(l, pj);
    const int pidx = j / PAGE;
    const int32_t pid = pidx < p.max_pages ? p.block_table[(size_t)b * p.max_pages + pidx] : -1;
    if (pid >= 0 && pid < p.num_pages) {
      const float4 v4 = reinterpret_cast<const float4*>(
          p.vc + (((size_t)pid * p.Hkv + g) * PAGE + j % PAGE) * HD)[lane];
      o.x = __fmaf_rn(pj, v4.x, o.x);
      o.y = __fmaf_rn(pj, v4.y, o.y);
      o.z = __fmaf_rn(pj, v4.z, o.z);
      o.w = __fmaf_rn(pj, v4.w, o.w);
    }
  }
  const size_t widx = ((size_t)tok * p.Hq + h) * p.n_split_max + s;
  reinterpret_cast<float4*>(p.ws_o + widx * HD)[lane] = o;
  if (lane == 0) *reinterpret_cast<float2*>(p.ws_ml + widx * 2) = make_float2(m, l);
}

// ---- merge in split order, fp32 output
__global__ void attn_f32_combine_kernel(const AttnParams p, float* __restrict__ out, int64_t ldo) {
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)p.n_tok * p.Hq) return;
  const int tok = (int)(wid / p.Hq), h = (int)(wid % p.Hq);
  float4* dst = reinterpret_cast<float4*>(out + (size_t)tok * ldo + (size_t)h * HD) + lane;
  int b, nb, qidx;
  if (!token_seq(p.cu_q, p.B, tok, p.n_tok, b, nb, qidx)) {
    *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const int L = p.seq_lens[b];
  if (L < nb || L > p.max_kv_len) {
    *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const int pos = L - nb + qidx;
  const int n = pos / SPLIT + 1;
  const size_t base = ((size_t)tok * p.Hq + h) * p.n_split_max;
  float M = -INFINITY;
  for (int s = 0; s < n; ++s) M = fmaxf(M, p.ws_ml[(base + s) * 2]);
  float Ls = 0.0f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < n; ++s) {
    const float2 ml = *reinterpret_cast<const float2*>(p.ws_ml + (base + s) * 2);
    const float wgt = exp2f(__fsub_rn(ml.x, M));
    Ls = __fmaf_rn(wgt, ml.y, Ls);
    const float4 os = reinterpret_cast<const float4*>(p.ws_o + (base + s) * HD)[lane];
    o.x = __fmaf_rn(wgt, os.x, o.x);
    o.y = __fmaf_rn(wgt, os.y, o.y);
    o.z = __fmaf_rn(wgt, os.z, o.z);
    o.w = __fmaf_rn(wgt, os.w, o.w);
  }
  *dst = make_float4(__fadd_rn(__fdiv_rn(o.x, Ls), 0.0f), __fadd_rn(__fdiv_rn(o.y, Ls), 0.0f),
                     __fadd_rn(__fdiv_rn(o.z, Ls), 0.0f), __fadd_rn(__fdiv_rn(o.w, Ls), 0.0f));
}

}  // namespace up

bi_status launch_split(const float* x, int64_t n, bf16* hi, bf16* lo, cudaStream_t s) {
  if (n == 0) return BI_OK;
  up::split_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(x, n, hi, lo);
  BI_CHECK_LAUNCH("split launch");
  return BI_OK;
}

bi_status launch_swiglu_split(const float* gu, int64_t n_tok, int64_t F, bf16* hi, bf16* lo,
                              cudaStream_t s) {
  const int64_t n = n_tok * F;
  if (n == 0) return BI_OK;
  up::swiglu_split_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(gu, n_tok, F, hi, lo);
  BI_CHECK_LAUNCH("swiglu_split launch");
  return BI_OK;
}

bi_status launch_rope_f32(float* x, int64_t ldx, int n_heads, const int32_t* pos, int64_t n_tok,
                          const float* cs, int max_pos, cudaStream_t s) {
  const int64_t n = n_tok * n_heads * 64;
  if (n == 0) return BI_OK;
  up::rope_f32_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(x, ldx, n_heads, pos, n_tok, cs,
                                                                  max_pos, status_word());
  BI_CHECK_LAUNCH("rope_f32 launch");
  return BI_OK;
}

bi_status launch_kv_append_f32(const float* k, const float* v, int64_t ld, const int32_t* slots,
                               int64_t n_tok, float* kc, float* vc, int Hkv, int num_pages,
                               cudaStream_t s) {
  const int64_t warps = n_tok * Hkv;
  if (warps == 0) return BI_OK;
  up::kv_append_f32_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(
      k, v, ld, slots, n_tok, Hkv, num_pages, kc, vc, status_word());
  BI_CHECK_LAUNCH("kv_append_f32 launch");
  return BI_OK;
}

static size_t attn_f32_ws(int64_t n_tok, int Hq, int n_split) {
  return (size_t)n_tok * Hq * n_split * (up::HD + 2) * sizeof(float);
}

bi_status run_attn_f32(const float* q, int64_t ldq, const int32_t* cu_q, int64_t n_tok,
                       const float* kc, const float* vc, const int32_t* block_table,
                       const int32_t* seq_lens, int32_t B, const bi_attn_shape* sh, float* out,
                       int64_t ldo, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (!sh || !q || !kc || !vc || !block_table || !seq_lens || !out || (n_tok > 0 && !ws))
    return fail(BI_ERR_INVALID_ARG, "attn_f32: null argument");
  if (sh->head_dim != up::HD || sh->page_size != up::PAGE) return fail(BI_ERR_SHAPE, "attn_f32: head_dim 128 and page_size 16 required");
  if (sh->num_q_heads <= 0 || sh->num_kv_heads <= 0 || sh->num_q_heads % sh->num_kv_heads)
    return fail(BI_ERR_SHAPE, "attn_f32: num_q_heads must be a positive multiple of num_kv_heads");
  const int G = sh->num_q_heads / sh->num_kv_heads;
  if (G > 32) return fail(BI_ERR_SHAPE, "attn_f32: at most 32 q heads per kv head");
  if (sh->max_kv_len <= 0 || sh->num_pages <= 0 || sh->max_pages_per_seq <= 0) return fail(BI_ERR_SHAPE, "attn_f32: bad cache shape");
  if (ldq < (int64_t)sh->num_q_heads * up::HD || ldo < (int64_t)sh->num_q_heads * up::HD || ldq % 4 || ldo % 4)
    return fail(BI_ERR_SHAPE, "attn_f32: bad ldq/ldo");
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(out) || !aligned16(ws))
    return fail(BI_ERR_ALIGN, "attn_f32: pointers must be 16-byte aligned");
  if (B == 0 || n_tok == 0) return BI_OK;
  if (n_tok > 65535) return fail(BI_ERR_SHAPE, "attn_f32: at most 65535 tokens per call");
  const int n_split = (sh->max_kv_len + up::SPLIT - 1) / up::SPLIT;
  if (ws_bytes < attn_f32_ws(n_tok, sh->num_q_heads, n_split)) return fail(BI_ERR_WORKSPACE, "attn_f32: workspace too small");
  bi_status st = require_sm100();
  if (st != BI_OK) return st;
  up::AttnParams p;
  p.q = q;
  p.ldq = ldq;
  p.cu_q = cu_q;
  p.kc = kc;
  p.vc = vc;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.ws_o = static_cast<float*>(ws);
  p.ws_ml = p.ws_o + (size_t)n_tok * sh->num_q_heads * n_split * up::HD;
  p.B = B;
  p.Hq = sh->num_q_heads;
  p.Hkv = sh->num_kv_heads;
  p.G = G;
  p.n_tok = (int32_t)n_tok;
  p.num_pages = sh->num_pages;
  p.max_pages = sh->max_pages_per_seq;
  p.max_kv_len = sh->max_kv_len;
  p.n_split_max = n_split;
  p.scale_log2 = (float)((double)sh->scale * 1.4426950408889634);
  p.status = status_word();
  dim3 grid(n_split, (unsigned)n_tok, sh->num_kv_heads);
  up::attn_f32_split_kernel<<<grid, 32 * G, G * up::SPLIT * sizeof(float), s>>>(p);
  BI_CHECK_LAUNCH("attn_f32 split launch");
  const int64_t warps = n_tok * sh->num_q_heads;
  up::attn_f32_combine_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(p, out, ldo);
  BI_CHECK_LAUNCH("attn_f32 combine launch");
  return BI_OK;
}

size_t attn_f32_workspace(int64_t n_tok, int Hq, int max_kv_len) {
  return attn_f32_ws(n_tok, Hq, (max_kv_len + up::SPLIT - 1) / up::SPLIT);
}

}  // namespace bi

using namespace bi;

extern "C" bi_status bi_split_bf16x2(const float* x, int64_t n, void* hi, void* lo, void* stream) {
  if (!x || !hi || !lo || n < 0) return fail(BI_ERR_INVALID_ARG, "split_bf16x2: bad arguments");
  if (n == 0) return BI_OK;
  bi_status st = require_sm100();
  if (st != BI_OK) return st;
  return launch_split(x, n, static_cast<bf16*>(hi), static_cast<bf16*>(lo), static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_attn_f32(const float* q, int64_t ldq, const int32_t* cu_q, int64_t n_tok,
                                 const float* k_cache, const float* v_cache,
                                 const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                                 const bi_attn_shape* shape, float* out, int64_t ldo, void* ws,
                                 size_t ws_bytes, void* stream) {
  if (!cu_q && n_tok != B) return fail(BI_ERR_INVALID_ARG, "attn_f32: without cu_q, n_tok must equal B (decode)");
  return run_attn_f32(q, ldq, cu_q, n_tok, k_cache, v_cache, block_table, seq_lens, B, shape, out,
                      ldo, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_attn_f32_workspace_size(const bi_attn_shape* shape, int64_t max_tokens,
                                                size_t* bytes) {
  if (!shape || !bytes || max_tokens < 0 || shape->max_kv_len <= 0 || shape->num_q_heads <= 0)
    return fail(BI_ERR_INVALID_ARG, "attn_f32_workspace_size: bad arguments");
  *bytes = attn_f32_workspace(max_tokens, shape->num_q_heads, shape->max_kv_len);
  return BI_OK;
}
