// forward.cu -- one step of a dense pre-norm decoder, composed only of the
// batch-invariant kernels of this library.
//
// Per layer: RMSNorm -> QKV GEMM -> RoPE(q, k) -> KV-cache append -> paged
// attention (split + ordered merge) -> O GEMM (fp32 out) -> residual add ->
// RMSNorm -> gate/up GEMM -> SwiGLU -> down GEMM (fp32 out) -> residual add.
// Then the final RMSNorm of the rows that want logits and the LM-head GEMM
// with fp32 logits, and optionally the greedy argmax. In the bf16 mode the
// residual adds and SwiGLU run in the GEMM epilogues, and so do RoPE and the
// cache append when the QKV projection has a tile for every SM; each fused
// step keeps the separate kernel's rounding points, so the bits are the same.
//
// Every kernel computes each row (token) with an order that depends only on
// that row's data and, for attention, on its sequence's cache, so a
// sequence's logits are the same bits whatever else shares the step
// ("Defeating Nondeterminism in LLM Inference", sections "Batch invariance and
// determinism" and "How do we make kernels batch-invariant?"). The residual
// stream is kept in fp32 and the two GEMMs that feed it write fp32 (a reading:
// the pages fix no activation precision; this keeps the stream's rounding
// error below the bf16 inputs'). The fp32-activation modes (the cross-vendor
// paper's FP32 upcast and its BF16-MLP-only variant) swap the attention
// and/or MLP block for the upcast kernels of upcast.cu.
#include <stdlib.h>

#include "common.cuh"
#include "host.h"

namespace bi {
bi_status launch_kv_append(const uint16_t* k, const uint16_t* v, int64_t ld_new, const int32_t* slots,
                           int64_t n_tok, uint16_t* kc, uint16_t* vc, int Hkv, int num_pages,
                           cudaStream_t s);
template <typename ET>
bi_status launch_embed(const int32_t* tok, int64_t n_tok, const ET* table, int64_t vocab,
                       int64_t D, float* out, cudaStream_t s);
template <typename ET>
bi_status launch_rope(ET* x, int64_t ldx, int n_heads, const int32_t* pos, int64_t n_tok,
                      const float* cs, int max_pos, cudaStream_t s);
template <typename ET>
bi_status gemm_e16(const void* A, int64_t lda, const void* W, int64_t ldw, void* C, int64_t ldc,
                   int32_t c_dtype, int64_t M, int64_t N, int64_t K, cudaStream_t s);
template <typename ET>
bi_status gemm_swiglu_e16(const void* A, int64_t lda, const void* W, int64_t ldw, void* out,
                          int64_t ldo, int64_t M, int64_t F, int64_t K, cudaStream_t s);
template <typename ET>
bi_status gemm_qkv_e16(const void* A, int64_t lda, const void* W, int64_t ldw, void* qkv, int64_t ldq,
                       int64_t M, int64_t K, int32_t n_q_heads, int32_t n_kv_heads, const int32_t* positions,
                       const float* cos_sin, int32_t max_pos, const int32_t* slot_mapping, void* k_cache,
                       void* v_cache, int32_t num_pages, cudaStream_t s);
bi_status rmsnorm_f32in_f16(const float* x, const void* gamma, void* y, int64_t M, int64_t D, float eps,
                            cudaStream_t s);
bi_status attn_decode_f16(const void* q, int64_t ldq, const void* k_cache, const void* v_cache,
                          const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                          const bi_attn_shape* shape, void* out, int64_t ldo, void* ws, size_t ws_bytes,
                          cudaStream_t s);
bi_status attn_prefill_f16(const void* q, int64_t ldq, const int32_t* cu_q, int32_t max_q_len, int64_t n_tok,
                           const void* k_cache, const void* v_cache, const int32_t* block_table,
                           const int32_t* seq_lens, int32_t B, const bi_attn_shape* shape, void* out,
                           int64_t ldo, void* ws, size_t ws_bytes, cudaStream_t s);
bi_status launch_argmax(const float* logits, int64_t rows, int64_t V, int64_t ld, int32_t* idx,
                        cudaStream_t s);
bi_status launch_split(const float* x, int64_t n, bf16* hi, bf16* lo, cudaStream_t s);
bi_status launch_swiglu_split(const float* gu, int64_t n_tok, int64_t F, bf16* hi, bf16* lo,
                              cudaStream_t s);
bi_status launch_rope_f32(float* x, int64_t ldx, int n_heads, const int32_t* pos, int64_t n_tok,
                          const float* cs, int max_pos, cudaStream_t s);
bi_status launch_kv_append_f32(const float* k, const float* v, int64_t ld, const int32_t* slots,
                               int64_t n_tok, float* kc, float* vc, int Hkv, int num_pages,
                               cudaStream_t s);
bi_status run_attn_f32(const float* q, int64_t ldq, const int32_t* cu_q, int64_t n_tok,
                       const float* kc, const float* vc, const int32_t* block_table,
                       const int32_t* seq_lens, int32_t B, const bi_attn_shape* sh, float* out,
                       int64_t ldo, void* ws, size_t ws_bytes, cudaStream_t s);
size_t attn_f32_workspace(int64_t n_tok, int Hq, int max_kv_len);

namespace fwd {

__global__ void gather_rows_kernel(const float* __restrict__ x, const int32_t* __restrict__ rows,
                                   int64_t n_rows, int64_t n_tok, int D, float* __restrict__ out,
                                   int32_t* status) {
  const int64_t r = blockIdx.x;
  const int32_t src = rows[r];
  const bool ok = src >= 0 && src < n_tok;
  if (!ok && threadIdx.x == 0) set_status(status, BI_DEV_BAD_TOKEN);
  for (int c = threadIdx.x; c < D; c += blockDim.x)
    out[r * D + c] = ok ? x[(size_t)src * D + c] : 0.0f;
}

struct Layout {  // workspace carve-up, all offsets 256-byte aligned
  size_t x, h, h_lo, qkv, qkv32, att, att_lo, att32, gu32, act, act_lo, xl, hl, hl_lo,
      rope, attn_ws, total;
  size_t attn_ws_bytes;
};

static size_t up(size_t v) { return (v + 255) & ~(size_t)255; }

static Layout layout(const bi_model_config& c, int64_t T, int64_t NL, int32_t max_kv_len) {
  Layout L;
  const size_t D = c.d_model, F = c.d_ff;
  const size_t QKV = (size_t)(c.n_q_heads + 2 * c.n_kv_heads) * BI_HEAD_DIM;
  const bool f32 = c.precision != BI_PREC_BF16;  // fp32 buffers needed
  size_t o = 0;
  L.x = o; o += up(T * D * 4);
  L.h = o; o += up(T * D * 2);
  L.h_lo = o; o += f32 ? up(T * D * 2) : 0;
  L.qkv = o; o += up(T * QKV * 2);
  L.qkv32 = o; o += f32 ? up(T * QKV * 4) : 0;
  L.att = o; o += up(T * D * 2);
  L.att_lo = o; o += f32 ? up(T * D * 2) : 0;
  L.att32 = o; o += f32 ? up(T * D * 4) : 0;
  L.gu32 = o; o += c.precision == BI_PREC_F32 ? up(T * 2 * F * 4) : 0;
  L.act = o; o += up(T * F * 2);
  L.act_lo = o; o += c.precision == BI_PREC_F32 ? up(T * F * 2) : 0;
  L.xl = o; o += up(NL * D * 4);
  L.hl = o; o += up(NL * D * 2);
  L.hl_lo = o; o += f32 ? up(NL * D * 2) : 0;
  L.rope = o; o += up((size_t)c.max_pos * 64 * 2 * 4);
  bi_attn_shape sh;
  sh.num_q_heads = c.n_q_heads;
  sh.num_kv_heads = c.n_kv_heads;
  sh.head_dim = BI_HEAD_DIM;
  sh.page_size = BI_PAGE_SIZE;
  sh.num_pages = 1;
  sh.max_pages_per_seq = 1;
  sh.max_kv_len = max_kv_len > 0 ? max_kv_len : 1;
  sh.scale = 1.0f;
  size_t a = 0;
  bi_attn_workspace_size(&sh, T, &a);
  const size_t a32 = attn_f32_workspace(T, c.n_q_heads, sh.max_kv_len);
  if (a32 > a) a = a32;
  L.attn_ws = o; o += up(a);
  L.attn_ws_bytes = a;
  L.total = o;
  return L;
}

}  // namespace fwd
}  // namespace bi

struct bi_model {
  bi_model_config cfg;
  bi_model_weights w;
};

using namespace bi;

extern "C" bi_status bi_model_create(const bi_model_config* cfg, const bi_model_weights* w,
                                     bi_model** out) {
  if (!cfg || !w || !out) return fail(BI_ERR_INVALID_ARG, "model_create: null argument");
  const bi_model_config& c = *cfg;
  if (c.n_layers < 0 || c.d_model <= 0 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 || c.d_ff <= 0 ||
      c.vocab <= 0 || c.max_pos <= 0)
    return fail(BI_ERR_INVALID_ARG, "model_create: sizes must be positive");
  if (c.d_model != c.n_q_heads * BI_HEAD_DIM) return fail(BI_ERR_SHAPE, "model_create: d_model must equal n_q_heads * 128");
  if (c.n_q_heads % c.n_kv_heads) return fail(BI_ERR_SHAPE, "model_create: n_q_heads must be a multiple of n_kv_heads");
  const int G = c.n_q_heads / c.n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(BI_ERR_SHAPE, "model_create: q heads per kv head must be 1, 2, 4 or 8");
  if (c.d_ff % 8 || c.vocab % 8) return fail(BI_ERR_SHAPE, "model_create: d_ff and vocab must be multiples of 8");
  if (!(c.rms_eps >= 0.0f) || !(c.rope_theta > 1.0)) return fail(BI_ERR_INVALID_ARG, "model_create: bad eps or rope_theta");
  if (c.precision != BI_PREC_BF16 && c.precision != BI_PREC_F32 && c.precision != BI_PREC_BF16_MLP &&
      c.precision != BI_PREC_F16)
    return fail(BI_ERR_INVALID_ARG, "model_create: unknown precision %d", c.precision);
  if (!w->embed || !w->final_norm || !w->lm_head) return fail(BI_ERR_INVALID_ARG, "model_create: missing weights");
  if (c.n_layers > 0 && (!w->attn_norm || !w->w_qkv || !w->w_o || !w->mlp_norm || !w->w_gate_up || !w->w_down))
    return fail(BI_ERR_INVALID_ARG, "model_create: missing layer weights");
  bi_model* m = static_cast<bi_model*>(malloc(sizeof(bi_model)));
  if (!m) return fail(BI_ERR_INVALID_ARG, "model_create: out of host memory");
  m->cfg = c;
  m->w = *w;
  *out = m;
  return BI_OK;
}

extern "C" void bi_model_destroy(bi_model* m) { free(m); }

extern "C" bi_status bi_forward_workspace_size(const bi_model* m, int64_t max_tokens,
                                               int64_t max_logits, int32_t max_kv_len,
                                               size_t* bytes) {
  if (!m || !bytes || max_tokens < 0 || max_logits < 0 || max_kv_len <= 0)
    return fail(BI_ERR_INVALID_ARG, "forward_workspace_size: bad arguments");
  *bytes = fwd::layout(m->cfg, max_tokens, max_logits, max_kv_len).total;
  return BI_OK;
}

#define BI_TRY(expr)                     \
  do {                                   \
    bi_status st_ = (expr);              \
    if (st_ != BI_OK) return st_;        \
  } while (0)

extern "C" bi_status bi_forward(const bi_model* m, const bi_batch* bt, void* k_cache,
                                void* v_cache, int32_t num_pages, float* logits,
                                int32_t* next_tokens, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !bt || !k_cache || !v_cache || !logits || !ws) return fail(BI_ERR_INVALID_ARG, "forward: null argument");
  const bi_model_config& c = m->cfg;
  const bi_batch& b = *bt;
  if (b.n_tok <= 0 || b.B <= 0 || b.n_logits < 0 || b.max_q_len <= 0 || b.max_kv_len <= 0 || b.max_pages_per_seq <= 0 || num_pages <= 0)
    return fail(BI_ERR_INVALID_ARG, "forward: bad batch sizes");
  if (!b.tokens || !b.positions || !b.slot_mapping || !b.cu_q || !b.seq_lens || !b.block_table || (b.n_logits && !b.logits_rows))
    return fail(BI_ERR_INVALID_ARG, "forward: null batch array");
  if (b.max_kv_len > c.max_pos) return fail(BI_ERR_SHAPE, "forward: max_kv_len above max_pos");
  if (b.n_decode < 0 || b.n_decode > b.B || b.n_decode > b.n_tok)
    return fail(BI_ERR_INVALID_ARG, "forward: n_decode %d outside 0 .. B", b.n_decode);
  const fwd::Layout L = fwd::layout(c, b.n_tok, b.n_logits, b.max_kv_len);
  if (ws_bytes < L.total) return fail(BI_ERR_WORKSPACE, "forward: workspace %zu < %zu", ws_bytes, L.total);
  if (!aligned16(ws) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(logits))
    return fail(BI_ERR_ALIGN, "forward: pointers must be 16-byte aligned");
  BI_TRY(require_sm100());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* x = reinterpret_cast<float*>(base + L.x);
  bf16* h = reinterpret_cast<bf16*>(base + L.h);
  bf16* h_lo = reinterpret_cast<bf16*>(base + L.h_lo);
  bf16* qkv = reinterpret_cast<bf16*>(base + L.qkv);
  float* qkv32 = reinterpret_cast<float*>(base + L.qkv32);
  bf16* att = reinterpret_cast<bf16*>(base + L.att);
  bf16* att_lo = reinterpret_cast<bf16*>(base + L.att_lo);
  float* att32 = reinterpret_cast<float*>(base + L.att32);
  float* gu32 = reinterpret_cast<float*>(base + L.gu32);
  bf16* act = reinterpret_cast<bf16*>(base + L.act);
  bf16* act_lo = reinterpret_cast<bf16*>(base + L.act_lo);
  float* xl = reinterpret_cast<float*>(base + L.xl);
  bf16* hl = reinterpret_cast<bf16*>(base + L.hl);
  bf16* hl_lo = reinterpret_cast<bf16*>(base + L.hl_lo);
  float* rope = reinterpret_cast<float*>(base + L.rope);
  void* attn_ws = base + L.attn_ws;

  const bool f16m = c.precision == BI_PREC_F16;       // the 16-bit path in fp16
  const bool attn_f32 = c.precision == BI_PREC_F32 || c.precision == BI_PREC_BF16_MLP;  // attention block (and LM head) upcast
  const bool mlp_f32 = c.precision == BI_PREC_F32;    // MLP block upcast
  const int64_t T = b.n_tok, D = c.d_model, F = c.d_ff;
  const int Hq = c.n_q_heads, Hkv = c.n_kv_heads;
  const int64_t QKV = (int64_t)(Hq + 2 * Hkv) * BI_HEAD_DIM;
  const size_t cache_layer = (size_t)num_pages * Hkv * BI_PAGE_SIZE * BI_HEAD_DIM;
  // a pair of CTAs per 256 x BI_GEMM_BN output tile
  const bool qkv_fused = ((T + BI_GEMM_BM - 1) / BI_GEMM_BM) * ((QKV + BI_GEMM_BN - 1) / BI_GEMM_BN) >= num_sms() / 2;

  BI_TRY(bi_rope_table(rope, c.max_pos, c.rope_theta, stream));
  if (f16m) BI_TRY(launch_embed<f16>(b.tokens, T, static_cast<const f16*>(m->w.embed), c.vocab, D, x, s));
  else BI_TRY(launch_embed<bf16>(b.tokens, T, static_cast<const bf16*>(m->w.embed), c.vocab, D, x, s));

  bi_attn_shape sh;
  sh.num_q_heads = Hq;
  sh.num_kv_heads = Hkv;
  sh.head_dim = BI_HEAD_DIM;
  sh.page_size = BI_PAGE_SIZE;
  sh.num_pages = num_pages;
  sh.max_pages_per_seq = b.max_pages_per_seq;
  sh.max_kv_len = b.max_kv_len;
  sh.scale = (float)(1.0 / sqrt((double)BI_HEAD_DIM));

  for (int l = 0; l < c.n_layers; ++l) {
    const bf16* attn_norm = static_cast<const bf16*>(m->w.attn_norm) + (size_t)l * D;
    const bf16* mlp_norm = static_cast<const bf16*>(m->w.mlp_norm) + (size_t)l * D;
    const bf16* w_qkv = static_cast<const bf16*>(m->w.w_qkv) + (size_t)l * QKV * D;
    const bf16* w_o = static_cast<const bf16*>(m->w.w_o) + (size_t)l * D * D;
    const bf16* w_gu = static_cast<const bf16*>(m->w.w_gate_up) + (size_t)l * 2 * F * D;
    const bf16* w_d = static_cast<const bf16*>(m->w.w_down) + (size_t)l * D * F;

    // ---- attention block
    if (attn_f32) {
      float* kc = static_cast<float*>(k_cache) + (size_t)l * cache_layer;
      float* vc = static_cast<float*>(v_cache) + (size_t)l * cache_layer;
      BI_TRY(bi_rmsnorm_split(x, attn_norm, h, h_lo, T, D, c.rms_eps, stream));
      BI_TRY(bi_gemm_x2(h, h_lo, D, w_qkv, D, qkv32, QKV, BI_F32, T, QKV, D, stream));
      BI_TRY(launch_rope_f32(qkv32, QKV, Hq, b.positions, T, rope, c.max_pos, s));
      BI_TRY(launch_rope_f32(qkv32 + (size_t)Hq * BI_HEAD_DIM, QKV, Hkv, b.positions, T, rope, c.max_pos, s));
      BI_TRY(launch_kv_append_f32(qkv32 + (size_t)Hq * BI_HEAD_DIM,
                                  qkv32 + (size_t)(Hq + Hkv) * BI_HEAD_DIM, QKV, b.slot_mapping, T,
                                  kc, vc, Hkv, num_pages, s));
      BI_TRY(run_attn_f32(qkv32, QKV, b.cu_q, T, kc, vc, b.block_table, b.seq_lens, b.B, &sh, att32,
                          D, attn_ws, L.attn_ws_bytes, s));
      BI_TRY(launch_split(att32, T * D, att, att_lo, s));
      BI_TRY(bi_gemm_x2(att, att_lo, D, w_o, D, x, D, BI_F32_ADD, T, D, D, stream));  // x += O proj
    } else {
      uint16_t* kc = static_cast<uint16_t*>(k_cache) + (size_t)l * cache_layer;
      uint16_t* vc = static_cast<uint16_t*>(v_cache) + (size_t)l * cache_layer;
      BI_TRY(f16m ? rmsnorm_f32in_f16(x, attn_norm, h, T, D, c.rms_eps, s)
                  : bi_rmsnorm_f32in(x, attn_norm, h, T, D, c.rms_eps, stream));
      // QKV projection, RoPE of the q and k heads, cache write: one launch
      // when every SM gets at least one output tile (RoPE and the scattered
      // cache stores then spread over all SMs and overlap later tiles'
      // MMAs); for fewer tiles the epilogue work would sit on those few SMs
      // after their only tile, so three launches are faster. Same bits.
      if (qkv_fused) {
        BI_TRY(f16m ? gemm_qkv_e16<f16>(h, D, w_qkv, D, qkv, QKV, T, D, Hq, Hkv, b.positions, rope, c.max_pos,
                                        b.slot_mapping, kc, vc, num_pages, s)
                    : gemm_qkv_e16<bf16>(h, D, w_qkv, D, qkv, QKV, T, D, Hq, Hkv, b.positions, rope, c.max_pos,
                                         b.slot_mapping, kc, vc, num_pages, s));
      } else {
        BI_TRY(f16m ? gemm_e16<f16>(h, D, w_qkv, D, qkv, QKV, BI_BF16, T, QKV, D, s)
                    : gemm_e16<bf16>(h, D, w_qkv, D, qkv, QKV, BI_BF16, T, QKV, D, s));
        // q and k heads are adjacent in a qkv row: one launch rotates both
        if (f16m) BI_TRY(launch_rope<f16>(reinterpret_cast<f16*>(qkv), QKV, Hq + Hkv, b.positions, T, rope, c.max_pos, s));
        else BI_TRY(launch_rope<bf16>(qkv, QKV, Hq + Hkv, b.positions, T, rope, c.max_pos, s));
        BI_TRY(launch_kv_append(reinterpret_cast<const uint16_t*>(qkv + (size_t)Hq * BI_HEAD_DIM),
                                reinterpret_cast<const uint16_t*>(qkv + (size_t)(Hq + Hkv) * BI_HEAD_DIM),
                                QKV, b.slot_mapping, T, kc, vc, Hkv, num_pages, s));
      }
      // one-token sequences go through the decode kernel, longer chunks
      // through the prefill kernel; a row gets the same bits from either
      // (same tiles, splits and per-row arithmetic)
      const int32_t nd = (T == b.B && b.max_q_len == 1) ? b.B : b.n_decode;
      if (nd > 0)
        BI_TRY(f16m ? attn_decode_f16(qkv, QKV, kc, vc, b.block_table, b.seq_lens, nd, &sh, att, D, attn_ws,
                                      L.attn_ws_bytes, s)
                    : bi_attn_decode(qkv, QKV, kc, vc, b.block_table, b.seq_lens, nd, &sh, att, D, attn_ws,
                                     L.attn_ws_bytes, stream));
      if (nd < b.B)
        BI_TRY(f16m ? attn_prefill_f16(qkv, QKV, b.cu_q + nd, b.max_q_len, T, kc, vc,
                                       b.block_table + (size_t)nd * b.max_pages_per_seq, b.seq_lens + nd, b.B - nd,
                                       &sh, att, D, attn_ws, L.attn_ws_bytes, s)
                    : bi_attn_prefill(qkv, QKV, b.cu_q + nd, b.max_q_len, T, kc, vc,
                                      b.block_table + (size_t)nd * b.max_pages_per_seq, b.seq_lens + nd, b.B - nd,
                                      &sh, att, D, attn_ws, L.attn_ws_bytes, stream));
      BI_TRY(f16m ? gemm_e16<f16>(att, D, w_o, D, x, D, BI_F32_ADD, T, D, D, s)
                  : bi_gemm(att, D, w_o, D, x, D, BI_F32_ADD, T, D, D, stream));  // x += O proj
    }

    // ---- MLP block
    if (mlp_f32) {
      BI_TRY(bi_rmsnorm_split(x, mlp_norm, h, h_lo, T, D, c.rms_eps, stream));
      BI_TRY(bi_gemm_x2(h, h_lo, D, w_gu, D, gu32, 2 * F, BI_F32, T, 2 * F, D, stream));
      BI_TRY(launch_swiglu_split(gu32, T, F, act, act_lo, s));
      BI_TRY(bi_gemm_x2(act, act_lo, F, w_d, F, x, D, BI_F32_ADD, T, D, F, stream));  // x += down proj
    } else {
      BI_TRY(f16m ? rmsnorm_f32in_f16(x, mlp_norm, h, T, D, c.rms_eps, s)
                  : bi_rmsnorm_f32in(x, mlp_norm, h, T, D, c.rms_eps, stream));
      // act = swiglu(gate, up); x += down proj
      BI_TRY(f16m ? gemm_swiglu_e16<f16>(h, D, w_gu, D, act, F, T, F, D, s)
                  : gemm_swiglu_e16<bf16>(h, D, w_gu, D, act, F, T, F, D, s));
      BI_TRY(f16m ? gemm_e16<f16>(act, F, w_d, F, x, D, BI_F32_ADD, T, D, F, s)
                  : gemm_e16<bf16>(act, F, w_d, F, x, D, BI_F32_ADD, T, D, F, s));
    }
  }
  if (b.n_logits == 0) return BI_OK;
  fwd::gather_rows_kernel<<<(unsigned)b.n_logits, 256, 0, s>>>(x, b.logits_rows, b.n_logits, T,
                                                               (int)D, xl, status_word());
  BI_CHECK_LAUNCH("forward gather");
  if (attn_f32) {
    BI_TRY(bi_rmsnorm_split(xl, m->w.final_norm, hl, hl_lo, b.n_logits, D, c.rms_eps, stream));
    BI_TRY(bi_gemm_x2(hl, hl_lo, D, m->w.lm_head, D, logits, c.vocab, BI_F32, b.n_logits, c.vocab, D,
                      stream));
  } else {
    BI_TRY(f16m ? rmsnorm_f32in_f16(xl, m->w.final_norm, hl, b.n_logits, D, c.rms_eps, s)
                : bi_rmsnorm_f32in(xl, m->w.final_norm, hl, b.n_logits, D, c.rms_eps, stream));
    BI_TRY(f16m ? gemm_e16<f16>(hl, D, m->w.lm_head, D, logits, c.vocab, BI_F32, b.n_logits, c.vocab, D, s)
                : gemm_e16<bf16>(hl, D, m->w.lm_head, D, logits, c.vocab, BI_F32, b.n_logits, c.vocab, D, s));
  }
  if (next_tokens) BI_TRY(launch_argmax(logits, b.n_logits, c.vocab, c.vocab, next_tokens, s));
  return BI_OK;
}
