/*
 * bi.h -- C ABI of libbi, batch-invariant inference kernels for NVIDIA B200 (sm_100a).
 *
 * What "batch-invariant" means here follows "Defeating Nondeterminism in LLM
 * Inference" (section "Batch invariance and determinism"): the value computed
 * for one row (one token) must not depend on how many other rows share the
 * launch, where in the batch the row sits, how the engine chunked its
 * sequence, or which run it is. Every kernel behind this header fixes the
 * floating-point reduction order of each output element as a function of the
 * reduced length only.
 *
 * Conventions shared by every entry point
 *  - All tensor arguments are DEVICE pointers owned by the caller. bf16 data
 *    is passed as `void*` (IEEE bfloat16, 2 bytes, round-to-nearest-even).
 *    Matrices are row-major; leading dimensions (ld*) count ELEMENTS.
 *  - `stream` is a cudaStream_t passed as `void*` (NULL = legacy stream).
 *    Every call is asynchronous on that stream; nothing synchronises the host
 *    except bi_device_status().
 *  - Arguments are validated on the host before anything is launched. On a
 *    non-BI_OK return nothing was enqueued and bi_last_error() (thread-local)
 *    holds a one-line reason.
 *  - No entry point allocates device memory. Scratch space is a caller-owned
 *    workspace whose size comes from the matching *_workspace_size query,
 *    with one exception: bi_attn_decode_noalloc takes no workspace and uses
 *    a fixed static device array of the library instead, shared by all calls
 *    on a device.
 *  - Data that only the device can see (page ids, slot ids, sequence lengths)
 *    is range-checked inside the kernels: an out-of-range value skips the
 *    access and sets a bit of the library's device status word, read with
 *    bi_device_status(). Kernels never trap and every device-side wait is
 *    bounded (a timeout also sets a status bit and the kernel returns).
 *  - No reduction uses atomics, split-K or stream-K; the launch shape never
 *    depends on the batch size in a way that reaches the arithmetic.
 */
#ifndef BI_H_
#define BI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BI_OK = 0,
  BI_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum */
  BI_ERR_SHAPE = 2,       /* size outside what the kernel supports */
  BI_ERR_ALIGN = 3,       /* pointer or leading dimension misaligned */
  BI_ERR_WORKSPACE = 4,   /* workspace missing or too small */
  BI_ERR_UNSUPPORTED = 5, /* no sm_100 device / feature unavailable */
  BI_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed */
  BI_ERR_DEVICE_CHECK = 7 /* device status word non-zero (bi_device_status) */
} bi_status;

/* Output element types of the GEMMs. BI_F32_ADD: C is fp32 and the product
 * is added to it (C = C + A W^T, one fp32 addition per element after the
 * whole K reduction), as a residual connection into an fp32 stream. */
typedef enum { BI_BF16 = 0, BI_F32 = 1, BI_F32_ADD = 2 } bi_dtype;

/* Fixed geometry. These are compile-time constants on purpose: a tile or split
 * size chosen at run time from the problem shape would make the reduction order
 * depend on the batch, which is exactly what the library must not do. */
#define BI_HEAD_DIM 128   /* attention head dimension d_h */
#define BI_PAGE_SIZE 16   /* tokens per KV-cache page */
#define BI_ATTN_TILE 128  /* keys per attention tile, at absolute key offsets */
#define BI_ATTN_SPLIT 512 /* keys per KV split (fixed split SIZE, not count) */
#define BI_GEMM_BM 256    /* GEMM output tile rows (a CTA pair, 128 rows each) */
#define BI_GEMM_BN 256    /* GEMM output tile columns */
#define BI_GEMM_BK 64     /* GEMM K stage */

/* Device status word bits (bi_device_status). */
#define BI_DEV_WAIT_TIMEOUT 0x1 /* a bounded mbarrier wait ran out */
#define BI_DEV_BAD_SLOT 0x2     /* slot_mapping entry outside the cache */
#define BI_DEV_BAD_PAGE 0x4     /* block_table entry outside the cache */
#define BI_DEV_BAD_SEQLEN 0x8   /* seq_lens entry outside [n_query, max_kv_len], or a prefill
                                   chunk with more than max_q_len rows */
#define BI_DEV_BAD_TOKEN 0x10   /* token id outside the vocabulary */

/* Thread-local description of the last failure on this host thread. */
const char* bi_last_error(void);

/* Reads the device status word of the current device into *status (after
 * synchronising `stream`), and clears it when `clear` is non-zero.
 * Returns BI_ERR_DEVICE_CHECK when the word was non-zero. */
bi_status bi_device_status(int32_t* status, int32_t clear, void* stream);

/* Self-check of the device wait bound (no counterpart on the pages; a test
 * and diagnostic entry point). Launches one CTA whose threads wait on an
 * mbarrier that nothing ever arrives on, through the same bounded wait the
 * kernels use, giving up after `limit_cycles` SM clock cycles (1000 .. 2^32;
 * the kernels use 2^32, about 2 s): the kernel then sets BI_DEV_WAIT_TIMEOUT
 * in the status word and returns, leaving the context usable. Nothing faults,
 * traps or hangs. BI_ERR_INVALID_ARG for a limit outside the range. */
bi_status bi_check_wait_bound(int64_t limit_cycles, void* stream);

/* ------------------------------------------------------------------------ */
/* RMSNorm.  "Defeating Nondeterminism in LLM Inference", section
 * "Batch-invariant RMSNorm": the reference definition x * rsqrt(mean(x^2)) *
 * weight, parallelised with one row per core so that no row's reduction is
 * ever split. eps is added inside the square root.
 *
 *   y[i, :] = bf16( x[i, :] * r_i * gamma ),  r_i = 1 / sqrt(sum_j x_ij^2 / D + eps)
 *
 * x [M, D] bf16 row-major (ld = D), gamma [D] bf16, y [M, D] bf16.
 * The sum of squares is fp32 in an order that depends on D only: each thread
 * adds its 8-element chunks in sequence, then a warp shuffle tree, then warp
 * partials in warp order. Needs D % 8 == 0, 8 <= D <= 32768, pointers 16-byte
 * aligned. M == 0 is a no-op. One CTA per row. */
bi_status bi_rmsnorm(const void* x, const void* gamma, void* y, int64_t M,
                     int64_t D, float eps, void* stream);

/* Same reduction, fp32 input rows (the residual stream of bi_forward) and bf16
 * output. x [M, D] fp32. */
bi_status bi_rmsnorm_f32in(const float* x, const void* gamma, void* y,
                           int64_t M, int64_t D, float eps, void* stream);

/* ------------------------------------------------------------------------ */
/* GEMM.  "Defeating Nondeterminism in LLM Inference", section "Batch-invariant
 * matmul": a data-parallel output tiling with each K reduction inside one
 * core, one kernel configuration for every shape, no split-K, no stream-K.
 *
 *   C[m, n] = sum_k A[m, k] * W[n, k]        (C = A * W^T, nn.Linear layout)
 *
 * A [M, K] bf16 (row stride lda), W [N, K] bf16 (row stride ldw), C [M, N]
 * (row stride ldc) bf16 (c_dtype = BI_BF16, round-to-nearest-even) or fp32
 * (BI_F32). Products are exact, accumulation is fp32 in tensor memory. One
 * configuration for every shape: 256 x 256 output tiles, each computed by a
 * pair of CTAs (a two-CTA cluster, 128 rows each) with one tcgen05.mma
 * kind::f16 shape (cta_group::2, 256 x 256 x 16), K walked 0, 16, 32, ... in
 * order inside the pair whatever M is. Needs K % 8 == 0, N % 8 == 0,
 * lda/ldw/ldc % 8 == 0, A, W, C 16-byte aligned. M == 0 or N == 0 is a
 * no-op. K == 0 writes zeros. */
bi_status bi_gemm(const void* A, int64_t lda, const void* W, int64_t ldw,
                  void* C, int64_t ldc, int32_t c_dtype, int64_t M, int64_t N,
                  int64_t K, void* stream);

/* bi_gemm with fp16 A and W (C fp16 for BI_BF16's slot, i.e. the 16-bit
 * output, or fp32 / fp32-add): the GEMM of the FP16 variant of the
 * cross-vendor paper's precision study (arXiv 2610.05458, abstract). The
 * same tiles, instruction shape (kind::f16 with fp16 operands) and K order;
 * the same constraints. */
bi_status bi_gemm_f16(const void* A, int64_t lda, const void* W, int64_t ldw,
                      void* C, int64_t ldc, int32_t c_dtype, int64_t M,
                      int64_t N, int64_t K, void* stream);

/* Gate/up projection with the SwiGLU activation in its epilogue. W is
 * [2F, K] (row stride ldw): gate rows 0..F-1, then up rows F..2F-1, as a
 * fused nn.Linear. out [M, F] bf16 (row stride ldo):
 *   g = bf16(A Wg^T), u = bf16(A Wu^T) exactly as bi_gemm computes them,
 *   out = bf16(g / (1 + e^-g) * u) in fp32 (the same steps as bi_swiglu).
 * Each 256 x 256 tile holds 128 gate and the matching 128 up columns, so the
 * per-element reduction is bi_gemm's, whatever M is. Constraints as bi_gemm
 * with N = F. */
bi_status bi_gemm_swiglu(const void* A, int64_t lda, const void* W,
                         int64_t ldw, void* out, int64_t ldo, int64_t M,
                         int64_t F, int64_t K, void* stream);

/* QKV projection with RoPE and the KV-cache write in its epilogue. W is the
 * fused [(Hq + 2 Hkv) * 128, K] weight (q heads, then k heads, then v heads,
 * 128 rows each, row stride ldw); qkv [M, (Hq + 2 Hkv) * 128] bf16 (row
 * stride ldq). The result is the same bits as these three calls in order:
 *   bi_gemm(A, lda, W, ldw, qkv, ldq, BI_BF16, M, (Hq + 2 Hkv) * 128, K);
 *   bi_rope(qkv, ldq, Hq + Hkv, positions, M, cos_sin, max_pos);
 *   bi_kv_append(k heads of qkv, v heads of qkv, ldq, slot_mapping, M, ...);
 * i.e. qkv holds the rotated q and k heads and the plain v heads, and row
 * m's k and v heads are in the caches at slot_mapping[m] (skipped when < 0;
 * outside the cache: skipped and BI_DEV_BAD_SLOT). One launch (K == 0: the
 * zeros, then the RoPE and append steps as separate launches). cos_sin
 * [max_pos, 64, 2] fp32 from bi_rope_table; caches as for bi_kv_append
 * (num_pages pages, Hkv heads). Constraints as bi_gemm; caches and cos_sin
 * 16-byte aligned. M == 0 is a no-op. */
bi_status bi_gemm_qkv(const void* A, int64_t lda, const void* W, int64_t ldw,
                      void* qkv, int64_t ldq, int64_t M, int64_t K,
                      int32_t n_q_heads, int32_t n_kv_heads,
                      const int32_t* positions, const float* cos_sin,
                      int32_t max_pos, const int32_t* slot_mapping,
                      void* k_cache, void* v_cache, int32_t num_pages,
                      void* stream);

/* RMSNorm folded into the next GEMM's A operand ("Defeating Nondeterminism
 * in LLM Inference", sections "Batch-invariant RMSNorm" and "Batch-invariant
 * matmul": the norm's per-row reduction and the matmul's per-element K loop
 * keep their own fixed orders, so the fused op is batch-invariant too).
 *   bi_gemm_rmsnorm:        C = bi_gemm(bi_rmsnorm_f32in(x, gamma, eps), W)
 *   bi_gemm_rmsnorm_swiglu: out = bi_gemm_swiglu(bi_rmsnorm_f32in(x, ...), W)
 * with exactly those calls' bits. x fp32 [M, K] contiguous (the residual
 * stream), gamma [K] bf16, W [N, K] (swiglu: [2F, K]) bf16 with row stride
 * ldw; C [M, N] bf16 or fp32 (c_dtype BI_BF16 / BI_F32), out [M, F] bf16.
 * When every output tile has a CTA pair of its own (small M), the GEMM's
 * otherwise idle epilogue warps write r16((x r_i) gamma) into each A stage
 * (after a pass computing r_i by bi_rmsnorm_f32in's reduction); otherwise
 * the normed rows go through the workspace and the plain GEMM runs. ws:
 * caller-owned device memory of bi_gemm_rmsnorm_workspace_size(M, K) bytes,
 * 16-byte aligned. Constraints as bi_gemm, K (the normed width) <= 32768,
 * x and gamma 16-byte aligned. M == 0 or N == 0 is a no-op. Measured on
 * B200 the folded path is slower than the two calls (0.097 vs 0.031 ms for
 * the 7B QKV projection at M = 64): the GEMM's SMs then read the fp32 rows,
 * twice the bytes of the bf16 normed rows, next to the weights they stream;
 * bi_forward uses the two calls. */
bi_status bi_gemm_rmsnorm_workspace_size(int64_t M, int64_t K, size_t* bytes);
bi_status bi_gemm_rmsnorm(const float* x, const void* gamma, float eps,
                          const void* W, int64_t ldw, void* C, int64_t ldc,
                          int32_t c_dtype, int64_t M, int64_t N, int64_t K,
                          void* ws, size_t ws_bytes, void* stream);
bi_status bi_gemm_rmsnorm_swiglu(const float* x, const void* gamma, float eps,
                                 const void* W, int64_t ldw, void* out,
                                 int64_t ldo, int64_t M, int64_t F, int64_t K,
                                 void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Paged KV cache.  "Defeating Nondeterminism in LLM Inference", section
 * "Batch-invariant attention": the cache and page table are updated BEFORE
 * the attention kernel runs, so every key is read from the same layout
 * whether it was cached earlier or belongs to the chunk in flight.
 *
 * Layout (one page = BI_PAGE_SIZE tokens, d_h = BI_HEAD_DIM): each cache is
 * num_pages x num_kv_heads blocks of 16 x 128 bf16 (4 KB), block (page, g) at
 * element offset (page * num_kv_heads + g) * 2048. Inside a block the
 * elements sit in the tensor core's canonical K-major no-swizzle order (8 x 8
 * core matrices of 128 bytes), so attention copies a block as one piece:
 *   k_cache: key (slot o, dim d) at (o/8)*1024 + (d/8)*64 + (o%8)*8 + d%8
 *   v_cache: value (dim d, slot o) at (d/8)*128 + (o/8)*64 + (d%8)*8 + o%8
 * Token slot s = page * 16 + offset. */
typedef struct {
  int32_t num_pages;
  int32_t num_kv_heads;
  int32_t head_dim;  /* must be BI_HEAD_DIM */
  int32_t page_size; /* must be BI_PAGE_SIZE */
} bi_kv_layout;

/* Writes token t's key and value rows (k_new + t*ld_new, num_kv_heads * 128
 * bf16 each) into slot slot_mapping[t]. A negative slot skips the token
 * (padding). A slot >= num_pages*16 is skipped and sets BI_DEV_BAD_SLOT.
 * Pure data movement: the cache holds the exact input bytes. */
bi_status bi_kv_append(const void* k_new, const void* v_new, int64_t ld_new,
                       const int32_t* slot_mapping, int64_t n_tok,
                       void* k_cache, void* v_cache, const bi_kv_layout* kv,
                       void* stream);

/* ------------------------------------------------------------------------ */
/* Attention over the paged cache, causal, grouped-query (q head h reads kv
 * head h / (num_q_heads / num_kv_heads)).
 *
 * "Defeating Nondeterminism in LLM Inference", section "Batch-invariant
 * attention": the reduction order for a query must not depend on how many
 * tokens of its sequence are processed at once, nor on how many are already
 * cached; decoding needs a split reduction over the keys. The split used
 * here has a fixed SIZE (BI_ATTN_SPLIT keys at absolute key offsets), so a
 * query at position p always reduces over splits 0..p/512, each walked in
 * 128-key tiles at absolute offsets with an online softmax, and the splits
 * are merged in index order by a separate finishing pass (same section and
 * "When are atomic adds needed?": split reduction plus a serial finish).
 *
 * Per split s and row: S = (q . k_j) * scale in fp32 (tcgen05, bf16 inputs),
 * keys j > p masked, m' = max(m, rowmax), alpha = exp(m - m'),
 * P = bf16(exp(S - m')), l = alpha*l + sum(P) (fixed order), O = alpha*O + P.V.
 * Merge: M = max_s m_s, w_s = exp(m_s - M), out = bf16(sum_s w_s O_s / sum_s
 * w_s l_s), sums in split order. Decode and prefill run the same kernels, so
 * a token's output is bitwise equal in both.
 *
 * q rows: token t, head h at q + t*ldq + h*128 (bf16). out likewise with ldo.
 * block_table [B, max_pages_per_seq] int32 (page ids, in key order),
 * seq_lens [B] int32 = number of keys in the cache for sequence b, INCLUDING
 * the tokens queried in this call (they were appended first). A seq_lens
 * entry outside [queried tokens, max_kv_len] sets BI_DEV_BAD_SEQLEN and the
 * sequence's rows are written as zeros. */
typedef struct {
  int32_t num_q_heads;       /* Hq */
  int32_t num_kv_heads;      /* Hkv; Hq / Hkv must be 1, 2, 4 or 8 */
  int32_t head_dim;          /* must be BI_HEAD_DIM */
  int32_t page_size;         /* must be BI_PAGE_SIZE */
  int32_t num_pages;         /* pages in each cache (device range check) */
  int32_t max_pages_per_seq; /* row stride of block_table */
  int32_t max_kv_len;        /* upper bound of seq_lens (grid + workspace) */
  float scale;               /* softmax scale, e.g. 1/sqrt(128) */
} bi_attn_shape;

/* Workspace bytes for up to `max_tokens` query tokens with keys up to
 * shape->max_kv_len: per (token, q head, split) 128 fp32 partial outputs plus
 * (m, l), rounded up to 256 bytes, then 256 bytes holding the split kernel's
 * work-item counter (reset by the call itself, on its stream, before the
 * launch; it only decides which SM takes which (split, head group) item, never
 * the order of any sum). One workspace serves one call in flight at a time. */
bi_status bi_attn_workspace_size(const bi_attn_shape* shape, int64_t max_tokens,
                                 size_t* bytes);

/* Decode: one query per sequence; q/out row b belongs to sequence b and sits
 * at position seq_lens[b] - 1. */
bi_status bi_attn_decode(const void* q, int64_t ldq, const void* k_cache,
                         const void* v_cache, const int32_t* block_table,
                         const int32_t* seq_lens, int32_t B,
                         const bi_attn_shape* shape, void* out, int64_t ldo,
                         void* ws, size_t ws_bytes, void* stream);

/* Decode without a caller workspace. The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory -- for example
 * a host application whose own pool owns all device memory and forbids later
 * allocations, or a latency-critical loop that cannot afford cudaMalloc's
 * implicit device synchronisation. Same arguments and the same kernels (so
 * the same bits) as bi_attn_decode, minus ws/ws_bytes.
 *
 * The scratch is a fixed array of BI_ATTN_NOALLOC_SCRATCH_BYTES (16 MiB) that
 * is part of the library's device image: every GPU that loads libbi holds it
 * until the process exits. A call needs
 * B * num_q_heads * ceil(max_kv_len / 512) * 520 bytes of it, rounded up
 * to 256, plus 256 (e.g. 32 sequences x 32 heads x 8192 keys = 8.5 MiB);
 * larger calls fail with
 * BI_ERR_WORKSPACE and launch nothing. Nothing is allocated: no cudaMalloc,
 * no cudaFree, no allocating library routine.
 *
 * The first call on each device looks the array's device address up with
 * cudaGetSymbolAddress (with that device current) and caches it; make that
 * first call before any stream capture. Every call on a device shares the one
 * array and leaves its contents behind (nothing in it needs to start at
 * zero), so calls that overlap on the GPU -- on different streams, or from
 * several host threads -- race on it: order them on one stream. */
#define BI_ATTN_NOALLOC_SCRATCH_BYTES (16u << 20)
bi_status bi_attn_decode_noalloc(const void* q, int64_t ldq, const void* k_cache,
                                 const void* v_cache, const int32_t* block_table,
                                 const int32_t* seq_lens, int32_t B,
                                 const bi_attn_shape* shape, void* out, int64_t ldo,
                                 void* stream);

/* Prefill (chunked): sequence b owns query rows cu_q[b] .. cu_q[b+1]-1
 * (cu_q [B+1] int32 on the device, increasing, 0 <= cu_q[0], cu_q[B] <=
 * n_tok); they are its LAST n_b = cu_q[b+1]-cu_q[b] tokens, so row cu_q[b]+i
 * sits at position seq_lens[b] - n_b + i. max_q_len bounds n_b (host-side
 * grid size; a longer chunk sets BI_DEV_BAD_SEQLEN and its rows past the
 * covered ones are written as zeros). q and out span all n_tok rows; rows
 * outside cu_q[0] ..
 * cu_q[B]-1 are not read or written (so a call can cover a subset of a
 * batch, e.g. the multi-token chunks after the batch's one-token ones). */
bi_status bi_attn_prefill(const void* q, int64_t ldq, const int32_t* cu_q,
                          int32_t max_q_len, int64_t n_tok, const void* k_cache,
                          const void* v_cache, const int32_t* block_table,
                          const int32_t* seq_lens, int32_t B,
                          const bi_attn_shape* shape, void* out, int64_t ldo,
                          void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Pointwise steps of the decoder. "Defeating Nondeterminism in LLM
 * Inference", section "How do we make kernels batch-invariant?": pointwise
 * operations are batch-invariant as long as every element takes the same code
 * path; each kernel below has exactly one path per element. */

/* Embedding gather: out[t, :] = float(table[tokens[t], :]), table [V, D] bf16,
 * out [n_tok, D] fp32 (the residual stream). Bad ids write zeros and set
 * BI_DEV_BAD_TOKEN. D % 8 == 0. */
bi_status bi_embed(const int32_t* tokens, int64_t n_tok, const void* table,
                   int64_t vocab, int64_t D, float* out, void* stream);

/* Rotary embedding in place, rotate-half pairing (i, i + 64) of each 128-wide
 * head, angle = pos * theta^(-2i/128) evaluated in fp64 on the host into an
 * fp32 cos/sin table. x row t, head h at x + t*ldx + h*128 (bf16), positions
 * [n_tok] int32 on the device, < max_pos. Writes bf16(x_i c - x_{i+64} s) and
 * bf16(x_{i+64} c + x_i s) computed in fp32. cos_sin: [max_pos, 64, 2] fp32
 * caller-owned table filled by bi_rope_table. */
bi_status bi_rope_table(float* cos_sin, int32_t max_pos, double theta,
                        void* stream);
bi_status bi_rope(void* x, int64_t ldx, int32_t n_heads, const int32_t* positions,
                  int64_t n_tok, const float* cos_sin, int32_t max_pos,
                  void* stream);

/* SwiGLU: out[t, i] = bf16( silu(g) * u ), g = gu[t, i], u = gu[t, F + i],
 * silu(g) = g / (1 + exp(-g)) in fp32. gu [n_tok, 2F] bf16, out [n_tok, F]. */
bi_status bi_swiglu(const void* gu, int64_t n_tok, int64_t F, void* out,
                    void* stream);

/* Residual add: x[t, :] += float(d[t, :]) in fp32, d bf16 [n_tok, D]. */
bi_status bi_residual_add(float* x, const void* d, int64_t n_tok, int64_t D,
                          void* stream);

/* Greedy token: idx[r] = argmax_j logits[r, j] over fp32 logits [rows, V]
 * (row stride ld), lowest index on ties. Max is exact, so the result is
 * order-free. NaN rows return the first NaN's index. */
bi_status bi_argmax(const float* logits, int64_t rows, int64_t V, int64_t ld,
                    int32_t* idx, void* stream);

/* ------------------------------------------------------------------------ */
/* fp32-activation ("upcast") steps. The cross-vendor logit-mismatch paper
 * (arXiv 2610.05458, abstract) reports that upcasting to FP32 reduces logit
 * differences at ~3x runtime and that keeping only the MLP in BF16 keeps most
 * of the gain at ~1.3x. In these steps an fp32 activation that feeds a GEMM is
 * carried as a bf16 pair hi = bf16(x), lo = bf16(x - hi) (~16 significant
 * bits); everything else stays fp32. Same batch-invariance rules as above. */

/* C = (A_hi + A_lo) W^T: both terms meet the same bf16 W tile; per output
 * element, each 64-wide K stage adds its 4 hi K-steps then its 4 lo K-steps,
 * stages in K order. One fixed configuration for every shape (bi_gemm's
 * 256 x 256 CTA-pair tile). Same constraints as bi_gemm; A_hi and A_lo
 * share lda. */
bi_status bi_gemm_x2(const void* A_hi, const void* A_lo, int64_t lda,
                     const void* W, int64_t ldw, void* C, int64_t ldc,
                     int32_t c_dtype, int64_t M, int64_t N, int64_t K,
                     void* stream);

/* RMSNorm of fp32 rows (same fixed reduction order as bi_rmsnorm) written as
 * a bf16 pair: v = x r gamma in fp32, y_hi = bf16(v), y_lo = bf16(v - y_hi). */
bi_status bi_rmsnorm_split(const float* x, const void* gamma, void* y_hi,
                           void* y_lo, int64_t M, int64_t D, float eps,
                           void* stream);

/* hi[i] = bf16(x[i]), lo[i] = bf16(x[i] - hi[i]) for n fp32 values. */
bi_status bi_split_bf16x2(const float* x, int64_t n, void* hi, void* lo,
                          void* stream);

/* fp32 attention over an fp32 paged cache (k and v both
 * [num_pages, num_kv_heads, 16, 128] fp32). cu_q as in bi_attn_prefill, or
 * NULL for decode (n_tok == B, row b = sequence b). One warp per (query, q
 * head, 512-key split): s_j = (q . k_j) scale (lane partial sums over d,
 * then a shuffle-down tree), p_j = exp(s_j - max), l and O summed over keys
 * in order; splits merged in order as in bi_attn_prefill. q, out fp32. */
bi_status bi_attn_f32_workspace_size(const bi_attn_shape* shape,
                                     int64_t max_tokens, size_t* bytes);
bi_status bi_attn_f32(const float* q, int64_t ldq, const int32_t* cu_q,
                      int64_t n_tok, const float* k_cache, const float* v_cache,
                      const int32_t* block_table, const int32_t* seq_lens,
                      int32_t B, const bi_attn_shape* shape, float* out,
                      int64_t ldo, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Dense decoder forward (pre-norm, RMSNorm, RoPE, GQA attention, SwiGLU MLP),
 * composed only of the kernels above, with an fp32 residual stream and fp32
 * logits. precision selects the activation path:
 *   BI_PREC_BF16      bf16 activations, bf16 KV cache (bi_kv_layout)
 *   BI_PREC_F32       fp32 activations everywhere, fp32 KV cache
 *   BI_PREC_BF16_MLP  fp32 activations except the MLP block, fp32 KV cache
 *   BI_PREC_F16       the bf16 path with fp16 in place of bf16 everywhere:
 *                     fp16 weights (all arrays of bi_model_weights), fp16
 *                     activations and KV cache (bi_kv_layout), fp16 P in
 *                     attention; the FP16 variant of the cross-vendor
 *                     paper's precision study (arXiv 2610.05458, abstract) */
#define BI_PREC_BF16 0
#define BI_PREC_F32 1
#define BI_PREC_BF16_MLP 2
#define BI_PREC_F16 3
typedef struct {
  int32_t n_layers;
  int32_t d_model;     /* D */
  int32_t n_q_heads;   /* Hq, head_dim = BI_HEAD_DIM, Hq * 128 == D */
  int32_t n_kv_heads;  /* Hkv */
  int32_t d_ff;        /* F */
  int32_t vocab;       /* V */
  int32_t max_pos;     /* positions < max_pos */
  float rms_eps;
  double rope_theta;
  int32_t precision; /* BI_PREC_* */
} bi_model_config;

/* Caller-owned device weights, bf16 (fp16 for BI_PREC_F16), nn.Linear layout
 * [out, in]. Per layer l
 * the arrays hold n_layers consecutive blocks:
 *   attn_norm [L][D], w_qkv [L][(Hq + 2 Hkv) * 128][D] (rows: q heads, then k
 *   heads, then v heads), w_o [L][D][Hq * 128], mlp_norm [L][D],
 *   w_gate_up [L][2F][D] (gate rows, then up rows), w_down [L][D][F];
 *   embed [V][D], final_norm [D], lm_head [V][D]. */
typedef struct {
  const void* embed;
  const void* attn_norm;
  const void* w_qkv;
  const void* w_o;
  const void* mlp_norm;
  const void* w_gate_up;
  const void* w_down;
  const void* final_norm;
  const void* lm_head;
} bi_model_weights;

typedef struct bi_model bi_model;

/* One forward step over n_tok tokens of B sequences (any mix of prefill
 * chunks and decode tokens). All arrays are device int32:
 *   tokens [n_tok], positions [n_tok], slot_mapping [n_tok],
 *   cu_q [B+1] (rows of each sequence, contiguous and in order),
 *   seq_lens [B] (keys cached after this step), block_table [B][max_pages_per_seq],
 *   logits_rows [n_logits] (which token rows produce logits).
 * Host ints: max_q_len bounds cu_q[b+1]-cu_q[b]; max_kv_len bounds seq_lens;
 * n_decode (0 .. B): the first n_decode sequences each bring exactly one
 * token (rows 0 .. n_decode-1); their attention runs in the decode kernel and
 * the rest in the prefill kernel, which give the same bits for a row (0 sends
 * every row through one kernel: the decode kernel when every chunk is one
 * token, else the prefill kernel). A wrong n_decode gives wrong rows, never
 * an out-of-range access. */
typedef struct {
  const int32_t* tokens;
  const int32_t* positions;
  const int32_t* slot_mapping;
  const int32_t* cu_q;
  const int32_t* seq_lens;
  const int32_t* block_table;
  const int32_t* logits_rows;
  int64_t n_tok;
  int32_t B;
  int32_t max_q_len;
  int32_t max_kv_len;
  int32_t max_pages_per_seq;
  int64_t n_logits;
  int32_t n_decode;
} bi_batch;

bi_status bi_model_create(const bi_model_config* cfg, const bi_model_weights* w,
                          bi_model** out);
void bi_model_destroy(bi_model* m);

/* Workspace for a step of up to max_tokens tokens, max_logits logit rows and
 * keys up to max_kv_len. */
bi_status bi_forward_workspace_size(const bi_model* m, int64_t max_tokens,
                                    int64_t max_logits, int32_t max_kv_len,
                                    size_t* bytes);

/* k_cache / v_cache: num_layers consecutive caches, layer l at offset
 * l * num_pages * Hkv * 16 * 128 elements; bf16 in bi_kv_layout for
 * BI_PREC_BF16, fp16 in bi_kv_layout for BI_PREC_F16, fp32 [num_pages, Hkv,
 * 16, 128] (k and v alike) otherwise. logits
 * [n_logits, V] fp32; next_tokens [n_logits] int32 (nullable) = greedy argmax. */
bi_status bi_forward(const bi_model* m, const bi_batch* batch, void* k_cache,
                     void* v_cache, int32_t num_pages, float* logits,
                     int32_t* next_tokens, void* ws, size_t ws_bytes,
                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BI_H_ */
