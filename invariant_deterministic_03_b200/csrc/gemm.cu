// gemm.cu -- batch-invariant GEMM on the 5th-generation tensor cores.
//
// "Defeating Nondeterminism in LLM Inference", section "Batch-invariant
// matmul": tile the OUTPUT and keep each element's whole K reduction inside
// one core; never split K (split-K) nor hand different K ranges of a tile to
// different cores (stream-K); and compile ONE kernel configuration for every
// shape, because different tensor-core instructions may reduce in different
// internal orders.
//
// The one configuration (for every M, N, K):
//   output tile 128 x 256, K stage 64, instruction tcgen05.mma.cta_group::1
//   .kind::f16 M=128 N=256 K=16 with bf16 operands and an fp32 accumulator in
//   tensor memory. Element (m, n) is accumulated by the K-steps k = 0, 16, 32,
//   ... in that order, whatever M is. Which CTA computes a tile (persistent
//   round-robin), how many rows an A copy carries and what is prefetched into
//   L2 change timing only, never arithmetic.
//
// Fixed K split (a function of N and K only, never of M): when a weight has
// few output tiles (N / 256 <= 37), so that small batches would leave most
// SMs idle, and a long K (>= 8192, so that each half still keeps the tensor
// cores busy long enough to hide the hand-over below), K is cut once, at
// k-block ceil(k_blocks / 2). A cluster of two
// CTAs computes each tile: rank r accumulates its half of K in order in its
// own tensor memory; each rank finishes half of the tile's columns, taking
// the other rank's fp32 partial for them through distributed shared memory
// (32 columns at a time) and forming acc0 + acc1 (one fp32 addition per
// element; the sum of two values does not depend on their order). Same split, same order, for every M ("Defeating
// Nondeterminism in LLM Inference", section "Batch-invariant RMSNorm": one
// reduction strategy with enough parallelism for small batches, used at
// every batch size).
//
// CTA layout (192 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: A [128 x 64] and W [256 x 64] tiles, 128-byte
//               swizzle, into a 4-stage shared-memory ring (3 stages with two
//               A operands; mbarrier full/empty).
//               Small M (every CTA holds at most one tile, W streams through
//               fewer SMs than the GPU has): W tiles are also prefetched into
//               L2 W_PREFETCH stages ahead of the loads, and when M <= 128
//               the A copy carries only the M rows rounded up to 8 (the rest
//               of the 128-row A stage is never written: the MMA still runs
//               M=128, and rows past M, never stored, read whatever the stage
//               held; no row of the product depends on another row).
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators);
//               lane 0 issues the MMAs and tcgen05.commit's
//   warps 2..5  epilogue: tcgen05.ld the accumulator row by row (thread = row),
//               round to bf16 (RNE) or keep fp32, store to global, or run one
//               of the fused epilogues (EPI_ADD, EPI_SWIGLU, EPI_QKV below)
//               on the finished values; then free the accumulator for the
//               tile after next.
// Every mbarrier wait is bounded (see common.cuh); a timeout sets a status
// bit and the CTA winds down, releasing its tensor memory.
#include <mutex>

#include "common.cuh"
#include "host.h"

namespace bi {
namespace gemm {

constexpr int BM = BI_GEMM_BM;  // 128
constexpr int BN = BI_GEMM_BN;  // 256
constexpr int BK = BI_GEMM_BK;  // 64 bf16 = 128 bytes = one swizzle row
constexpr int UMMA_K = 16;
constexpr uint32_t A_BYTES = BM * BK * 2;  // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;  // 32 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr int THREADS = 192;
constexpr int W_PREFETCH = 8;  // W stages prefetched into L2 ahead of the loads (small M)
constexpr int SPLIT_MAX_TILES_N = 37;       // weights with at most this many column tiles
constexpr int SPLIT_MIN_K = 8192;           // and at least this K split K in two
constexpr uint32_t XFER_SLOT = 128 * 32 * 4;  // one 32-column chunk of a 128-row fp32 accumulator

// TERMS = number of bf16 A operands summed into the product: 1 for plain
// bf16 activations, 2 for an activation carried as a hi/lo pair (A = A_hi +
// A_lo, ~16 significant bits). Both terms meet the same W tile in shared
// memory, so W is read once.
template <int TERMS>
struct Cfg {
  static constexpr int STAGES = TERMS == 1 ? 4 : 3;
  static constexpr uint32_t STAGE_BYTES = TERMS * A_BYTES + B_BYTES;
  static constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + 2 * XFER_SLOT + 256;
  static_assert(SMEM_BYTES <= 232448, "gemm: shared memory above the per-CTA limit");
};

struct Params {
  void* C;
  int64_t ldc;
  int32_t c_f32;
  int32_t M, N, K;
  int32_t m_blocks, n_blocks, k_blocks;
  int32_t w_prefetch;  // W_PREFETCH or 0 (off)
  int32_t split;       // CTAs (cluster ranks) per tile: 1, or 2 with K cut in two
  int32_t kb_per_rank; // k-blocks of rank 0 (rank 1 takes the rest)
  uint32_t a_bytes;    // bytes of one A copy: 128 rows, or M rounded up to 8 when M < 128
  int32_t* status;
  // EPI_QKV only: RoPE of the q and k heads and the paged-cache write
  const int32_t* pos;    // [M] absolute positions
  const float* cs;       // [max_pos, 64, 2] cos / sin
  const int32_t* slots;  // [M] cache slots (page * 16 + offset), < 0: padding row
  bf16* kc;              // key cache, 4 KB per (page, kv head)
  bf16* vc;              // value cache, same blocking, transposed per page
  int32_t max_pos, num_pages, hq, hkv;
};

__device__ __forceinline__ void store_row_chunk(const Params& p, int row, int col0,
                                                const uint32_t (&r)[32]) {
  // 32 consecutive columns col0 .. col0+31 of one row; N % 8 == 0, so each
  // group of 8 columns is either fully inside or fully outside.
  if (p.c_f32) {
    float* dst = static_cast<float*>(p.C) + (size_t)row * p.ldc + col0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (col0 + g * 8 < p.N) {
        float4 a = make_float4(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]),
                               __uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
        float4 b = make_float4(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]),
                               __uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
        *reinterpret_cast<float4*>(dst + 8 * g) = a;
        *reinterpret_cast<float4*>(dst + 8 * g + 4) = b;
      }
    }
  } else {
    bf16* dst = static_cast<bf16*>(p.C) + (size_t)row * p.ldc + col0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (col0 + g * 8 < p.N) {
        uint4 o;
        o.x = pack_bf16x2(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]));
        o.y = pack_bf16x2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
        o.z = pack_bf16x2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]));
        o.w = pack_bf16x2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
        *reinterpret_cast<uint4*>(dst + 8 * g) = o;
      }
    }
  }
}

// C[row, col0 .. col0+31] (fp32) += the accumulator chunk, one fp32
// addition per element.
__device__ __forceinline__ void add_row_chunk(const Params& p, int row, int col0, const uint32_t (&r)[32]) {
  float* dst = static_cast<float*>(p.C) + (size_t)row * p.ldc + col0;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    if (col0 + g * 8 < p.N) {
      float4 a = *reinterpret_cast<const float4*>(dst + 8 * g);
      float4 b = *reinterpret_cast<const float4*>(dst + 8 * g + 4);
      a.x = __fadd_rn(a.x, __uint_as_float(r[8 * g + 0]));
      a.y = __fadd_rn(a.y, __uint_as_float(r[8 * g + 1]));
      a.z = __fadd_rn(a.z, __uint_as_float(r[8 * g + 2]));
      a.w = __fadd_rn(a.w, __uint_as_float(r[8 * g + 3]));
      b.x = __fadd_rn(b.x, __uint_as_float(r[8 * g + 4]));
      b.y = __fadd_rn(b.y, __uint_as_float(r[8 * g + 5]));
      b.z = __fadd_rn(b.z, __uint_as_float(r[8 * g + 6]));
      b.w = __fadd_rn(b.w, __uint_as_float(r[8 * g + 7]));
      *reinterpret_cast<float4*>(dst + 8 * g) = a;
      *reinterpret_cast<float4*>(dst + 8 * g + 4) = b;
    }
  }
}

__device__ __forceinline__ float round_bf16(uint32_t acc) {
  return __bfloat162float(__float2bfloat16_rn(__uint_as_float(acc)));
}

// out[row, f0 .. f0+31] = bf16(swiglu(bf16(gate), bf16(up))); F % 8 == 0.
__device__ __forceinline__ void store_swiglu_chunk(const Params& p, int row, int f0, const uint32_t (&g)[32],
                                                   const uint32_t (&u)[32]) {
  bf16* dst = static_cast<bf16*>(p.C) + (size_t)row * p.ldc + f0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (f0 + q * 8 < p.N) {
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = swiglu_f32(round_bf16(g[8 * q + k]), round_bf16(u[8 * q + k]));
      uint4 o;
      o.x = pack_bf16x2(v[0], v[1]);
      o.y = pack_bf16x2(v[2], v[3]);
      o.z = pack_bf16x2(v[4], v[5]);
      o.w = pack_bf16x2(v[6], v[7]);
      *reinterpret_cast<uint4*>(dst + 8 * q) = o;
    }
  }
}

// Epilogue of a tile (EPI):
//   EPI_STORE   C = acc, rounded to bf16 (RNE) or kept fp32;
//   EPI_ADD     C (fp32) = C + acc: one fp32 addition per element after the
//               whole K reduction (a residual connection in the stream);
//   EPI_SWIGLU  the tile's 256 accumulator columns are 128 gate features
//               (W rows f) and the same 128 up features (W rows F + f):
//               C[m, f] = bf16(swiglu_f32(bf16(g), bf16(u))), the same
//               rounding points as a bf16 GEMM followed by bi_swiglu.
constexpr int EPI_STORE = 0, EPI_ADD = 1, EPI_SWIGLU = 2, EPI_QKV = 3;

// EPI_QKV: the fused [q | k | v] projection (heads of 128 columns, so a
// 256-column tile is heads 2 nb and 2 nb + 1). Every element is first
// rounded to bf16 as EPI_STORE does. q and k heads then rotate each pair
// (i, i + 64) with the RoPE kernel's arithmetic (rope_rotate on the bf16
// values and the fp32 table) and are stored rounded again; k and v heads are
// also written to the paged caches at the row's slot, in the KV append's
// layout:
//   keys:   element (slot o, d) at (o/8)*1024 + (d/8)*64 + (o%8)*8 + d%8
//   values: element (d, slot o) at (d/8)*128 + (o/8)*64 + (d%8)*8 + o%8
// of the (page, kv head) block. The qkv rows and both caches end up with the
// same bits as bi_gemm, then bi_rope over the q and k heads, then
// bi_kv_append. The tensor-memory loads are warp-collective, so every lane
// runs them; only rows < M store.
__device__ __forceinline__ void qkv_tile(const Params& p, int row, int nb, uint32_t taddr) {
  const bool live = row < p.M;
  int pos = 0, slot = -1;
  if (live) {
    pos = p.pos[row];
    slot = p.slots[row];
  }
  const bool rot = pos >= 0 && pos < p.max_pos;
  const bool slot_bad = slot >= p.num_pages * BI_PAGE_SIZE;
  const bool to_cache = live && slot >= 0 && !slot_bad;
  const int sl = to_cache ? slot : 0;
  const int page = sl / BI_PAGE_SIZE, o = sl % BI_PAGE_SIZE;
  if (live && !rot && nb * 2 < p.hq + p.hkv) set_status(p.status, BI_DEV_BAD_TOKEN);
  const int n_heads = p.hq + 2 * p.hkv;
  bf16* crow = static_cast<bf16*>(p.C) + (size_t)(live ? row : 0) * p.ldc;
  // q / k heads of this tile rotate with the row's cos / sin: loaded once per
  // 32-pair block for both heads, before the accumulator reads
  const int n_rot = max(0, min(2, p.hq + p.hkv - nb * 2));  // leading heads of the tile that rotate
  const float* csrow = p.cs + (size_t)(rot ? pos : 0) * 128;
#pragma unroll 1
  for (int j = 0; j < 2 && n_rot > 0; ++j) {
    float4 t[16];  // cos / sin of pairs 32 j .. 32 j + 31
#pragma unroll
    for (int q = 0; q < 16; ++q)
      t[q] = (live && rot) ? reinterpret_cast<const float4*>(csrow + j * 64)[q] : make_float4(1.f, 0.f, 1.f, 0.f);
#pragma unroll 1
    for (int hh = 0; hh < n_rot; ++hh) {
      const int H = nb * 2 + hh;
      const bool is_k = H >= p.hq;
      bf16* out = crow + (size_t)H * BI_HEAD_DIM;
      if (j == 0 && is_k && live && slot_bad) set_status(p.status, BI_DEV_BAD_SLOT);
      bf16* kdst = p.kc + ((size_t)page * p.hkv + (is_k ? H - p.hq : 0)) * (BI_PAGE_SIZE * BI_HEAD_DIM) +
                   (o >> 3) * 1024 + (o & 7) * 8;
      uint32_t ra[32], rb[32];  // columns 32 j .. 32 j + 31 and their partners 64 further on
      tmem_ld32(taddr + (hh * 4 + j) * 32, ra);
      tmem_ld32(taddr + (hh * 4 + j + 2) * 32, rb);
      tmem_ld_wait();
      if (!live) continue;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float ya[8], yb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float4 c = t[g * 4 + (e >> 1)];
          const float a = round_bf16(ra[8 * g + e]), b = round_bf16(rb[8 * g + e]);
          if (rot) rope_rotate(a, b, (e & 1) ? c.z : c.x, (e & 1) ? c.w : c.y, ya[e], yb[e]);
          else { ya[e] = a; yb[e] = b; }
        }
        const uint4 A = make_uint4(pack_bf16x2(ya[0], ya[1]), pack_bf16x2(ya[2], ya[3]),
                                   pack_bf16x2(ya[4], ya[5]), pack_bf16x2(ya[6], ya[7]));
        const uint4 B = make_uint4(pack_bf16x2(yb[0], yb[1]), pack_bf16x2(yb[2], yb[3]),
                                   pack_bf16x2(yb[4], yb[5]), pack_bf16x2(yb[6], yb[7]));
        const int d0 = j * 32 + g * 8;
        *reinterpret_cast<uint4*>(out + d0) = A;
        *reinterpret_cast<uint4*>(out + 64 + d0) = B;
        if (is_k && to_cache) {
          *reinterpret_cast<uint4*>(kdst + (d0 >> 3) * 64) = A;
          *reinterpret_cast<uint4*>(kdst + ((d0 + 64) >> 3) * 64) = B;
        }
      }
    }
  }
  // v heads of this tile: stored and written to the value cache
#pragma unroll 1
  for (int hh = n_rot; hh < 2; ++hh) {
    const int H = nb * 2 + hh;
    if (H >= n_heads) break;  // uniform across the warp
    bf16* out = crow + (size_t)H * BI_HEAD_DIM;
    if (live && slot_bad) set_status(p.status, BI_DEV_BAD_SLOT);
    {
      bf16* vdst = p.vc + ((size_t)page * p.hkv + (H - p.hq - p.hkv)) * (BI_PAGE_SIZE * BI_HEAD_DIM) +
                   (o >> 3) * 64 + (o & 7);
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        uint32_t r[32];
        tmem_ld32(taddr + (hh * 4 + j) * 32, r);
        tmem_ld_wait();
        if (!live) continue;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint4 V = make_uint4(pack_bf16x2(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1])),
                                     pack_bf16x2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3])),
                                     pack_bf16x2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5])),
                                     pack_bf16x2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7])));
          const int d0 = j * 32 + g * 8;
          *reinterpret_cast<uint4*>(out + d0) = V;
          if (to_cache) {
            const bf16* v8 = reinterpret_cast<const bf16*>(&V);
#pragma unroll
            for (int e = 0; e < 8; ++e) vdst[((d0 + e) >> 3) * 128 + ((d0 + e) & 7) * 8] = v8[e];
          }
        }
      }
    }
  }
}

template <int TERMS, int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmA2,
                        const __grid_constant__ CUtensorMap tmB, const Params p) {
  constexpr int STAGES = Cfg<TERMS>::STAGES;
  constexpr uint32_t STAGE_BYTES = Cfg<TERMS>::STAGE_BYTES;
  const uint32_t tx_bytes = TERMS * p.a_bytes + B_BYTES;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzled tiles want 1024-byte aligned bases.
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* xfer = smem + STAGES * STAGE_BYTES;  // [2 slots] partial-accumulator chunks from the peer
  uint64_t* full = reinterpret_cast<uint64_t*>(xfer + 2 * XFER_SLOT);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* xfer_full = acc_empty + 2;   // [2] the peer's chunk is in my slot
  uint64_t* xfer_free = xfer_full + 2;   // [2] the peer has read my chunk from its slot
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(xfer_free + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = p.m_blocks * p.n_blocks;
  const int CL = p.split;
  const uint32_t rank = CL > 1 ? cluster_rank() : 0u;
  const int tile0 = (int)blockIdx.x / CL, tile_step = (int)gridDim.x / CL;
  const int kb_lo = (int)rank * p.kb_per_rank;
  const int kb_hi = min(p.k_blocks, kb_lo + p.kb_per_rank);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);    // one arrive per epilogue warp
      mbar_init(&xfer_full[a], 4);  // lane 0 of each epilogue warp of the peer
      mbar_init(&xfer_free[a], 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    if (TERMS == 2) prefetch_tmap(&tmA2);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (CL > 1) cluster_sync();  // both ranks' barriers initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int fills[STAGES];
      for (int s = 0; s < STAGES; ++s) fills[s] = 0;
      for (int tile = tile0; tile < num_tiles && ok; tile += tile_step) {
        const int mb = tile % p.m_blocks, nb = tile / p.m_blocks;
        const int pf = p.w_prefetch;
        // W rows of this tile: 256 from nb * 256, or (SwiGLU) 128 gate rows
        // from nb * 128 and the matching 128 up rows from F + nb * 128
        const int w_row0 = EPI == EPI_SWIGLU ? nb * (BN / 2) : nb * BN;
        const int w_row1 = p.N + nb * (BN / 2);
        for (int kb = kb_lo; kb < kb_lo + pf && kb < kb_hi; ++kb) {
          tma_prefetch_2d(&tmB, kb * BK, w_row0);
          if (EPI == EPI_SWIGLU) tma_prefetch_2d(&tmB, kb * BK, w_row1);
        }
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, p.status, abort_flag)) { ok = false; break; }
          if (pf && kb + pf < kb_hi) {
            tma_prefetch_2d(&tmB, (kb + pf) * BK, w_row0);
            if (EPI == EPI_SWIGLU) tma_prefetch_2d(&tmB, (kb + pf) * BK, w_row1);
          }
          uint8_t* sa = tiles + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], tx_bytes);
          tma_load_2d(sa, &tmA, &full[stage], kb * BK, mb * BM);
          if (TERMS == 2) tma_load_2d(sa + A_BYTES, &tmA2, &full[stage], kb * BK, mb * BM);
          tma_load_2d(sa + TERMS * A_BYTES, &tmB, &full[stage], kb * BK, w_row0);
          if (EPI == EPI_SWIGLU)
            tma_load_2d(sa + TERMS * A_BYTES + B_BYTES / 2, &tmB, &full[stage], kb * BK, w_row1);
          ++fills[stage];
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // Let copies already in flight land before the CTA can exit: wait
        // (bounded) for every stage's last fill.
        for (int s = 0; s < STAGES; ++s) {
          if (fills[s] == 0) continue;
          const uint32_t par = (uint32_t)(fills[s] - 1) & 1u;
          const long long t0 = clock64();
          while (!mbar_try_wait(&full[s], par) && clock64() - t0 < kWaitLimitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = tile0; tile < num_tiles && ok; tile += tile_step) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, p.status, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.status, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(tiles + stage * STAGE_BYTES);
          const uint32_t sb = sa + TERMS * A_BYTES;
#pragma unroll
          for (int term = 0; term < TERMS; ++term) {
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              // Advancing the start address by 32 bytes per 16-element K step
              // inside the 128-byte swizzle atom; the hardware applies the
              // swizzle on the absolute address (tile bases are 1024-aligned).
              uint64_t ad = smem_desc(sa + term * A_BYTES + k * 32, 16, 1024, 2);
              uint64_t bd = smem_desc(sb + k * 32, 16, 1024, 2);
              mma_bf16(d_tmem, ad, bd, idesc, (kb != kb_lo || term != 0 || k != 0));
            }
          }
          mma_commit(&empty[stage]);  // frees the stage once these MMAs retire
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);   // accumulator complete
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // ---------------- epilogue warps 2..5: TMEM lanes 32*(warp%4) .. +31
    const int quarter = warp & 3;
    const int trow = quarter * 32 + lane;  // accumulator row (TMEM lane) of this thread
    int acc = 0;
    uint32_t acc_phase = 0;
    int nx_out = 0, nx_in = 0;  // chunks sent to / received from the peer rank (slot n & 1)
    bool ok = true;
    for (int tile = tile0; tile < num_tiles && ok; tile += tile_step) {
      const int mb = tile % p.m_blocks, nb = tile / p.m_blocks;
      if (!mbar_wait(&acc_full[acc], acc_phase, p.status, abort_flag)) break;
      tc_fence_after();
      const int row = mb * BM + trow;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      uint32_t held[32];  // SwiGLU: a gate chunk until its up chunk arrives
      auto col_of = [&](int c) {
        return EPI == EPI_SWIGLU ? nb * (BN / 2) + (c & 3) * 32 : nb * BN + c * 32;
      };
      // the epilogue of one finished 32-column chunk c (values in r)
      auto finish = [&](int c, uint32_t (&r)[32]) {
        if (row >= p.M) return;
        if constexpr (EPI == EPI_SWIGLU) {
          if (c >= 4) {
            store_swiglu_chunk(p, row, col_of(c), held, r);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) held[i] = r[i];
          }
        } else if constexpr (EPI == EPI_ADD) {
          add_row_chunk(p, row, col_of(c), r);
        } else {
          store_row_chunk(p, row, col_of(c), r);
        }
      };
      if constexpr (EPI == EPI_QKV) {
        qkv_tile(p, row, nb, taddr);  // never split (the host only fuses unsplit weights)
      } else if (CL == 1) {
#pragma unroll 1
        for (int q = 0; q < BN / 32; ++q) {
          // SwiGLU pairs gate chunk c with up chunk c + 4
          const int c = EPI == EPI_SWIGLU ? ((q & 1) ? 4 + (q >> 1) : (q >> 1)) : q;
          if (col_of(c) >= p.N) break;  // uniform across the warp
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          finish(c, r);
        }
      } else {
        // K split across the two ranks: rank r finishes half of the chunks
        // (acc0 + acc1, one fp32 addition) and sends the other half to its
        // partner. Chunks owned by rank r, in order: 0-3 / 4-7, or for SwiGLU
        // gate/up pairs 0,4,1,5 / 2,6,3,7. Sends and receives alternate
        // S S R S R S R R so that each direction keeps two chunks in flight
        // in the partner's two slots and neither rank can block the other.
        auto owned = [&](uint32_t rk, int i) {
          return EPI == EPI_SWIGLU ? (int)rk * 2 + (i >> 1) + (i & 1) * 4 : (int)rk * 4 + i;
        };
        int own[4], oth[4], n_own = 0, n_oth = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int co = owned(rank, i), ct = owned(rank ^ 1u, i);
          if (col_of(co) < p.N) own[n_own++] = co;  // live chunks: the same test on both ranks
          if (col_of(ct) < p.N) oth[n_oth++] = ct;
        }
        const uint32_t peer = rank ^ 1u;
        int is = 0, ir = 0;
#pragma unroll 1
        for (int step = 0; step < 8 && ok; ++step) {
          const bool pref_send = step == 0 || step == 1 || step == 3 || step == 5;
          const bool send = pref_send ? is < n_oth : !(ir < n_own);
          if (send ? is >= n_oth : ir >= n_own) continue;
          const int c = send ? oth[is++] : own[ir++];
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          // One lane per warp waits (acquire) and arrives (release) at
          // cluster scope; __syncwarp orders the other lanes' accesses
          // around it (release and acquire are cumulative), so each hand-over
          // costs one cluster fence per warp, not one per thread.
          if (send) {
            const int slot = nx_out & 1;  // a slot of the peer's staging area
            int w_ok = 1;
            if (lane == 0)
              w_ok = mbar_wait_cluster(&xfer_free[slot], (((uint32_t)nx_out >> 1) & 1u) ^ 1u, p.status,
                                       abort_flag);
            if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
              ok = false;
              break;
            }
            if (row < p.M) {
              const uint32_t dst = cluster_addr(xfer + slot * XFER_SLOT + trow * 128, peer);
#pragma unroll
              for (int j = 0; j < 8; ++j)  // 16-byte units swizzled by row: no bank conflicts
                st_cluster_v4(dst + ((uint32_t)(j ^ (trow & 7)) << 4), r[4 * j], r[4 * j + 1],
                              r[4 * j + 2], r[4 * j + 3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(cluster_addr(&xfer_full[slot], peer));
            ++nx_out;
          } else {
            const int slot = nx_in & 1;
            int w_ok = 1;
            if (lane == 0)
              w_ok = mbar_wait_cluster(&xfer_full[slot], ((uint32_t)nx_in >> 1) & 1u, p.status, abort_flag);
            if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
              ok = false;
              break;
            }
            if (row < p.M) {
              const uint8_t* src = xfer + slot * XFER_SLOT + trow * 128;
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const uint4 v = *reinterpret_cast<const uint4*>(src + ((j ^ (trow & 7)) << 4));
                r[4 * j] = __float_as_uint(__fadd_rn(__uint_as_float(r[4 * j]), __uint_as_float(v.x)));
                r[4 * j + 1] = __float_as_uint(__fadd_rn(__uint_as_float(r[4 * j + 1]), __uint_as_float(v.y)));
                r[4 * j + 2] = __float_as_uint(__fadd_rn(__uint_as_float(r[4 * j + 2]), __uint_as_float(v.z)));
                r[4 * j + 3] = __float_as_uint(__fadd_rn(__uint_as_float(r[4 * j + 3]), __uint_as_float(v.w)));
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(cluster_addr(&xfer_free[slot], peer));
            ++nx_in;
            finish(c, r);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  // no rank leaves while the other may still write into, or arrive on, its
  // shared memory
  if (CL > 1) cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

__global__ void zero_fill_kernel(void* C, int64_t ldc, int32_t c_f32, int32_t M, int32_t N) {
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t total = (int64_t)M * N;
  for (; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    int64_t m = i / N, n = i % N;
    if (c_f32) static_cast<float*>(C)[m * ldc + n] = 0.0f;
    else static_cast<bf16*>(C)[m * ldc + n] = __float2bfloat16_rn(0.0f);
  }
}

}  // namespace gemm
}  // namespace bi

using namespace bi;

namespace bi {
namespace gemm {

static bi_status check_args(const void* A, int64_t lda, const void* W, int64_t ldw, const void* C,
                            int64_t ldc, int32_t c_dtype, int64_t M, int64_t N, int64_t K) {
  if (!A || !W || !C) return fail(BI_ERR_INVALID_ARG, "gemm: null pointer");
  if (M < 0 || N < 0 || K < 0) return fail(BI_ERR_INVALID_ARG, "gemm: negative size");
  if (c_dtype != BI_BF16 && c_dtype != BI_F32 && c_dtype != BI_F32_ADD)
    return fail(BI_ERR_INVALID_ARG, "gemm: bad c_dtype %d", c_dtype);
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30)) return fail(BI_ERR_SHAPE, "gemm: size above 2^30");
  if (K % 8 || N % 8) return fail(BI_ERR_SHAPE, "gemm: K (%lld) and N (%lld) must be multiples of 8", (long long)K, (long long)N);
  if (lda < K || ldw < K || ldc < N) return fail(BI_ERR_SHAPE, "gemm: leading dimension smaller than the row");
  if (lda % 8 || ldw % 8 || ldc % 8) return fail(BI_ERR_ALIGN, "gemm: leading dimensions must be multiples of 8");
  if (!aligned16(A) || !aligned16(W) || !aligned16(C)) return fail(BI_ERR_ALIGN, "gemm: pointers must be 16-byte aligned");
  return BI_OK;
}

template <int TERMS, int EPI>
static bi_status set_smem_attr() {
  static bool done[64] = {false};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!done[dev & 63]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tcgen05_kernel<TERMS, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<TERMS>::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e, "gemm: smem attribute");
    done[dev & 63] = true;
  }
  return BI_OK;
}

// How many two-CTA clusters of this kernel the device runs at once (queried
// once per device).
template <int TERMS, int EPI>
static bi_status pair_clusters(int* out) {
  static int cache[64] = {0};
  static std::mutex mu;
  bi_status st = set_smem_attr<TERMS, EPI>();
  if (st != BI_OK) return st;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  int& v = cache[dev & 63];
  if (v == 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = Cfg<TERMS>::SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveClusters(&n, gemm_tcgen05_kernel<TERMS, EPI>, &cfg);
    if (e != cudaSuccess) return cuda_fail(e, "gemm: cluster occupancy");
    if (n <= 0) return fail(BI_ERR_UNSUPPORTED, "gemm: no two-CTA cluster fits on this device");
    v = n;
  }
  *out = v;
  return BI_OK;
}

struct QkvArgs {
  const int32_t* pos;
  const float* cs;
  const int32_t* slots;
  bf16* kc;
  bf16* vc;
  int32_t max_pos, num_pages, hq, hkv;
};

// The fixed K split of a weight: a function of its shape (N, K) only.
static int split_of(int64_t N, int64_t K, bool swiglu) {
  const int64_t cols = swiglu ? BN / 2 : BN;
  return ((N + cols - 1) / cols <= SPLIT_MAX_TILES_N && K >= SPLIT_MIN_K) ? 2 : 1;
}

// N is the output width: the W rows for EPI_STORE / EPI_ADD / EPI_QKV, the
// feature count F (W has 2F rows) for EPI_SWIGLU.
template <int TERMS, int EPI>
static bi_status launch(const void* A, const void* A2, int64_t lda, const void* W, int64_t ldw,
                        void* C, int64_t ldc, int32_t c_dtype, int64_t M, int64_t N, int64_t K,
                        cudaStream_t s, const QkvArgs* qa = nullptr) {
  bi_status st;
  const int32_t c_f32 = c_dtype != BI_BF16;
  if (K == 0) {
    if (EPI == EPI_ADD) return BI_OK;  // C += 0
    zero_fill_kernel<<<296, 256, 0, s>>>(C, ldc, c_f32, (int32_t)M, (int32_t)N);
    BI_CHECK_LAUNCH("gemm zero fill");
    return BI_OK;
  }
  CUtensorMap tmA, tmA2, tmB;
  {
    uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
    uint64_t strides[1] = {(uint64_t)lda * 2};
    const uint32_t a_rows = M < BM ? (uint32_t)((M + 7) / 8 * 8) : (uint32_t)BM;
    uint32_t box[2] = {BK, a_rows};
    if ((st = encode_tmap(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(A), dims,
                          strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != BI_OK)
      return st;
    if (TERMS == 2) {
      if ((st = encode_tmap(&tmA2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(A2), dims,
                            strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != BI_OK)
        return st;
    } else {
      tmA2 = tmA;
    }
  }
  {
    uint64_t dims[2] = {(uint64_t)K, (uint64_t)(EPI == EPI_SWIGLU ? 2 * N : N)};
    uint64_t strides[1] = {(uint64_t)ldw * 2};
    uint32_t box[2] = {BK, EPI == EPI_SWIGLU ? BN / 2 : BN};
    if ((st = encode_tmap(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), dims,
                          strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != BI_OK)
      return st;
  }
  Params p;
  p.C = C;
  p.ldc = ldc;
  p.c_f32 = c_f32;
  p.M = (int32_t)M;
  p.N = (int32_t)N;
  p.K = (int32_t)K;
  p.m_blocks = (int32_t)((M + BM - 1) / BM);
  const int64_t cols_per_tile = EPI == EPI_SWIGLU ? BN / 2 : BN;
  p.n_blocks = (int32_t)((N + cols_per_tile - 1) / cols_per_tile);
  p.k_blocks = (int32_t)((K + BK - 1) / BK);
  p.status = status_word();
  p.pos = qa ? qa->pos : nullptr;
  p.cs = qa ? qa->cs : nullptr;
  p.slots = qa ? qa->slots : nullptr;
  p.kc = qa ? qa->kc : nullptr;
  p.vc = qa ? qa->vc : nullptr;
  p.max_pos = qa ? qa->max_pos : 0;
  p.num_pages = qa ? qa->num_pages : 0;
  p.hq = qa ? qa->hq : 0;
  p.hkv = qa ? qa->hkv : 0;
  if ((st = set_smem_attr<TERMS, EPI>()) != BI_OK) return st;
  // the K split depends on the weight's shape only, never on M
  p.split = split_of(N, K, EPI == EPI_SWIGLU);
  if (EPI == EPI_QKV && p.split != 1) return fail(BI_ERR_UNSUPPORTED, "gemm_qkv: split weight");
  p.kb_per_rank = (p.k_blocks + p.split - 1) / p.split;
  const int64_t tiles = (int64_t)p.m_blocks * p.n_blocks;
  const int sms = num_sms();
  p.w_prefetch = tiles * p.split <= sms ? W_PREFETCH : 0;
  p.a_bytes = (uint32_t)(M < BM ? (M + 7) / 8 * 8 : BM) * BK * 2;
  if (p.split == 1) {
    const int grid = (int)(tiles < sms ? tiles : sms);
    gemm_tcgen05_kernel<TERMS, EPI><<<grid, THREADS, Cfg<TERMS>::SMEM_BYTES, s>>>(tmA, tmA2, tmB, p);
  } else {
    int fit = 0;
    if ((st = pair_clusters<TERMS, EPI>(&fit)) != BI_OK) return st;
    const int64_t clusters = tiles < fit ? tiles : fit;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = Cfg<TERMS>::SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_tcgen05_kernel<TERMS, EPI>, tmA, tmA2, tmB, p);
    if (e != cudaSuccess) return cuda_fail(e, "gemm: cluster launch");
  }
  BI_CHECK_LAUNCH("gemm launch");
  return BI_OK;
}

}  // namespace gemm
}  // namespace bi

extern "C" bi_status bi_gemm(const void* A, int64_t lda, const void* W, int64_t ldw, void* C,
                             int64_t ldc, int32_t c_dtype, int64_t M, int64_t N, int64_t K,
                             void* stream) {
  bi_status st = gemm::check_args(A, lda, W, ldw, C, ldc, c_dtype, M, N, K);
  if (st != BI_OK || M == 0 || N == 0) return st;
  if ((st = require_sm100()) != BI_OK) return st;
  if (c_dtype == BI_F32_ADD)
    return gemm::launch<1, gemm::EPI_ADD>(A, nullptr, lda, W, ldw, C, ldc, c_dtype, M, N, K,
                                          static_cast<cudaStream_t>(stream));
  return gemm::launch<1, gemm::EPI_STORE>(A, nullptr, lda, W, ldw, C, ldc, c_dtype, M, N, K,
                                          static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_gemm_swiglu(const void* A, int64_t lda, const void* W, int64_t ldw, void* out,
                                    int64_t ldo, int64_t M, int64_t F, int64_t K, void* stream) {
  bi_status st = gemm::check_args(A, lda, W, ldw, out, ldo, BI_BF16, M, F, K);
  if (st != BI_OK || M == 0 || F == 0) return st;
  if (F > (1ll << 29)) return fail(BI_ERR_SHAPE, "gemm_swiglu: F above 2^29");
  if ((st = require_sm100()) != BI_OK) return st;
  return gemm::launch<1, gemm::EPI_SWIGLU>(A, nullptr, lda, W, ldw, out, ldo, BI_BF16, M, F, K,
                                           static_cast<cudaStream_t>(stream));
}

namespace bi {
bi_status launch_kv_append(const bf16* k, const bf16* v, int64_t ld_new, const int32_t* slots,
                           int64_t n_tok, bf16* kc, bf16* vc, int Hkv, int num_pages,
                           cudaStream_t s);
bi_status launch_rope(bf16* x, int64_t ldx, int n_heads, const int32_t* pos, int64_t n_tok,
                      const float* cs, int max_pos, cudaStream_t s);
}  // namespace bi

extern "C" bi_status bi_gemm_qkv(const void* A, int64_t lda, const void* W, int64_t ldw, void* qkv,
                                 int64_t ldq, int64_t M, int64_t K, int32_t n_q_heads,
                                 int32_t n_kv_heads, const int32_t* positions, const float* cos_sin,
                                 int32_t max_pos, const int32_t* slot_mapping, void* k_cache,
                                 void* v_cache, int32_t num_pages, void* stream) {
  if (n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads > 4096 || n_kv_heads > 4096)
    return fail(BI_ERR_INVALID_ARG, "gemm_qkv: bad head counts");
  const int64_t N = (int64_t)(n_q_heads + 2 * n_kv_heads) * BI_HEAD_DIM;
  bi_status st = gemm::check_args(A, lda, W, ldw, qkv, ldq, BI_BF16, M, N, K);
  if (st != BI_OK) return st;
  if (!positions || !cos_sin || !slot_mapping || !k_cache || !v_cache)
    return fail(BI_ERR_INVALID_ARG, "gemm_qkv: null pointer");
  if (max_pos <= 0 || num_pages <= 0) return fail(BI_ERR_INVALID_ARG, "gemm_qkv: bad max_pos / num_pages");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(cos_sin))
    return fail(BI_ERR_ALIGN, "gemm_qkv: caches and table must be 16-byte aligned");
  if (M == 0) return BI_OK;
  if ((st = require_sm100()) != BI_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  bf16* out = static_cast<bf16*>(qkv);
  if (K == 0 || gemm::split_of(N, K, false) != 1) {
    // the same steps as three launches: the fused epilogue handles unsplit weights only
    if ((st = gemm::launch<1, gemm::EPI_STORE>(A, nullptr, lda, W, ldw, qkv, ldq, BI_BF16, M, N, K, s)) != BI_OK)
      return st;
    if ((st = launch_rope(out, ldq, n_q_heads + n_kv_heads, positions, M, cos_sin, max_pos, s)) != BI_OK)
      return st;
    return launch_kv_append(out + (size_t)n_q_heads * BI_HEAD_DIM,
                            out + (size_t)(n_q_heads + n_kv_heads) * BI_HEAD_DIM, ldq, slot_mapping, M,
                            static_cast<bf16*>(k_cache), static_cast<bf16*>(v_cache), n_kv_heads,
                            num_pages, s);
  }
  gemm::QkvArgs qa{positions, cos_sin, slot_mapping, static_cast<bf16*>(k_cache),
                   static_cast<bf16*>(v_cache), max_pos, num_pages, n_q_heads, n_kv_heads};
  return gemm::launch<1, gemm::EPI_QKV>(A, nullptr, lda, W, ldw, qkv, ldq, BI_BF16, M, N, K, s, &qa);
}

extern "C" bi_status bi_gemm_x2(const void* A_hi, const void* A_lo, int64_t lda, const void* W,
                                int64_t ldw, void* C, int64_t ldc, int32_t c_dtype, int64_t M,
                                int64_t N, int64_t K, void* stream) {
  bi_status st = gemm::check_args(A_hi, lda, W, ldw, C, ldc, c_dtype, M, N, K);
  if (st != BI_OK) return st;
  if (!A_lo) return fail(BI_ERR_INVALID_ARG, "gemm_x2: A_lo is null");
  if (!aligned16(A_lo)) return fail(BI_ERR_ALIGN, "gemm_x2: A_lo must be 16-byte aligned");
  if (M == 0 || N == 0) return BI_OK;
  if ((st = require_sm100()) != BI_OK) return st;
  if (c_dtype == BI_F32_ADD)
    return gemm::launch<2, gemm::EPI_ADD>(A_hi, A_lo, lda, W, ldw, C, ldc, c_dtype, M, N, K,
                                          static_cast<cudaStream_t>(stream));
  return gemm::launch<2, gemm::EPI_STORE>(A_hi, A_lo, lda, W, ldw, C, ldc, c_dtype, M, N, K,
                                          static_cast<cudaStream_t>(stream));
}
