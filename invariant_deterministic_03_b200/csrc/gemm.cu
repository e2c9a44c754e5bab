// gemm.cu -- batch-invariant GEMM on the 5th-generation tensor cores.
//
// "Defeating Nondeterminism in LLM Inference", section "Batch-invariant
// matmul": tile the OUTPUT and keep each element's whole K reduction inside
// one core; never split K (split-K) nor hand different K ranges of a tile to
// different cores (stream-K); and compile ONE kernel configuration for every
// shape, because different tensor-core instructions may reduce in different
// internal orders. The page accepts the cost of this at small batches.
//
// The one configuration (for every M, N, K):
//   output tile 256 x BN (BN = BI_GEMM_BN), computed by a pair of CTAs (a
//   two-CTA cluster) with the instruction tcgen05.mma.cta_group::2.kind::f16
//   M=256 N=BN K=16, bf16 operands, fp32 accumulator in tensor memory, K
//   stage 64. Each CTA of the pair holds 128 rows of A and BN/2 rows of W in
//   its own shared memory and its 128 x BN half of the accumulator in its own
//   tensor memory; rank 0 issues the MMAs for both. Element (m, n) is
//   accumulated by the K-steps k = 0, 16, 32, ... in that order, whatever M
//   is; no K range of a tile is ever handed to another pair. Which pair
//   computes a tile (persistent round-robin), how many rows an A copy carries
//   and what is prefetched into L2 change timing only, never arithmetic.
//
// CTA layout (192 threads, one CTA per SM, pairs persistent over tiles):
//   warp 0      TMA producer of this CTA's half: A [128 x 64] and W [BN/2 x
//               64] tiles, 128-byte swizzle, into a shared-memory stage ring;
//               every copy of both CTAs completes on rank 0's "full" barrier
//               of the stage, the MMAs free the stage in both CTAs.
//               Small M (every pair holds at most one tile): W tiles are also
//               prefetched into L2 W_PREFETCH stages ahead of the loads; when
//               M < 128 rank 0's A copy carries only the M rows rounded up to
//               8, and a CTA whose 128 rows all lie past M copies no A at all
//               (its stage keeps stale rows: the MMA still runs M=256, and
//               rows past M, never stored, read whatever the stage held; no
//               row of the product depends on another row).
//   warp 1      allocates 2 x BN tensor-memory columns (two accumulators) for
//               the pair; on rank 0 lane 0 issues the MMAs and commits, each
//               commit one tcgen05.commit multicast to the same barrier in
//               both CTAs (stage free, accumulator full), which each CTA
//               waits on at CTA scope (one commit to both measured ~5 %
//               faster than a commit per CTA with cluster-scope waits)
//   warps 2..5  (FOLD only, first) write the A stages from fp32 rows, see
//               gemm_tcgen05_kernel; then
//               epilogue of this CTA's 128 rows: tcgen05.ld the accumulator
//               row by row (thread = row), round to bf16 (RNE) or keep fp32,
//               store to global, or run one of the fused epilogues (EPI_ADD,
//               EPI_SWIGLU, EPI_QKV below) on the finished values; then free
//               the accumulator (an arrival on rank 0's barrier).
// Every mbarrier wait is bounded (see common.cuh); a timeout sets a status
// bit and both CTAs wind down, releasing their tensor memory.
#include <mutex>

#include "common.cuh"
#include "host.h"

namespace bi {
namespace gemm {

constexpr int BM = BI_GEMM_BM;       // 256: rows of a pair tile
constexpr int BM_CTA = BM / 2;       // 128: rows held by one CTA of the pair
constexpr int BN = BI_GEMM_BN;       // columns of a tile (the MMA's N)
constexpr int BK = BI_GEMM_BK;       // 64 bf16 = 128 bytes = one swizzle row
constexpr int UMMA_K = 16;
static_assert(BM == 256, "the pair tile is 256 rows");
static_assert(BN % 128 == 0 && BN >= 128 && BN <= 256, "BN: 128 or 256 (whole 128-column heads per tile)");
constexpr uint32_t A_BYTES = BM_CTA * BK * 2;        // 16 KB per CTA
constexpr uint32_t B_BYTES = (BN / 2) * BK * 2;      // half of the W tile per CTA
constexpr uint32_t TMEM_COLS = 2 * BN;               // two accumulators (power of two)
constexpr int THREADS = 192;
constexpr int W_PREFETCH = 8;  // W stages prefetched into L2 ahead of the loads (small M)
constexpr size_t SMEM_LIMIT = 232448;  // dynamic shared memory per CTA on sm_100
constexpr size_t BAR_BYTES = 512;

// TERMS = number of bf16 A operands summed into the product: 1 for plain
// bf16 activations, 2 for an activation carried as a hi/lo pair (A = A_hi +
// A_lo, ~16 significant bits). Both terms meet the same W tile in shared
// memory, so W is read once.
template <int TERMS>
struct Cfg {
  static constexpr uint32_t STAGE_BYTES = TERMS * A_BYTES + B_BYTES;
  static constexpr int FIT = (int)((SMEM_LIMIT - 1024 - BAR_BYTES) / STAGE_BYTES);
  static constexpr int STAGES = FIT < 12 ? FIT : 12;
  static constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + BAR_BYTES;
  static_assert(STAGES >= 3, "gemm: too few stages");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "gemm: shared memory above the per-CTA limit");
  static_assert((2 * STAGES + 6) * 8 + 8 <= BAR_BYTES, "gemm: barrier area too small");
};

struct Params {
  void* C;
  int64_t ldc;
  int32_t c_f32;
  int32_t M, N, K;
  int32_t m_blocks, n_blocks, k_blocks;  // m_blocks counts 256-row pair tiles
  int32_t w_prefetch;  // W_PREFETCH or 0 (off)
  uint32_t a_bytes;    // bytes of one A copy: 128 rows, or M rounded up to 8 when M < 128
  int32_t* status;
  // EPI_QKV only: RoPE of the q and k heads and the paged-cache write
  const int32_t* pos;    // [M] absolute positions
  const float* cs;       // [max_pos, 64, 2] cos / sin
  const int32_t* slots;  // [M] cache slots (page * 16 + offset), < 0: padding row
  uint16_t* kc;          // key cache (16-bit elements), 4 KB per (page, kv head)
  uint16_t* vc;          // value cache, same blocking, transposed per page
  int32_t max_pos, num_pages, hq, hkv;
  // FOLD only: A[m, k] = r16((x[m, k] * r[m]) * gamma[k]), the RMSNorm of the
  // fp32 rows x applied while the A tile is written to shared memory
  const float* fx;       // [M, ldx] fp32 rows
  int64_t ldx;
  const float* fr;       // [M] row scales (rmsnorm_scales_f32)
  const uint16_t* fg;    // [K] gamma, 16-bit (the element type)
};

template <typename ET>
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
    ET* dst = static_cast<ET*>(p.C) + (size_t)row * p.ldc + col0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (col0 + g * 8 < p.N) {
        uint4 o;
        o.x = E16<ET>::pack2(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]));
        o.y = E16<ET>::pack2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
        o.z = E16<ET>::pack2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]));
        o.w = E16<ET>::pack2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
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

template <typename ET>
__device__ __forceinline__ float round16(uint32_t acc) {
  return E16<ET>::round(__uint_as_float(acc));
}

// out[row, f0 .. f0+31] = r16(swiglu(r16(gate), r16(up))); F % 8 == 0 (r16:
// rounding to the 16-bit element type).
template <typename ET>
__device__ __forceinline__ void store_swiglu_chunk(const Params& p, int row, int f0, const uint32_t (&g)[32],
                                                   const uint32_t (&u)[32]) {
  ET* dst = static_cast<ET*>(p.C) + (size_t)row * p.ldc + f0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (f0 + q * 8 < p.N) {
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = swiglu_f32(round16<ET>(g[8 * q + k]), round16<ET>(u[8 * q + k]));
      uint4 o;
      o.x = E16<ET>::pack2(v[0], v[1]);
      o.y = E16<ET>::pack2(v[2], v[3]);
      o.z = E16<ET>::pack2(v[4], v[5]);
      o.w = E16<ET>::pack2(v[6], v[7]);
      *reinterpret_cast<uint4*>(dst + 8 * q) = o;
    }
  }
}

// Epilogue of a tile (EPI):
//   EPI_STORE   C = acc, rounded to bf16 (RNE) or kept fp32;
//   EPI_ADD     C (fp32) = C + acc: one fp32 addition per element after the
//               whole K reduction (a residual connection in the stream);
//   EPI_SWIGLU  the tile's BN accumulator columns are BN/2 gate features
//               (W rows f, held by rank 0) and the same BN/2 up features (W
//               rows F + f, held by rank 1):
//               C[m, f] = bf16(swiglu_f32(bf16(g), bf16(u))), the same
//               rounding points as a bf16 GEMM followed by bi_swiglu.
constexpr int EPI_STORE = 0, EPI_ADD = 1, EPI_SWIGLU = 2, EPI_QKV = 3;

// EPI_QKV: the fused [q | k | v] projection (heads of 128 columns, so a
// BN-column tile is heads HPT nb .. HPT nb + HPT - 1, HPT = BN / 128). Every
// element is first rounded to bf16 as EPI_STORE does. q and k heads then
// rotate each pair (i, i + 64) with the RoPE kernel's arithmetic
// (rope_rotate on the bf16 values and the fp32 table) and are stored rounded
// again; k and v heads are also written to the paged caches at the row's
// slot, in the KV append's layout:
//   keys:   element (slot o, d) at (o/8)*1024 + (d/8)*64 + (o%8)*8 + d%8
//   values: element (d, slot o) at (d/8)*128 + (o/8)*64 + (d%8)*8 + o%8
// of the (page, kv head) block. The qkv rows and both caches end up with the
// same bits as bi_gemm, then bi_rope over the q and k heads, then
// bi_kv_append. The tensor-memory loads are warp-collective, so every lane
// runs them; only rows < M store.
constexpr int HPT = BN / 128;
template <typename ET>
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
  if (live && !rot && nb * HPT < p.hq + p.hkv) set_status(p.status, BI_DEV_BAD_TOKEN);
  const int n_heads = p.hq + 2 * p.hkv;
  uint16_t* crow = static_cast<uint16_t*>(p.C) + (size_t)(live ? row : 0) * p.ldc;
  // q / k heads of this tile rotate with the row's cos / sin: loaded once per
  // 32-pair block for both heads, before the accumulator reads
  const int n_rot = max(0, min(HPT, p.hq + p.hkv - nb * HPT));  // leading heads of the tile that rotate
  const float* csrow = p.cs + (size_t)(rot ? pos : 0) * 128;
#pragma unroll 1
  for (int j = 0; j < 2 && n_rot > 0; ++j) {
    float4 t[16];  // cos / sin of pairs 32 j .. 32 j + 31
#pragma unroll
    for (int q = 0; q < 16; ++q)
      t[q] = (live && rot) ? reinterpret_cast<const float4*>(csrow + j * 64)[q] : make_float4(1.f, 0.f, 1.f, 0.f);
#pragma unroll 1
    for (int hh = 0; hh < n_rot; ++hh) {
      const int H = nb * HPT + hh;
      const bool is_k = H >= p.hq;
      uint16_t* out = crow + (size_t)H * BI_HEAD_DIM;
      if (j == 0 && is_k && live && slot_bad) set_status(p.status, BI_DEV_BAD_SLOT);
      uint16_t* kdst = p.kc + ((size_t)page * p.hkv + (is_k ? H - p.hq : 0)) * (BI_PAGE_SIZE * BI_HEAD_DIM) +
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
          const float a = round16<ET>(ra[8 * g + e]), b = round16<ET>(rb[8 * g + e]);
          if (rot) rope_rotate(a, b, (e & 1) ? c.z : c.x, (e & 1) ? c.w : c.y, ya[e], yb[e]);
          else { ya[e] = a; yb[e] = b; }
        }
        const uint4 A = make_uint4(E16<ET>::pack2(ya[0], ya[1]), E16<ET>::pack2(ya[2], ya[3]),
                                   E16<ET>::pack2(ya[4], ya[5]), E16<ET>::pack2(ya[6], ya[7]));
        const uint4 B = make_uint4(E16<ET>::pack2(yb[0], yb[1]), E16<ET>::pack2(yb[2], yb[3]),
                                   E16<ET>::pack2(yb[4], yb[5]), E16<ET>::pack2(yb[6], yb[7]));
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
  for (int hh = n_rot; hh < HPT; ++hh) {
    const int H = nb * HPT + hh;
    if (H >= n_heads) break;  // uniform across the warp
    uint16_t* out = crow + (size_t)H * BI_HEAD_DIM;
    if (live && slot_bad) set_status(p.status, BI_DEV_BAD_SLOT);
    {
      uint16_t* vdst = p.vc + ((size_t)page * p.hkv + (H - p.hq - p.hkv)) * (BI_PAGE_SIZE * BI_HEAD_DIM) +
                   (o >> 3) * 64 + (o & 7);
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        uint32_t r[32];
        tmem_ld32(taddr + (hh * 4 + j) * 32, r);
        tmem_ld_wait();
        if (!live) continue;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint4 V = make_uint4(E16<ET>::pack2(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1])),
                                     E16<ET>::pack2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3])),
                                     E16<ET>::pack2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5])),
                                     E16<ET>::pack2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7])));
          const int d0 = j * 32 + g * 8;
          *reinterpret_cast<uint4*>(out + d0) = V;
          if (to_cache) {
            const uint16_t* v8 = reinterpret_cast<const uint16_t*>(&V);
#pragma unroll
            for (int e = 0; e < 8; ++e) vdst[((d0 + e) >> 3) * 128 + ((d0 + e) & 7) * 8] = v8[e];
          }
        }
      }
    }
  }
}

// FOLD (TERMS = 1, only when every pair holds at most one tile): warps 2..5
// write each A stage themselves before their epilogue, as r16((x * r) * gamma)
// from fp32 rows -- the operations of bi_rmsnorm_f32in, so A holds the same
// bits as that kernel's output and the product is the same as bi_rmsnorm_f32in
// then bi_gemm. Each of the 8 warps (4 per CTA) arrives on rank 0's "full"
// barrier of the stage after its rows are written and fenced for the tensor
// core; the W copies arrive as in the TMA path.
template <int TERMS, int EPI, typename ET, bool FOLD = false>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmA2,
                        const __grid_constant__ CUtensorMap tmB, const Params p) {
  constexpr int STAGES = Cfg<TERMS>::STAGES;
  constexpr uint32_t STAGE_BYTES = Cfg<TERMS>::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzled tiles want 1024-byte aligned bases; the offsets are the
  // same in both CTAs of the pair (the MMA descriptors name them for both).
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);  // used on rank 0
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2] used on rank 0: 4 epilogue warps x 2 CTAs
  uint64_t* drain = acc_empty + 2;       // rank 0's MMA thread, on abort only
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = p.m_blocks * p.n_blocks;
  const uint32_t rank = cluster_rank();  // 0: issues the MMAs, 1: its peer
  const int tile0 = (int)blockIdx.x >> 1, tile_step = (int)gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], FOLD ? 9 : 1);  // FOLD: + one arrival per A-writing warp of both CTAs
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    if (TERMS == 2) prefetch_tmap(&tmA2);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_base_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised and tensor memory allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;

  if (warp == 0) {
    // ---------------- TMA producer (this CTA's half of every stage)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int fills[STAGES];
      for (int s = 0; s < STAGES; ++s) fills[s] = 0;
      for (int tile = tile0; tile < num_tiles && ok; tile += tile_step) {
        const int mb = tile % p.m_blocks, nb = tile / p.m_blocks;
        const int pf = p.w_prefetch;
        const int a_row = mb * BM + (int)rank * BM_CTA;  // this CTA's first A row
        const bool a_live = a_row < p.M;
        // bytes landing on rank 0's full barrier per stage: both CTAs' copies
        const bool a1_live = mb * BM + BM_CTA < p.M;
        const uint32_t tx = FOLD ? 2u * B_BYTES : TERMS * p.a_bytes * (a1_live ? 2u : 1u) + 2u * B_BYTES;
        // W rows of this CTA: BN/2 from nb * BN + rank * BN/2, or (SwiGLU)
        // BN/2 gate rows from nb * BN/2 (rank 0) or the matching up rows
        // from F + nb * BN/2 (rank 1)
        const int w_row = EPI == EPI_SWIGLU ? (int)rank * p.N + nb * (BN / 2) : nb * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < pf && kb < p.k_blocks; ++kb) tma_prefetch_2d(&tmB, kb * BK, w_row);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, p.status, abort_flag)) { ok = false; break; }
          if (pf && kb + pf < p.k_blocks) tma_prefetch_2d(&tmB, (kb + pf) * BK, w_row);
          uint8_t* sa = tiles + stage * STAGE_BYTES;
          const uint32_t fb = cluster_addr(&full[stage], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], tx);
          if (!FOLD && a_live) {
            tma_load_2d_pair(sa, &tmA, fb, kb * BK, a_row);
            if (TERMS == 2) tma_load_2d_pair(sa + A_BYTES, &tmA2, fb, kb * BK, a_row);
          }
          tma_load_2d_pair(sa + TERMS * A_BYTES, &tmB, fb, kb * BK, w_row);
          ++fills[stage];
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // Let copies already in flight land before the CTA can exit. Rank 0
        // waits (bounded) for each stage's last fill; rank 1's copies
        // complete on rank 0's barriers, which it cannot observe, so it
        // waits a fixed ~2^22 cycles, far longer than a copy takes.
        if (rank == 0) {
          for (int s = 0; s < STAGES; ++s) {
            if (fills[s] == 0) continue;
            const uint32_t par = (uint32_t)(fills[s] - 1) & 1u;
            const long long t0 = clock64();
            while (!mbar_try_wait(&full[s], par) && clock64() - t0 < kWaitLimitCycles) {
            }
          }
        } else {
          const long long t0 = clock64();
          while (clock64() - t0 < (1ll << 22)) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread of rank 0, for both CTAs)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(BM, BN, E16<ET>::kMmaFormat);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, issued = false;
      for (int tile = tile0; tile < num_tiles && ok; tile += tile_step) {
        if (!mbar_wait_cluster(&acc_empty[acc], acc_phase ^ 1, p.status, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
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
              mma_f16k_pair(d_tmem, ad, bd, idesc, (kb != 0 || term != 0 || k != 0));
            }
          }
          issued = true;
          // frees the stage in both CTAs once these MMAs retire
          mma_commit_pair_both(smem_u32(&empty[stage]));
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        // accumulator complete, in both CTAs' tensor memory
        mma_commit_pair_both(smem_u32(&acc_full[acc]));
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      if (!ok && issued) {
        // no MMA may still be writing tensor memory or reading a stage when
        // the pair frees them: wait (bounded) until every issued MMA is done
        mma_commit_pair(smem_u32(drain));
        const long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitLimitCycles) {
        }
      }
    }
  } else {
    // ---------------- epilogue warps 2..5: TMEM lanes 32*(warp%4) .. +31
    const int quarter = warp & 3;
    const int trow = quarter * 32 + lane;  // accumulator row (TMEM lane) of this thread
    const uint32_t acc_empty0 = cluster_addr(acc_empty, 0);
    if constexpr (FOLD) {
      // A stages of this CTA's 128 rows (the pair's only tile). The 128
      // threads of warps 2..5 share the rows below M: eight threads per row,
      // one 16-byte chunk (8 columns) each, so a row's fp32 x is read in one
      // coalesced 256-byte piece; a thread has at most 8 chunks per stage.
      // Two register sets hold the loads of two stages, so a stage's loads
      // are in flight while the one before it is converted.
      constexpr int CH = 8;
      bool ok = tile0 < num_tiles;
      const int mb = ok ? tile0 % p.m_blocks : 0;
      const int row_base = mb * BM + (int)rank * BM_CTA;
      const int live = max(0, min(BM_CTA, p.M - row_base));
      const int ct = (int)threadIdx.x - 64;          // 0 .. 127
      const uint32_t full0 = cluster_addr(full, 0);  // rank 0's barriers
      float4 xa[CH][2], xb[CH][2];
      uint4 ga[CH], gb[CH];
      float ra[CH], rb[CH];
      // the loads of stage kb's chunks into one register set
      auto load = [&](int kb, float4 (&x)[CH][2], uint4 (&g)[CH], float (&r)[CH]) {
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const int c = ct + 128 * j;
          const int row = c >> 3, k0 = kb * BK + (c & 7) * 8;
          if (row < live && k0 < p.K) {  // K % 8 == 0: a chunk is wholly inside or outside
            const float* xr = p.fx + (size_t)(row_base + row) * p.ldx + k0;
            x[j][0] = *reinterpret_cast<const float4*>(xr);
            x[j][1] = *reinterpret_cast<const float4*>(xr + 4);
            g[j] = *reinterpret_cast<const uint4*>(p.fg + k0);
            r[j] = p.fr[row_base + row];
          }
        }
      };
      // r16((x r) gamma) of stage kb's chunks into the stage's A tile
      auto store = [&](int kb, uint8_t* sa, const float4 (&x)[CH][2], const uint4 (&g)[CH], const float (&r)[CH]) {
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const int c = ct + 128 * j;
          const int row = c >> 3, ch = c & 7, k0 = kb * BK + ch * 8;
          if (row >= live) continue;  // rows past M are never stored; they keep stale values
          uint4 o = make_uint4(0u, 0u, 0u, 0u);  // columns past K: zeros, as a TMA copy would fill
          if (k0 < p.K) {
            const float xv[8] = {x[j][0].x, x[j][0].y, x[j][0].z, x[j][0].w,
                                 x[j][1].x, x[j][1].y, x[j][1].z, x[j][1].w};
            const uint32_t g2[4] = {g[j].x, g[j].y, g[j].z, g[j].w};
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float lo = __fmul_rn(__fmul_rn(xv[2 * e], r[j]), E16<ET>::lo(g2[e]));
              const float hi = __fmul_rn(__fmul_rn(xv[2 * e + 1], r[j]), E16<ET>::hi(g2[e]));
              w[e] = E16<ET>::pack2(lo, hi);
            }
            o = make_uint4(w[0], w[1], w[2], w[3]);
          }
          // 128-byte swizzle of a 1024-byte aligned tile: chunk ch of row
          // `row` sits at chunk ch ^ (row % 8) of the row
          *reinterpret_cast<uint4*>(sa + row * 128 + ((ch ^ (row & 7)) << 4)) = o;
        }
      };
      int stage = 0;
      uint32_t phase = 0;
      if (ok) load(0, xa, ga, ra);
      if (ok && p.k_blocks > 1) load(1, xb, gb, rb);
      for (int kb = 0; kb < p.k_blocks && ok; ++kb) {
        const bool even = (kb & 1) == 0;
        if (!mbar_wait(&empty[stage], phase ^ 1, p.status, abort_flag)) { ok = false; break; }
        uint8_t* sa = tiles + stage * STAGE_BYTES;
        if (even) store(kb, sa, xa, ga, ra);
        else store(kb, sa, xb, gb, rb);
        fence_proxy_async_smem();  // the writes, visible to the tensor core
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive(&full[stage]);
          else mbar_arrive_cluster(full0 + stage * 8);
        }
        // the loads of the stage two ahead into the registers just used,
        // issued after the fence so that it does not wait for them
        if (kb + 2 < p.k_blocks) {
          if (even) load(kb + 2, xa, ga, ra);
          else load(kb + 2, xb, gb, rb);
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = tile0; tile < num_tiles; tile += tile_step) {
      const int mb = tile % p.m_blocks, nb = tile / p.m_blocks;
      if (!mbar_wait(&acc_full[acc], acc_phase, p.status, abort_flag)) break;
      tc_fence_after();
      const int row = mb * BM + (int)rank * BM_CTA + trow;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      constexpr int UP = BN / 64;  // SwiGLU: the up chunk paired with gate chunk c is c + UP
      uint32_t held[32];  // SwiGLU: a gate chunk until its up chunk arrives
      auto col_of = [&](int c) {
        return EPI == EPI_SWIGLU ? nb * (BN / 2) + (c % UP) * 32 : nb * BN + c * 32;
      };
      if constexpr (EPI == EPI_QKV) {
        qkv_tile<ET>(p, row, nb, taddr);
      } else {
#pragma unroll 1
        for (int q = 0; q < BN / 32; ++q) {
          const int c = EPI == EPI_SWIGLU ? ((q & 1) ? UP + (q >> 1) : (q >> 1)) : q;
          if (col_of(c) >= p.N) break;  // uniform across the warp
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          if (row >= p.M) continue;
          if constexpr (EPI == EPI_SWIGLU) {
            if (c >= UP) {
              store_swiglu_chunk<ET>(p, row, col_of(c), held, r);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) held[i] = r[i];
            }
          } else if constexpr (EPI == EPI_ADD) {
            add_row_chunk(p, row, col_of(c), r);
          } else {
            store_row_chunk<ET>(p, row, col_of(c), r);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + acc * 8);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA leaves (or frees tensor memory) while the other may still
  // arrive on its barriers or its MMAs may still run
  cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

__global__ void zero_fill_kernel(void* C, int64_t ldc, int32_t c_f32, int32_t M, int32_t N) {
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t total = (int64_t)M * N;
  for (; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    int64_t m = i / N, n = i % N;
    if (c_f32) static_cast<float*>(C)[m * ldc + n] = 0.0f;
    else static_cast<uint16_t*>(C)[m * ldc + n] = 0;  // +0 in bf16 and fp16 alike
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

template <int TERMS, int EPI, typename ET, bool FOLD = false>
static bi_status set_smem_attr() {
  static bool done[64] = {false};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return fail(BI_ERR_UNSUPPORTED, "gemm: device id %d out of range", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tcgen05_kernel<TERMS, EPI, ET, FOLD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<TERMS>::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e, "gemm: smem attribute");
    done[dev] = true;
  }
  return BI_OK;
}

// How many CTA pairs of this kernel the device runs at once (queried once per
// device).
template <int TERMS, int EPI, typename ET, bool FOLD = false>
static bi_status pair_slots(int* out) {
  static int cache[64] = {0};
  static std::mutex mu;
  bi_status st = set_smem_attr<TERMS, EPI, ET, FOLD>();
  if (st != BI_OK) return st;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  int& v = cache[dev];
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
    cudaError_t e = cudaOccupancyMaxActiveClusters(&n, gemm_tcgen05_kernel<TERMS, EPI, ET, FOLD>, &cfg);
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
  uint16_t* kc;
  uint16_t* vc;
  int32_t max_pos, num_pages, hq, hkv;
};

struct FoldArgs {
  const float* x;
  int64_t ldx;
  const float* r;
  const void* gamma;
};

// N is the output width: the W rows for EPI_STORE / EPI_ADD / EPI_QKV, the
// feature count F (W has 2F rows) for EPI_SWIGLU. FOLD: A comes from fa (the
// caller has checked that every pair holds at most one tile).
template <int TERMS, int EPI, typename ET, bool FOLD = false>
static bi_status launch(const void* A, const void* A2, int64_t lda, const void* W, int64_t ldw,
                        void* C, int64_t ldc, int32_t c_dtype, int64_t M, int64_t N, int64_t K,
                        cudaStream_t s, const QkvArgs* qa = nullptr, const FoldArgs* fa = nullptr) {
  bi_status st;
  const int32_t c_f32 = c_dtype != BI_BF16;
  if (K == 0) {
    if (EPI == EPI_ADD) return BI_OK;  // C += 0
    zero_fill_kernel<<<296, 256, 0, s>>>(C, ldc, c_f32, (int32_t)M, (int32_t)N);
    BI_CHECK_LAUNCH("gemm zero fill");
    return BI_OK;
  }
  CUtensorMap tmA, tmA2, tmB;
  const uint32_t a_rows = M < BM_CTA ? (uint32_t)((M + 7) / 8 * 8) : (uint32_t)BM_CTA;
  if (!FOLD) {
    uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
    uint64_t strides[1] = {(uint64_t)lda * 2};
    uint32_t box[2] = {BK, a_rows};
    if ((st = encode_tmap(&tmA, E16<ET>::kTmap, 2, const_cast<void*>(A), dims,
                          strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != BI_OK)
      return st;
    if (TERMS == 2) {
      if ((st = encode_tmap(&tmA2, E16<ET>::kTmap, 2, const_cast<void*>(A2), dims,
                            strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != BI_OK)
        return st;
    } else {
      tmA2 = tmA;
    }
  }
  {
    uint64_t dims[2] = {(uint64_t)K, (uint64_t)(EPI == EPI_SWIGLU ? 2 * N : N)};
    uint64_t strides[1] = {(uint64_t)ldw * 2};
    uint32_t box[2] = {BK, BN / 2};
    if ((st = encode_tmap(&tmB, E16<ET>::kTmap, 2, const_cast<void*>(W), dims,
                          strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != BI_OK)
      return st;
  }
  if (FOLD) tmA = tmA2 = tmB;  // not read: the A stages are written by the kernel
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
  p.fx = fa ? fa->x : nullptr;
  p.ldx = fa ? fa->ldx : 0;
  p.fr = fa ? fa->r : nullptr;
  p.fg = fa ? static_cast<const uint16_t*>(fa->gamma) : nullptr;
  p.a_bytes = a_rows * BK * 2;
  int slots = 0;
  if ((st = pair_slots<TERMS, EPI, ET, FOLD>(&slots)) != BI_OK) return st;
  const int64_t tiles = (int64_t)p.m_blocks * p.n_blocks;
  if (FOLD && (tiles > slots || !fa)) return fail(BI_ERR_SHAPE, "gemm fold: more tiles than CTA pairs");
  p.w_prefetch = tiles <= slots ? W_PREFETCH : 0;
  const int64_t pairs = tiles < slots ? tiles : slots;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = Cfg<TERMS>::SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_tcgen05_kernel<TERMS, EPI, ET, FOLD>, tmA, tmA2, tmB, p);
  if (e != cudaSuccess) return cuda_fail(e, "gemm: cluster launch");
  BI_CHECK_LAUNCH("gemm launch");
  return BI_OK;
}

}  // namespace gemm
}  // namespace bi

namespace bi {
bi_status launch_kv_append(const uint16_t* k, const uint16_t* v, int64_t ld_new, const int32_t* slots,
                           int64_t n_tok, uint16_t* kc, uint16_t* vc, int Hkv, int num_pages,
                           cudaStream_t s);
template <typename ET>
bi_status launch_rope(ET* x, int64_t ldx, int n_heads, const int32_t* pos, int64_t n_tok,
                      const float* cs, int max_pos, cudaStream_t s);

// The GEMM entry points for one 16-bit element type (bf16: the C ABI's
// bi_gemm*, fp16: bi_gemm_f16 and the FP16 precision mode of bi_forward).
template <typename ET>
bi_status gemm_e16(const void* A, int64_t lda, const void* W, int64_t ldw, void* C, int64_t ldc,
                   int32_t c_dtype, int64_t M, int64_t N, int64_t K, cudaStream_t s) {
  bi_status st = gemm::check_args(A, lda, W, ldw, C, ldc, c_dtype, M, N, K);
  if (st != BI_OK || M == 0 || N == 0) return st;
  if ((st = require_sm100()) != BI_OK) return st;
  if (c_dtype == BI_F32_ADD)
    return gemm::launch<1, gemm::EPI_ADD, ET>(A, nullptr, lda, W, ldw, C, ldc, c_dtype, M, N, K, s);
  return gemm::launch<1, gemm::EPI_STORE, ET>(A, nullptr, lda, W, ldw, C, ldc, c_dtype, M, N, K, s);
}

template <typename ET>
bi_status gemm_swiglu_e16(const void* A, int64_t lda, const void* W, int64_t ldw, void* out,
                          int64_t ldo, int64_t M, int64_t F, int64_t K, cudaStream_t s) {
  bi_status st = gemm::check_args(A, lda, W, ldw, out, ldo, BI_BF16, M, F, K);
  if (st != BI_OK || M == 0 || F == 0) return st;
  if (F > (1ll << 29)) return fail(BI_ERR_SHAPE, "gemm_swiglu: F above 2^29");
  if ((st = require_sm100()) != BI_OK) return st;
  return gemm::launch<1, gemm::EPI_SWIGLU, ET>(A, nullptr, lda, W, ldw, out, ldo, BI_BF16, M, F, K, s);
}

template <typename ET>
bi_status gemm_qkv_e16(const void* A, int64_t lda, const void* W, int64_t ldw, void* qkv, int64_t ldq,
                       int64_t M, int64_t K, int32_t n_q_heads, int32_t n_kv_heads, const int32_t* positions,
                       const float* cos_sin, int32_t max_pos, const int32_t* slot_mapping, void* k_cache,
                       void* v_cache, int32_t num_pages, cudaStream_t s) {
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
  ET* out = static_cast<ET*>(qkv);
  if (K == 0) {
    // zeros, then the same steps as three launches
    if ((st = gemm::launch<1, gemm::EPI_STORE, ET>(A, nullptr, lda, W, ldw, qkv, ldq, BI_BF16, M, N, K, s)) != BI_OK)
      return st;
    if ((st = launch_rope<ET>(out, ldq, n_q_heads + n_kv_heads, positions, M, cos_sin, max_pos, s)) != BI_OK)
      return st;
    return launch_kv_append(reinterpret_cast<const uint16_t*>(out + (size_t)n_q_heads * BI_HEAD_DIM),
                            reinterpret_cast<const uint16_t*>(out + (size_t)(n_q_heads + n_kv_heads) * BI_HEAD_DIM),
                            ldq, slot_mapping, M, static_cast<uint16_t*>(k_cache), static_cast<uint16_t*>(v_cache),
                            n_kv_heads, num_pages, s);
  }
  gemm::QkvArgs qa{positions, cos_sin, slot_mapping, static_cast<uint16_t*>(k_cache),
                   static_cast<uint16_t*>(v_cache), max_pos, num_pages, n_q_heads, n_kv_heads};
  return gemm::launch<1, gemm::EPI_QKV, ET>(A, nullptr, lda, W, ldw, qkv, ldq, BI_BF16, M, N, K, s, &qa);
}

template bi_status gemm_e16<bf16>(const void*, int64_t, const void*, int64_t, void*, int64_t, int32_t, int64_t,
                                  int64_t, int64_t, cudaStream_t);
template bi_status gemm_swiglu_e16<bf16>(const void*, int64_t, const void*, int64_t, void*, int64_t, int64_t,
                                         int64_t, int64_t, cudaStream_t);
template bi_status gemm_qkv_e16<bf16>(const void*, int64_t, const void*, int64_t, void*, int64_t, int64_t, int64_t,
                                      int32_t, int32_t, const int32_t*, const float*, int32_t, const int32_t*,
                                      void*, void*, int32_t, cudaStream_t);
template bi_status gemm_e16<f16>(const void*, int64_t, const void*, int64_t, void*, int64_t, int32_t, int64_t,
                                 int64_t, int64_t, cudaStream_t);
template bi_status gemm_swiglu_e16<f16>(const void*, int64_t, const void*, int64_t, void*, int64_t, int64_t,
                                        int64_t, int64_t, cudaStream_t);
template bi_status gemm_qkv_e16<f16>(const void*, int64_t, const void*, int64_t, void*, int64_t, int64_t, int64_t,
                                     int32_t, int32_t, const int32_t*, const float*, int32_t, const int32_t*,
                                     void*, void*, int32_t, cudaStream_t);
}  // namespace bi

namespace bi {
bi_status rmsnorm_scales_f32(const float* x, int64_t M, int64_t D, float eps, float* r, cudaStream_t s);

namespace gemm {
// Workspace of the RMSNorm-folded GEMM: the row scales (M fp32, 256-byte
// rounded), then room for the normed rows (M x K bf16) used when the fold
// does not apply.
static size_t fold_ws_bytes(int64_t M, int64_t K) {
  return (((size_t)M * 4 + 255) & ~(size_t)255) + (size_t)M * K * 2;
}

// C = (RMSNorm(x) with gamma) W^T, x fp32 [M, K] contiguous. When every CTA
// pair holds at most one output tile the norm is applied inside the GEMM
// (FOLD: the row scales first, by bi_rmsnorm_f32in's reduction, then the
// GEMM writes r16((x r) gamma) into its A stages); otherwise the normed rows
// go through the workspace (bi_rmsnorm_f32in, then the plain GEMM). Either
// way the bits are those of bi_rmsnorm_f32in followed by bi_gemm (or
// bi_gemm_swiglu for EPI_SWIGLU).
template <int EPI>
static bi_status rmsnorm_gemm(const float* x, const void* gamma, float eps, const void* W, int64_t ldw, void* C,
                              int64_t ldc, int32_t c_dtype, int64_t M, int64_t N, int64_t K, void* ws,
                              size_t ws_bytes, cudaStream_t s) {
  if (!x || !gamma || !ws) return fail(BI_ERR_INVALID_ARG, "gemm_rmsnorm: null pointer");
  bi_status st = check_args(ws, K, W, ldw, C, ldc, c_dtype, M, N, K);
  if (st != BI_OK) return st;
  if (c_dtype == BI_F32_ADD) return fail(BI_ERR_INVALID_ARG, "gemm_rmsnorm: c_dtype must be BI_BF16 or BI_F32");
  if (EPI == EPI_SWIGLU && c_dtype != BI_BF16) return fail(BI_ERR_INVALID_ARG, "gemm_rmsnorm_swiglu: output is bf16");
  if (K <= 0 || K > 32768) return fail(BI_ERR_SHAPE, "gemm_rmsnorm: K (the normed width) must be 8 .. 32768");
  if (!aligned16(x) || !aligned16(gamma)) return fail(BI_ERR_ALIGN, "gemm_rmsnorm: x and gamma must be 16-byte aligned");
  if (!(eps >= 0.0f)) return fail(BI_ERR_INVALID_ARG, "gemm_rmsnorm: eps must be >= 0");
  if (ws_bytes < fold_ws_bytes(M, K)) return fail(BI_ERR_WORKSPACE, "gemm_rmsnorm: workspace %zu < %zu", ws_bytes,
                                                  fold_ws_bytes(M, K));
  if (M == 0 || N == 0) return BI_OK;
  if ((st = require_sm100()) != BI_OK) return st;
  float* r = static_cast<float*>(ws);
  bf16* h = reinterpret_cast<bf16*>(static_cast<uint8_t*>(ws) + (((size_t)M * 4 + 255) & ~(size_t)255));
  int slots = 0;
  if ((st = pair_slots<1, EPI, bf16, true>(&slots)) != BI_OK) return st;
  const int64_t cols_per_tile = EPI == EPI_SWIGLU ? BN / 2 : BN;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + cols_per_tile - 1) / cols_per_tile);
  if (tiles <= slots) {
    if ((st = rmsnorm_scales_f32(x, M, K, eps, r, s)) != BI_OK) return st;
    const FoldArgs fa{x, K, r, gamma};
    return launch<1, EPI, bf16, true>(nullptr, nullptr, K, W, ldw, C, ldc, c_dtype, M, N, K, s, nullptr, &fa);
  }
  if ((st = bi_rmsnorm_f32in(x, gamma, h, M, K, eps, s)) != BI_OK) return st;
  return launch<1, EPI, bf16>(h, nullptr, K, W, ldw, C, ldc, c_dtype, M, N, K, s);
}
}  // namespace gemm
}  // namespace bi

extern "C" bi_status bi_gemm_rmsnorm_workspace_size(int64_t M, int64_t K, size_t* bytes) {
  if (!bytes || M < 0 || K < 0) return fail(BI_ERR_INVALID_ARG, "gemm_rmsnorm_workspace_size: bad arguments");
  *bytes = gemm::fold_ws_bytes(M, K);
  return BI_OK;
}

extern "C" bi_status bi_gemm_rmsnorm(const float* x, const void* gamma, float eps, const void* W, int64_t ldw,
                                     void* C, int64_t ldc, int32_t c_dtype, int64_t M, int64_t N, int64_t K,
                                     void* ws, size_t ws_bytes, void* stream) {
  return gemm::rmsnorm_gemm<gemm::EPI_STORE>(x, gamma, eps, W, ldw, C, ldc, c_dtype, M, N, K, ws, ws_bytes,
                                             static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_gemm_rmsnorm_swiglu(const float* x, const void* gamma, float eps, const void* W,
                                            int64_t ldw, void* out, int64_t ldo, int64_t M, int64_t F, int64_t K,
                                            void* ws, size_t ws_bytes, void* stream) {
  if (F > (1ll << 29)) return fail(BI_ERR_SHAPE, "gemm_rmsnorm_swiglu: F above 2^29");
  return gemm::rmsnorm_gemm<gemm::EPI_SWIGLU>(x, gamma, eps, W, ldw, out, ldo, BI_BF16, M, F, K, ws, ws_bytes,
                                              static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_gemm(const void* A, int64_t lda, const void* W, int64_t ldw, void* C,
                             int64_t ldc, int32_t c_dtype, int64_t M, int64_t N, int64_t K,
                             void* stream) {
  return gemm_e16<bf16>(A, lda, W, ldw, C, ldc, c_dtype, M, N, K, static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_gemm_f16(const void* A, int64_t lda, const void* W, int64_t ldw, void* C,
                                 int64_t ldc, int32_t c_dtype, int64_t M, int64_t N, int64_t K,
                                 void* stream) {
  return gemm_e16<f16>(A, lda, W, ldw, C, ldc, c_dtype, M, N, K, static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_gemm_swiglu(const void* A, int64_t lda, const void* W, int64_t ldw, void* out,
                                    int64_t ldo, int64_t M, int64_t F, int64_t K, void* stream) {
  return gemm_swiglu_e16<bf16>(A, lda, W, ldw, out, ldo, M, F, K, static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_gemm_qkv(const void* A, int64_t lda, const void* W, int64_t ldw, void* qkv,
                                 int64_t ldq, int64_t M, int64_t K, int32_t n_q_heads,
                                 int32_t n_kv_heads, const int32_t* positions, const float* cos_sin,
                                 int32_t max_pos, const int32_t* slot_mapping, void* k_cache,
                                 void* v_cache, int32_t num_pages, void* stream) {
  return gemm_qkv_e16<bf16>(A, lda, W, ldw, qkv, ldq, M, K, n_q_heads, n_kv_heads, positions, cos_sin, max_pos,
                            slot_mapping, k_cache, v_cache, num_pages, static_cast<cudaStream_t>(stream));
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
    return gemm::launch<2, gemm::EPI_ADD, bf16>(A_hi, A_lo, lda, W, ldw, C, ldc, c_dtype, M, N, K,
                                          static_cast<cudaStream_t>(stream));
  return gemm::launch<2, gemm::EPI_STORE, bf16>(A_hi, A_lo, lda, W, ldw, C, ldc, c_dtype, M, N, K,
                                          static_cast<cudaStream_t>(stream));
}
