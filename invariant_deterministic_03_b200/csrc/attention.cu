// attention.cu -- batch-invariant paged attention (decode and chunked
// prefill share every instruction of the per-row arithmetic).
//
// "Defeating Nondeterminism in LLM Inference", section "Batch-invariant
// attention":
//  - parallelise over queries (FlashAttention-2 style) and reduce over the
//    keys inside one core;
//  - the reduction order of a query must be the same whether its sequence is
//    processed whole, in chunks, or one token at a time (query 1000 with 0 or
//    999 cached tokens): keys are always read from the paged cache, which is
//    updated BEFORE this kernel, and walked in 128-key tiles at ABSOLUTE key
//    offsets (multiples of 128 from key 0);
//  - decode needs a split reduction over the keys (Split-KV / FlashDecoding).
//    Here a split is a fixed SIZE of 512 keys at absolute offsets, so a query
//    at position p always uses splits 0 .. p/512, and a separate finishing
//    pass merges them in split order (section "When are atomic adds
//    needed?": split reduction plus a serial finishing reduction).
//
// Split kernel: persistent, one CTA per SM, working through items (split s,
// sequence b, query block, kv head g) claimed at run time. The CTA's 128 MMA
// rows are (query, q head of group g) pairs. Per 128-key tile:
//   S  = Q K^T            tcgen05.mma M128 N128 K16 x8, fp32 in tensor memory
//   per row: m' = the row's reference maximum (log2 domain; see
//        new_reference), alpha = 2^(m-m'), P_j = r16(2^(s_j - m')) (r16:
//        rounding to the 16-bit element type), and for each 32-key quarter q
//        l_q = alpha*l_q + (the quarter's P_j summed left to right)
//   O  = alpha*O          in tensor memory (skipped when alpha == 1)
//   O += P V              tcgen05.mma M128 N128 K16 x8 (one 16-key page per MMA),
//                         O accumulated in tensor memory
// At the end of a split the unnormalised O, m and l = ((l_0 + l_1) + l_2) +
// l_3 go to the workspace. Decode (one query per item) and prefill (chunks)
// run exactly this arithmetic per row, in two layouts of the softmax work.
// A row takes part only in tiles whose first key is <= its position, so the
// update sequence of a row is a function of (position, split) alone.
// Masked keys get P = 0 by selection (never by arithmetic on -inf), and
// cache slots at or past the sequence length are zeroed in shared memory so
// that stale cache contents cannot reach the P.V products.
//
// Each (page, kv head) block of the cache is stored in the tensor core's
// canonical K-major no-swizzle order (8 x 16-byte core matrices), so a tile is
// 8 + 8 contiguous 4 KB bulk copies straight into MMA operand layout.
#include <mutex>

#include "common.cuh"
#include "host.h"

namespace bi {
namespace attn {

constexpr int HD = BI_HEAD_DIM;        // 128
constexpr int TILE = BI_ATTN_TILE;     // 128 keys
constexpr int SPLIT = BI_ATTN_SPLIT;   // 512 keys
constexpr int PAGE = BI_PAGE_SIZE;     // 16 keys
constexpr int PAGES_PER_TILE = TILE / PAGE;
constexpr uint32_t TILE_BYTES = 128 * 128 * 2;  // 32 KB: one K or V tile (128 keys x 128 d)
constexpr int ITEM_RING = 16;                   // claimed work items in flight inside a CTA

// Shared-memory layout. Prefill: Q and P are full 128-row tiles; two Q
// buffers (the next item's Q loads while the current item runs), one P
// buffer, two K and two V buffers (seven 32 KB tiles fill the 227 KB: two Q
// and two V measured 1.6 % faster than one Q and three V, one Q and three V
// ~2 % faster than one Q, three K and two V, and a second P buffer in place
// of the third V gained nothing). Decode: the MMA rows that matter are the G <= 8
// head rows of one query, so Q and P keep just one 8-row core-matrix group
// per 64-column half and the MMA operand descriptor repeats it for all 16
// groups (8-row-group stride 0): the same 128-row MMA reads the same values
// in every row that matters, and the ~90 KB saved buy a third K and a third
// V buffer and a second P buffer (so the softmax of tile j+1 can store its P
// while the P V product of tile j still runs); decode keeps two compact Q
// buffers.
template <bool DECODE>
struct Lay {
  static constexpr int NK = DECODE ? 3 : 2;                 // K tile buffers
  static constexpr int NQ = 2;                              // Q buffers
  static constexpr int NV = DECODE ? 3 : 2;                 // V tile buffers
  static constexpr int NP = DECODE ? 2 : 1;                 // P buffers
  static constexpr int NS = DECODE ? 3 : 2;                 // S buffers in tensor memory
  static constexpr int SOFTMAX_WARPS = DECODE ? 4 : 16;     // one 32-key quarter of 32 rows each
  static constexpr int SOFTMAX_THREADS = SOFTMAX_WARPS * 32;
  static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;       // then the MMA / tensor-memory warp, the scheduler warp
  static constexpr int THREADS = SOFTMAX_THREADS + 96;
  static constexpr uint32_t HALF = DECODE ? 1024 : 16384;   // bytes between the 64-column halves of Q / P
  static constexpr uint32_t ROW_SBO = DECODE ? 0 : 1024;    // bytes between 8-row groups of Q / P
  static constexpr uint32_t QP_BYTES = 2 * HALF;            // one Q or P buffer
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + NK * TILE_BYTES;
  static constexpr uint32_t OFF_Q = OFF_V + NV * TILE_BYTES;  // NQ buffers
  static constexpr uint32_t OFF_P = OFF_Q + NQ * QP_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + NP * QP_BYTES;
  static constexpr uint32_t OFF_RING = OFF_BAR + 256;   // producer's page-id ring [16 tiles][8 pages]
  static constexpr uint32_t OFF_RED = OFF_RING + 512;   // decode quarter exchange [2 slots][4 warps][8 heads] fp32
  static constexpr uint32_t OFF_ITEMS = OFF_RED + (DECODE ? 256 : 0);  // item ring [16] x 48 B, then one mbarrier per slot
  static constexpr size_t SMEM_BYTES = 1024 + OFF_ITEMS + ITEM_RING * 48 + ITEM_RING * 8;
  static_assert(NK + NV <= 6, "barrier area holds six K / V buffers");
  static_assert(OFF_Q % 1024 == 0 && OFF_P % 1024 == 0, "swizzled Q / P tiles need 1 KB alignment");
  static_assert(SMEM_BYTES <= 232448, "attention: shared memory above the 227 KB per-CTA limit");
};
// Warps 0 .. SOFTMAX_WARPS-1: softmax, O rescale and partials (one 32-key
// quarter of 32 MMA rows per warp); then the TMA producer warp, the
// tensor-memory allocator and MMA issuer warp, and the scheduler warp.
// Tensor memory: S buffers at columns [0,128), [128,256) and (decode)
// [256,384); in prefill columns [256,264) carry the quarter exchange; O at
// [384,512).
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_X = 256;
constexpr uint32_t TMEM_O = 384;

struct Params {
  const uint8_t* kc;  // 16-bit key cache, 4 KB per (page, kv head) block
  const uint8_t* vc;  // 16-bit value cache, same blocking
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* cu_q;  // null: decode (one query per sequence, row b)
  float* ws_o;          // [n_tok, Hq, n_split_max, 128]
  float* ws_ml;         // [n_tok, Hq, n_split_max, 2]
  int32_t B, Hq, Hkv, G, QR, qblocks, q_box, n_tok;
  int32_t num_pages, max_pages, max_kv_len, n_split_max;
  int32_t total_items;
  int32_t* work_counter;  // next unclaimed work item (zeroed before the launch)
  float scale_log2;
  int32_t* status;
  int32_t ws_wide;  // ws_o is 32-byte aligned: partial rows go out in 256-bit stores
};

// One unit of work: (split s, sequence b, query block, kv head g).
struct Item {
  int s, b, g, r0, nb, L, q_lo, q_hi, key_lo, t0, ntiles;
};

// An entry of the shared item ring: the claimed index (-1: no more work) and
// its decoded coordinates, so that no role repeats the global loads of item_at.
struct RingItem {
  int32_t idx;
  Item it;
};
static_assert(sizeof(RingItem) == 48, "item ring entry");

// Work item idx -> its coordinates; false when it has nothing to do. The kv
// head varies fastest and the split slowest, so the persistent CTAs first take
// every sequence's first split and empty items gather at the end.
__device__ __forceinline__ bool item_at(const Params& p, int idx, Item& it, bool report) {
  it.g = idx % p.Hkv;
  int rest = idx / p.Hkv;
  it.b = rest % p.B;
  rest /= p.B;
  const int jb = rest % p.qblocks;
  it.s = rest / p.qblocks;
  it.L = p.seq_lens[it.b];
  if (p.cu_q) {
    it.r0 = p.cu_q[it.b];
    it.nb = p.cu_q[it.b + 1] - it.r0;
  } else {
    it.r0 = it.b;
    it.nb = 1;
  }
  // a chunk with more rows than max_q_len (the grid covers max_q_len rows)
  if (report && jb == 0 && it.s == 0 && it.g == 0 && it.nb > p.qblocks * p.QR)
    set_status(p.status, BI_DEV_BAD_SEQLEN);
  if (it.nb <= 0 || jb * p.QR >= it.nb) return false;
  if (it.L < it.nb || it.L > p.max_kv_len || it.r0 < 0 || it.r0 + it.nb > p.n_tok) {
    if (report && it.s == 0 && jb == 0 && it.g == 0) set_status(p.status, BI_DEV_BAD_SEQLEN);
    return false;
  }
  it.q_lo = jb * p.QR;
  it.q_hi = min(it.nb, it.q_lo + p.QR);
  const int p_last = it.L - it.nb + it.q_hi - 1;
  it.key_lo = it.s * SPLIT;
  if (it.key_lo > p_last) return false;
  const int key_hi = min((it.s + 1) * SPLIT, p_last + 1);  // exclusive
  it.t0 = it.key_lo / TILE;
  it.ntiles = (key_hi - 1) / TILE - it.t0 + 1;
  return true;
}

// A zero (page, head) block: the source for pages past a sequence's end (and
// for bad page ids), so the masked keys of a tile always meet zero values.
__device__ __align__(128) uint8_t g_attn_zero_block[4096];

constexpr uint32_t BLOCK_BYTES = PAGE * HD * 2;  // 4 KB: one (page, kv head) block

// Page id of page i (0..7) of one 128-key tile, looked up in the sequence's
// block table; -1 marks a page past the sequence end or a bad id. The entry
// is read unconditionally at a clamped index (always inside the row), so the
// load can be issued early and validated later (page_valid).
__device__ __forceinline__ int32_t tile_page_raw(const Params& p, int b, int tile, int i) {
  return p.block_table[(size_t)b * p.max_pages + min(tile * PAGES_PER_TILE + i, p.max_pages - 1)];
}

__device__ __forceinline__ int32_t page_valid(const Params& p, int L, int tile, int i, int32_t pid) {
  const int pidx = tile * PAGES_PER_TILE + i;
  const bool in_seq = pidx * PAGE < L;
  const bool ok = in_seq && pidx < p.max_pages && pid >= 0 && pid < p.num_pages;
  if (in_seq && !ok) set_status(p.status, BI_DEV_BAD_PAGE);
  return ok ? pid : -1;
}

__device__ __forceinline__ const uint8_t* block_src(const uint8_t* cache, int32_t pid, int Hkv,
                                                    int g) {
  return pid < 0 ? g_attn_zero_block : cache + ((size_t)pid * Hkv + g) * BLOCK_BYTES;
}

// Work items are claimed at run time: the scheduler warp takes the next
// index from a global counter (atomicAdd -- scheduling only, no value is ever
// reduced through it), skips items with no work, and publishes each claimed
// item, decoded (or -1 at the end), in a shared ring with one mbarrier per
// slot; every other role walks the ring in order. Which CTA runs an item
// never reaches its arithmetic.
__device__ __forceinline__ int claim_item(const Params& p, int lane, Item& it) {
  while (true) {
    int v = 0;
    if (lane == 0) v = atomicAdd(p.work_counter, 1);
    v = __shfl_sync(0xffffffffu, v, 0);
    if (v >= p.total_items) return -1;
    if (item_at(p, v, it, true)) return v;
  }
}

// Walks the (item, tile) sequence of this CTA through the item ring.
struct Cursor {
  int n, t;  // ring sequence number of the current item, tile within it
  Item it;
  bool valid;
};

// Advances to the next tile; on a new item, reads ring entry n (waiting for
// its publication). Returns false only when a wait timed out.
// Ring entry n once published (waits for it): false when the wait timed out.
__device__ __forceinline__ bool ring_read(const Params& p, const RingItem* ring, uint64_t* ibar, int n,
                                          volatile int* abort_flag, int& idx, Item& it) {
  const int slot = n & (ITEM_RING - 1);
  if (!mbar_wait(&ibar[slot], ((uint32_t)n / ITEM_RING) & 1u, p.status, abort_flag)) return false;
  const volatile int32_t* e = reinterpret_cast<const volatile int32_t*>(&ring[slot]);
  idx = e[0];
  int* dst = reinterpret_cast<int*>(&it);
#pragma unroll
  for (int i = 0; i < 11; ++i) dst[i] = e[1 + i];
  return true;
}

__device__ __forceinline__ bool cursor_next(const Params& p, Cursor& c, const RingItem* ring,
                                            uint64_t* ibar, volatile int* abort_flag) {
  if (c.valid && ++c.t < c.it.ntiles) return true;
  c.valid = false;
  c.t = 0;
  ++c.n;
  int idx;
  if (!ring_read(p, ring, ibar, c.n, abort_flag, idx, c.it)) return false;
  c.valid = idx >= 0;
  return true;
}

__device__ __forceinline__ bool cursor_start(const Params& p, Cursor& c, const RingItem* ring,
                                             uint64_t* ibar, volatile int* abort_flag) {
  c.n = -1;
  c.t = 0;
  c.valid = false;
  return cursor_next(p, c, ring, ibar, abort_flag);
}

constexpr int PF_AHEAD = 4;     // page-table lookups run this many tiles ahead of the K loads
constexpr int PF_RING = 16;     // looked-up page ids, from the oldest V load to the newest lookup
constexpr int SCHED_AHEAD = 1;  // ring entries the scheduler publishes ahead of the page look-ahead
static_assert(PF_RING * 8 * 4 <= 512, "page-id ring overflows its region");
// Ring bounds. With j the tile the softmax is on: S(n) is issued only once
// the softmax has read S(n - NS), K(n) only once S(n - NK) is done, and the
// look-ahead is PF_AHEAD tiles past the K copies, so it is at most NS + NK +
// PF_AHEAD tiles past j; the softmax passes tile j only after the P V of
// tile j - NP was issued, so every V copy up to j - NP + 1 is out. Every role
// reads its items from the ring in order and every item has a tile, so from
// the slowest reader to the look-ahead there are at most NS + NK + PF_AHEAD +
// NP - 1 tiles (11 in decode, 8 in prefill), and the scheduler adds
// SCHED_AHEAD entries; both rings hold 16.
template <bool DECODE>
constexpr bool rings_fit() {
  using L = Lay<DECODE>;
  return L::NS + L::NK + PF_AHEAD + L::NP - 1 + SCHED_AHEAD <= ITEM_RING &&
         L::NS + L::NK + PF_AHEAD + L::NP - 1 < PF_RING;
}
static_assert(rings_fit<true>() && rings_fit<false>(), "item or page-id ring too small for the look-ahead");

// S = Q K^T. Q: 128 rows x 128 d, 128-byte swizzle in two 64-column halves.
// K: 8 page blocks of 16 keys, canonical no-swizzle K-major: core matrices of
// 8 keys x 8 d (128 B), d-chunks 128 B apart (LBO), 8-key groups 2 KB apart
// (SBO, uniform across the blocks of a tile).
template <bool DECODE, typename ET>
__device__ __forceinline__ void issue_s(uint32_t tmem_s, uint32_t q_addr, uint32_t k_addr) {
  using L = Lay<DECODE>;
  constexpr uint32_t idesc = idesc_f32acc(128, 128, E16<ET>::kMmaFormat);
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t qoff = (kk >> 2) * L::HALF + (kk & 3) * 32;
    mma_f16k(tmem_s, smem_desc(q_addr + qoff, 16, L::ROW_SBO, 2), smem_desc(k_addr + kk * 256, 128, 2048, 0),
             idesc, kk != 0);
  }
}

// O (+)= P V: accumulate = 0 on the first tile of a split, 1 after.
template <bool DECODE, typename ET>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t p_addr, uint32_t v_addr,
                                         bool accumulate) {
  using L = Lay<DECODE>;
  constexpr uint32_t idesc = idesc_f32acc(128, 128, E16<ET>::kMmaFormat);
#pragma unroll
  for (int j = 0; j < PAGES_PER_TILE; ++j) {
    const uint32_t poff = (j >> 2) * L::HALF + (j & 3) * 32;
    // V page block j (16 keys = one K step): canonical no-swizzle K-major with
    // rows = d: core matrices of 8 d x 8 keys, key-chunks 128 B apart (LBO),
    // 8-d groups 256 B apart (SBO).
    mma_f16k(tmem_o, smem_desc(p_addr + poff, 16, L::ROW_SBO, 2),
             smem_desc(v_addr + j * BLOCK_BYTES, 128, 256, 0), idesc, (accumulate || j != 0) ? 1u : 0u);
  }
}

// 2^x by the hardware approximation (ex2.approx.ftz: relative error below
// 2^-22, results under 2^-126 flushed to zero). Used identically by every row.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One quarter (32 keys) of a row's tile: P_c = r16(2^(S_c * scale_log2 -
// m)) for c < nvalid (else 0), r16 the rounding to the 16-bit element type,
// packed two per word into P[0..15], and the quarter sum of the rounded
// values, added left to right. P may alias S[0..15]: word c2 of P is written
// after S[2 c2] and S[2 c2 + 1], the last elements it depends on, are read. Decode and prefill both build a row from
// exactly these quarters, so their arithmetic is the same.
template <typename ET>
__device__ __forceinline__ float quarter_p(const uint32_t (&S)[32], int nvalid, float neg_m,
                                           float scale_log2, uint32_t (&P)[16]) {
  float q = 0.0f;
#pragma unroll
  for (int c2 = 0; c2 < 16; ++c2) {
    // every element is evaluated and masked ones are replaced by zero with a
    // select, so no branch serialises the loop
    const float e0 = ex2_approx(__fmaf_rn(__uint_as_float(S[2 * c2]), scale_log2, neg_m));
    const float e1 = ex2_approx(__fmaf_rn(__uint_as_float(S[2 * c2 + 1]), scale_log2, neg_m));
    const uint32_t pk = E16<ET>::pack2(2 * c2 < nvalid ? e0 : 0.0f, 2 * c2 + 1 < nvalid ? e1 : 0.0f);
    q = __fadd_rn(q, E16<ET>::lo(pk));  // rounded element 2*c2
    q = __fadd_rn(q, E16<ET>::hi(pk));  // rounded element 2*c2+1
    P[c2] = pk;
  }
  return q;
}

// The row's reference maximum for tile t (log2 domain), given the previous
// reference m and this tile's scaled maximum: the first tile of a split takes
// its maximum; a later tile keeps m unless the new maximum exceeds it by more
// than 2^RESCALE_LOG2 (then P values stay below 2^8, exact to bf16 like any
// others, and O and l need no rescale, so the softmax of the next tile rarely
// waits for the P V of this one). The choice depends on the row's own values
// only, and decode and prefill make it identically; the split's final O / l
// (and the merge, which takes each split's m as its reference) do not depend
// on which reference was used beyond rounding.
constexpr float RESCALE_LOG2 = 8.0f;
__device__ __forceinline__ float new_reference(float m, float tile_max, int t) {
  const float mc = fmaxf(m, tile_max);
  return (t > 0 && __fsub_rn(mc, m) <= RESCALE_LOG2) ? m : mc;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// The maximum of a quarter's first nvalid scores (-inf when none), by a tree
// of three-input maxima (17 operations, depth 4, instead of a 32-long chain):
// max is exact, so any order gives the same value for non-NaN scores; masked
// keys enter as -inf. With nvalid = 32 (a constant) no select is left.
__device__ __forceinline__ float quarter_max(const uint32_t (&S)[32], int nvalid) {
  float v[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) v[c] = c < nvalid ? __uint_as_float(S[c]) : -INFINITY;
  float a[11];
#pragma unroll
  for (int k = 0; k < 10; ++k) a[k] = max3(v[3 * k], v[3 * k + 1], v[3 * k + 2]);
  a[10] = fmaxf(v[30], v[31]);
  const float b0 = max3(a[0], a[1], a[2]), b1 = max3(a[3], a[4], a[5]), b2 = max3(a[6], a[7], a[8]);
  const float b3 = fmaxf(a[9], a[10]);
  return fmaxf(max3(b0, b1, b2), b3);
}

// P row `row`, keys 32*quarter .. +31, into the 128-byte-swizzled P tile whose
// two 64-key halves lie `half` bytes apart.
__device__ __forceinline__ void store_p_chunks(uint8_t* p_smem, uint32_t half, int row, int quarter,
                                               const uint32_t (&P)[16]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int chunk = quarter * 4 + k;  // 8 keys per 16-byte chunk
    const uint32_t addr = (uint32_t)(chunk >> 3) * half + (uint32_t)row * 128u +
                          (uint32_t)(((chunk & 7) ^ (row & 7)) << 4);
    *reinterpret_cast<uint4*>(p_smem + addr) = make_uint4(P[4 * k], P[4 * k + 1], P[4 * k + 2], P[4 * k + 3]);
  }
}

// Bounded wait for the fills a producer issued into a buffer, so that no copy
// is still landing in shared memory when an aborted CTA exits.
__device__ __forceinline__ void drain(uint64_t* bar, int fills) {
  if (fills <= 0) return;
  const uint32_t parity = (uint32_t)(fills - 1) & 1u;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 < kWaitLimitCycles) {
  }
}

// Split kernel. Persistent: one CTA per SM takes work items as they are
// claimed at run time (claim_item); the three roles walk the same item
// sequence through the shared item ring.
// Tiles j are counted across items. The producer keeps K and V loads apart
// (a K buffer is free once its QK^T is done, a V buffer once its PV is done)
// and the MMA warp issues S(j) = Q K_j^T and O += P_j V_j as soon as each is
// ready, so loads, QK^T and the softmax of neighbouring tiles overlap.
// DECODE selects the softmax layout (see below); both layouts run the same
// per-row arithmetic.
//
// Row arithmetic (fixed order, the same in decode and prefill):
//   first tile of the split:  m = max_j s_j (log2 domain, s_j = S_ij * scale*log2e),
//                             P_j = r16(2^(s_j - m)), l_q = sum_{j in quarter q} P_j, O = P V
//   later tiles:              c = max(m, max_j s_j); m' = m if c - m <= 8 else c
//                             (new_reference), alpha = 2^(m - m'),
//                             P_j = r16(2^(s_j - m')), l_q = alpha*l_q + sum_{j in q} P_j,
//                             O = alpha*O (fp32, skipped when alpha == 1), O += P V (MMA)
//   end of the split:         l = ((l_0 + l_1) + l_2) + l_3
// sums over j run left to right inside each 32-key quarter; masked keys have
// P_j = 0 by selection.
template <bool DECODE, typename ET>
__global__ void __launch_bounds__(Lay<DECODE>::THREADS, 1)
    attn_split_kernel(const __grid_constant__ CUtensorMap tmQ, const Params p) {
  using L = Lay<DECODE>;
  constexpr int NK = L::NK, NV = L::NV;
  constexpr uint32_t OFF_Q = L::OFF_Q, OFF_K = L::OFF_K, OFF_V = L::OFF_V, OFF_P = L::OFF_P;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars + 0;                // [2]
  uint64_t* q_empty = bars + 2;               // [2]
  uint64_t* k_full = bars + 4;                // [NK]
  uint64_t* k_empty = k_full + NK;            // [NK]
  uint64_t* v_full = k_empty + NK;            // [NV]
  uint64_t* v_empty = v_full + NV;            // [NV]
  uint64_t* s_full = bars + 16;               // [NS]
  uint64_t* s_free = bars + 19;               // [NS]
  uint64_t* p_ready = bars + 22;              // [NP]
  uint64_t* o_ready = bars + 24;              // [NP]: P V of the tile that read P buffer i is done
  uint64_t* x_bar = bars + 26;                // quarter exchange: decode [1], prefill [4] (one per lane group)
  static_assert(4 + 2 * (NK + NV) <= 16, "K / V barriers overlap the S barriers");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 30);
  // ring entry (item) the producer's page look-ahead is on; the scheduler stays
  // at most SCHED_AHEAD entries in front of it
  volatile int* pf_item = reinterpret_cast<volatile int*>(bars + 31);
  static_assert(32 * 8 <= 256, "barrier region");
  RingItem* item_ring = reinterpret_cast<RingItem*>(smem + L::OFF_ITEMS);
  uint64_t* item_bar = reinterpret_cast<uint64_t*>(smem + L::OFF_ITEMS + ITEM_RING * 48);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < L::NS; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], L::SOFTMAX_THREADS);
    }
    for (int i = 0; i < NK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < L::NP; ++i) {
      mbar_init(&p_ready[i], L::SOFTMAX_THREADS);
      mbar_init(&o_ready[i], 1);
    }
    for (int i = 0; i < (DECODE ? 1 : 4); ++i) mbar_init(&x_bar[i], 128);
    for (int i = 0; i < ITEM_RING; ++i) mbar_init(&item_bar[i], 1);
    *abort_flag = 0;
    *pf_item = -1;
    fence_barrier_init();
  }
  if (warp == L::PRODUCER_WARP + 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == L::PRODUCER_WARP) {
    // ------------------------------------------------ producer warp
    // Lane 0 owns the barriers and the Q loads; lanes 0..7 each own one page
    // of a tile: its block-table entry is fetched PF_AHEAD tiles early by
    // cp.async into the page-id ring (one commit group per tile), checked
    // when the tile's K copies are issued, and each lane issues its page's
    // 4 KB copy, so a tile's eight copies go out together. All lanes walk
    // the same cursors (kc: K copies, vc: V copies, pf: page look-ahead).
    if (lane == 0) prefetch_tmap(&tmQ);
    const uint32_t q_bytes = 2u * 64u * 2u * (uint32_t)(p.G * p.q_box);
    int32_t* ring = reinterpret_cast<int32_t*>(smem + L::OFF_RING);  // [PF_RING][8]
    // lanes 0..7: the block-table entries of the pf cursor's tile into a ring slot
    auto lookup_pages = [&](const Cursor& c, int32_t* slot) {
      if (lane < PAGES_PER_TILE) {
        const int i = min((c.it.t0 + c.t) * PAGES_PER_TILE + lane, p.max_pages - 1);
        cp_async4(slot + lane, p.block_table + (size_t)c.it.b * p.max_pages + i);
      }
    };
    Cursor kc, vc, pf;
    bool ok = cursor_start(p, pf, item_ring, item_bar, abort_flag);
    if (lane == 0) *pf_item = pf.n;
    if (ok) ok = cursor_start(p, kc, item_ring, item_bar, abort_flag);
    vc = kc;
    int nk = 0, nv = 0, npf = 0, qi = 0;
    for (int i = 0; i < PF_AHEAD; ++i) {  // the first PF_AHEAD tiles' lookups
      if (ok && pf.valid) {
        lookup_pages(pf, ring + (npf & (PF_RING - 1)) * 8);
        ++npf;
        if (!cursor_next(p, pf, item_ring, item_bar, abort_flag)) ok = false;
        if (lane == 0) *pf_item = pf.n;
      }
      cp_async_commit();  // one group per tile slot, empty past the last tile
    }
    long long t_last = clock64();
    while ((kc.valid || vc.valid) && ok) {
      bool progressed = false;
      if (kc.valid) {
        const int kb = nk % NK, qb = L::NQ == 2 ? (qi & 1) : 0;
        const uint32_t qpar = L::NQ == 2 ? (((uint32_t)qi >> 1) & 1u) : ((uint32_t)qi & 1u);
        int ready = 0;
        if (lane == 0) {
          ready = mbar_test(&k_empty[kb], (((uint32_t)nk / NK) & 1u) ^ 1u);
          if (ready && kc.t == 0) ready = mbar_test(&q_empty[qb], qpar ^ 1u);
        }
        if (__shfl_sync(0xffffffffu, ready, 0)) {
          if (kc.t == 0) {  // first tile of an item: its Q rows
            if (lane == 0) {
              // both 64-column halves (decode: the G head rows, which the
              // MMA descriptor repeats over all 128 rows)
              uint8_t* qdst = smem + OFF_Q + qb * L::QP_BYTES;
              mbar_arrive_expect_tx(&q_full[qb], q_bytes);
              tma_load_3d(qdst, &tmQ, &q_full[qb], 0, kc.it.g * p.G, kc.it.r0 + kc.it.q_lo);
              tma_load_3d(qdst + L::HALF, &tmQ, &q_full[qb], 64, kc.it.g * p.G, kc.it.r0 + kc.it.q_lo);
            }
            ++qi;
          }
          // this tile's lookups (committed PF_AHEAD groups ago) have landed
          cp_async_wait<PF_AHEAD - 1>();
          int32_t* kslot = ring + (nk & (PF_RING - 1)) * 8;
          int32_t pid = -1;
          if (lane < PAGES_PER_TILE) {
            pid = page_valid(p, kc.it.L, kc.it.t0 + kc.t, lane, kslot[lane]);
            kslot[lane] = pid;  // the checked id, for this tile's V copy
          }
          if (pf.valid) {  // keep the lookups PF_AHEAD tiles ahead
            lookup_pages(pf, ring + (npf & (PF_RING - 1)) * 8);
            ++npf;
            if (!cursor_next(p, pf, item_ring, item_bar, abort_flag)) ok = false;
            if (lane == 0) *pf_item = pf.n;
          }
          cp_async_commit();
          if (lane == 0) mbar_arrive_expect_tx(&k_full[kb], TILE_BYTES);
          __syncwarp();
          if (lane < PAGES_PER_TILE)
            bulk_load(smem + OFF_K + kb * TILE_BYTES + lane * BLOCK_BYTES, block_src(p.kc, pid, p.Hkv, kc.it.g),
                      BLOCK_BYTES, &k_full[kb]);
          ++nk;
          if (!cursor_next(p, kc, item_ring, item_bar, abort_flag)) ok = false;
          progressed = true;
        }
      }
      if (vc.valid && nv < nk) {
        const int vb = nv % NV;
        int ready = 0;
        if (lane == 0) ready = mbar_test(&v_empty[vb], (((uint32_t)nv / NV) & 1u) ^ 1u);
        if (__shfl_sync(0xffffffffu, ready, 0)) {
          if (lane == 0) mbar_arrive_expect_tx(&v_full[vb], TILE_BYTES);
          __syncwarp();
          if (lane < PAGES_PER_TILE)
            bulk_load(smem + OFF_V + vb * TILE_BYTES + lane * BLOCK_BYTES,
                      block_src(p.vc, ring[(nv & (PF_RING - 1)) * 8 + lane], p.Hkv, vc.it.g), BLOCK_BYTES,
                      &v_full[vb]);
          ++nv;
          if (!cursor_next(p, vc, item_ring, item_bar, abort_flag)) ok = false;
          progressed = true;
        }
      }
      int stop = 0;
      if (lane == 0) {
        if (progressed) {
          t_last = clock64();
        } else if (__nanosleep(32), *abort_flag) {
          stop = 1;
        } else if (clock64() - t_last > kWaitLimitCycles) {
          set_status(p.status, BI_DEV_WAIT_TIMEOUT);
          *abort_flag = 1;
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) ok = false;
    }
    cp_async_wait<0>();  // no lookup still landing in shared memory
    if (!ok && lane == 0) {
      // buffer i of a ring of nb took the copies numbered i, i + nb, ... below the count
      auto fills = [](int count, int i, int nb) { return (count - i + nb - 1) / nb; };
      for (int i = 0; i < L::NQ; ++i) drain(&q_full[i], fills(qi, i, L::NQ));
      for (int i = 0; i < NK; ++i) drain(&k_full[i], fills(nk, i, NK));
      for (int i = 0; i < NV; ++i) drain(&v_full[i], fills(nv, i, NV));
    }
  } else if (warp == L::PRODUCER_WARP + 2) {
    // ------------------------------------------------ scheduler warp
    // Claims work items (claim_item) and publishes each, decoded, as the next
    // ring entry (the end marker -1 last), at most SCHED_AHEAD entries in
    // front of the one the producer's page look-ahead is on: the claim's
    // atomic and the item's global loads overlap the copies instead of
    // stalling the producer.
    long long t_last = clock64();
    for (int n = 0;; ++n) {
      int go;
      do {  // 0: wait for the look-ahead, 1: claim, 2: stop
        go = 0;
        if (lane == 0) {
          if (n <= *pf_item + SCHED_AHEAD) {
            go = 1;
          } else if (*abort_flag) {
            go = 2;
          } else if (clock64() - t_last > kWaitLimitCycles) {
            set_status(p.status, BI_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
            go = 2;
          } else {
            __nanosleep(64);
          }
        }
        go = __shfl_sync(0xffffffffu, go, 0);
      } while (go == 0);
      if (go == 2) break;
      Item it;
      const int idx = claim_item(p, lane, it);
      if (lane == 0) {
        const int slot = n & (ITEM_RING - 1);
        volatile int32_t* e = reinterpret_cast<volatile int32_t*>(&item_ring[slot]);
        e[0] = idx;
        const int* src = reinterpret_cast<const int*>(&it);
#pragma unroll
        for (int i = 0; i < 11; ++i) e[1 + i] = src[i];
        mbar_arrive(&item_bar[slot]);  // release: the entry is visible to whoever sees the phase
      }
      t_last = clock64();
      if (idx < 0) break;
    }
  } else if (warp == L::PRODUCER_WARP + 1) {
    // ------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      const uint32_t sQ0 = smem_u32(smem + OFF_Q), sK0 = smem_u32(smem + OFF_K);
      const uint32_t sV0 = smem_u32(smem + OFF_V), sP = smem_u32(smem + OFF_P);
      Cursor sc;
      int nS = 0, nP = 0, qi = 0;
      // per issued S tile (bit n & 31): P V accumulates
      uint32_t acc_bits = 0;
      bool ok = cursor_start(p, sc, item_ring, item_bar, abort_flag);
      long long t_last = clock64();
      while ((sc.valid || nP < nS) && ok) {
        bool progressed = false;
        if (sc.valid && nS - nP < L::NS) {
          const int sb = nS % L::NS, kb = nS % NK, qb = L::NQ == 2 ? (qi & 1) : 0;
          const uint32_t qpar = L::NQ == 2 ? (((uint32_t)qi >> 1) & 1u) : ((uint32_t)qi & 1u);
          const bool ready = (sc.t != 0 || mbar_test(&q_full[qb], qpar)) &&
                             mbar_test(&k_full[kb], ((uint32_t)nS / NK) & 1u) &&
                             mbar_test(&s_free[sb], (((uint32_t)nS / L::NS) & 1u) ^ 1u);
          if (ready) {
            tc_fence_after();
            issue_s<DECODE, ET>(tmem + sb * 128, sQ0 + qb * L::QP_BYTES, sK0 + kb * TILE_BYTES);
            mma_commit(&s_full[sb]);
            mma_commit(&k_empty[kb]);
            if (sc.t == sc.it.ntiles - 1) mma_commit(&q_empty[qb]);  // Q is read by QK^T only
            const uint32_t bit = 1u << (nS & 31);
            acc_bits = sc.t > 0 ? (acc_bits | bit) : (acc_bits & ~bit);
            if (sc.t == sc.it.ntiles - 1) ++qi;
            ++nS;
            if (!cursor_next(p, sc, item_ring, item_bar, abort_flag)) ok = false;
            progressed = true;
          }
        }
        if (nP < nS) {
          const int vb = nP % NV, pb = nP % L::NP;
          if (mbar_test(&p_ready[pb], ((uint32_t)nP / L::NP) & 1u) &&
              mbar_test(&v_full[vb], ((uint32_t)nP / NV) & 1u)) {
            const uint32_t bit = 1u << (nP & 31);
            tc_fence_after();
            issue_pv<DECODE, ET>(tmem + TMEM_O, sP + pb * L::QP_BYTES, sV0 + vb * TILE_BYTES, (acc_bits & bit) != 0);
            mma_commit(&o_ready[pb]);
            mma_commit(&v_empty[vb]);
            ++nP;
            progressed = true;
          }
        }
        if (progressed) {
          t_last = clock64();
        } else if (__nanosleep(32), *abort_flag) {
          ok = false;
        } else if (clock64() - t_last > kWaitLimitCycles) {
          set_status(p.status, BI_DEV_WAIT_TIMEOUT);
          *abort_flag = 1;
          ok = false;
        }
      }
    }
  } else {
    // ------------------------------------------------ softmax warps
    // Warp w owns one 32-key quarter of the S and P columns (and the same 32
    // d columns of O) for the 32 MMA rows of its tensor-memory lane group.
    // Prefill: 16 warps; lane group w % 4 (rows 32 (w % 4) .. +31), quarter
    // w / 4; MMA row r = (query r / G, head r % G).
    // Decode (one query per item): 4 warps; the item's G head rows are loaded
    // into rows 32w + i of every lane group (identical rows, identical S), and
    // warp w takes quarter w of every head i < G.
    // The four quarters of a row meet in exchange(): their maxima once per
    // tile and their sums l_q once per split. (In decode a layout in which the
    // four lanes of a head in one warp each take a quarter and combine by
    // shuffles was measured slower: each lane then needs its own column
    // range, four tensor-memory loads per tile instead of one.)
    constexpr bool decode = DECODE;
    const int rg = decode ? warp : (warp & 3);        // tensor-memory lane group
    const int quarter = decode ? warp : (warp >> 2);  // columns 32 quarter .. +31
    const uint32_t lane_off = (uint32_t)(rg * 32) << 16;
    const int r = decode ? lane : rg * 32 + lane;     // prefill: the MMA row
    const int qr = decode ? 0 : r / p.G;
    const int hj = decode ? lane : r - qr * p.G;
    float* red = reinterpret_cast<float*>(smem + L::OFF_RED);  // decode: [2 slots][4 warps][8 head rows]
    uint64_t* xbar = decode ? x_bar : &x_bar[rg];
    int j = 0, xc = 0;
    bool ok = true;
    // waits until the P V product of tile jj (counted across this CTA's items) is done
    auto pv_done = [&](int jj) -> bool {
      if (!mbar_wait(&o_ready[jj % L::NP], ((uint32_t)jj / L::NP) & 1u, p.status, abort_flag)) return false;
      tc_fence_after();
      return true;
    };
    // The four warps that share this thread's row each contribute v, the
    // value of their quarter; x[q] receives quarter q's value for the row.
    // Decode meets in shared memory (its four warps sit in different lane
    // groups), prefill in tensor-memory columns TMEM_X .. +7 of the lane group
    // (shared memory is full). Exchange k uses slot k & 1: a warp can be at
    // most one exchange ahead of another (it passes exchange k + 1 only once
    // every warp has arrived there, i.e. has read exchange k), so two slots
    // keep a fast warp from overwriting values a slow one still reads.
    // False when the wait timed out.
    auto exchange = [&](float v, float (&x)[4]) -> bool {
      const int which = xc & 1;
      if constexpr (decode) {
        if (lane < 8) red[(which * 4 + warp) * 8 + lane] = v;
      } else {
        tmem_st1(tmem + lane_off + TMEM_X + which * 4 + quarter, __float_as_uint(v));
        tmem_st_wait();
        tc_fence_before();
      }
      mbar_arrive(xbar);
      const bool done = mbar_wait(xbar, (uint32_t)xc & 1u, p.status, abort_flag);
      ++xc;
      if (!done) return false;
      if constexpr (decode) {
#pragma unroll
        for (int w = 0; w < 4; ++w) x[w] = red[(which * 4 + w) * 8 + (lane & 7)];
      } else {
        tc_fence_after();
        uint32_t u[4];
        tmem_ld4(tmem + lane_off + TMEM_X + which * 4, u);
        tmem_ld_wait();
#pragma unroll
        for (int w = 0; w < 4; ++w) x[w] = __uint_as_float(u[w]);
      }
      return true;
    };
    for (int n = 0; ok; ++n) {
      int idx;
      Item it;
      if (!ring_read(p, item_ring, item_bar, n, abort_flag, idx, it)) break;
      if (idx < 0) break;
      const int q_idx = it.q_lo + qr;
      const int pos = it.L - it.nb + q_idx;
      const bool row_valid = (decode ? lane < p.G : true) && (q_idx < it.q_hi) && (pos >= it.key_lo);
      // the same for the four warps of a lane group (they hold the same rows)
      const bool warp_valid = decode ? true : __any_sync(0xffffffffu, row_valid);
      const int last_page = (it.L - 1) / PAGE;
      const int tail = it.L % PAGE;
      // the tile of this item whose last page holds slots past the sequence end (-1: none)
      const int zero_t = tail != 0 ? last_page / PAGES_PER_TILE - it.t0 : -1;
      const uint32_t zero_off = (uint32_t)(last_page % PAGES_PER_TILE) * BLOCK_BYTES;
      const size_t widx = ((size_t)(it.r0 + q_idx) * p.Hq + (size_t)(it.g * p.G + hj)) * p.n_split_max + it.s;
      float m = -INFINITY, l = 0.0f;  // l: this warp's quarter sum l_q
      for (int t = 0; t < it.ntiles; ++t, ++j) {
        const int sb = j % L::NS;
        const int kb0 = (it.t0 + t) * TILE;
        const bool need = row_valid && kb0 <= pos;
        const int nvalid = need ? min(TILE, pos + 1 - kb0) : 0;
        const int nq = min(32, max(0, nvalid - quarter * 32));
        if (!mbar_wait(&s_full[sb], ((uint32_t)j / L::NS) & 1u, p.status, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float alpha = 1.0f;
        // P is packed (two 16-bit values per word) into S[0..15] as S is consumed
        uint32_t S[32];
        uint32_t(&P)[16] = *reinterpret_cast<uint32_t(*)[16]>(&S[0]);
        if (warp_valid) {
          tmem_ld32(tmem + sb * 128 + lane_off + quarter * 32, S);
          tmem_ld_wait();
        }
        tc_fence_before();
        mbar_arrive(&s_free[sb]);
        if (warp_valid) {
          float xm[4];
          // prefill: a warp whose rows all see this whole quarter skips the
          // masking selects (the same operations on the same values)
          const bool full_q = !decode && __all_sync(0xffffffffu, nq >= 32);
          if (!exchange(full_q ? quarter_max(S, 32) : quarter_max(S, nq), xm)) { ok = false; break; }
          float mraw = -INFINITY;
#pragma unroll
          for (int q = 0; q < 4; ++q) mraw = fmaxf(mraw, xm[q]);
          float m_new = 0.0f;
          if (need) {
            m_new = new_reference(m, __fmul_rn(mraw, p.scale_log2), t);
            alpha = ex2_approx(__fsub_rn(m, m_new));
          }
          const float qs = full_q ? quarter_p<ET>(S, 32, -m_new, p.scale_log2, P)
                                  : quarter_p<ET>(S, nq, -m_new, p.scale_log2, P);
          if (need) {
            l = (t == 0) ? qs : __fadd_rn(__fmul_rn(alpha, l), qs);
            m = m_new;
          }
        }
        // P buffer j % NP was last read by the P V of tile j - NP
        if (j >= L::NP && !pv_done(j - L::NP)) { ok = false; break; }
        if (warp_valid) {
          if (decode ? lane < p.G : true)
            store_p_chunks(smem + OFF_P + (j % L::NP) * L::QP_BYTES, L::HALF, r, quarter, P);
          // rescale this warp's 32 columns of O in tensor memory (not on the
          // split's first tile, whose P V overwrites O)
          if (t > 0 && __any_sync(0xffffffffu, need && alpha != 1.0f)) {
            // O may be rescaled only once the P V of tile j-1 has landed in it
            if (L::NP > 1 && !pv_done(j - 1)) { ok = false; break; }
            uint32_t o[32];
            tmem_ld32(tmem + TMEM_O + lane_off + quarter * 32, o);
            tmem_ld_wait();
            const float a = need ? alpha : 1.0f;
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__fmul_rn(__uint_as_float(o[c]), a));
            tmem_st32(tmem + TMEM_O + lane_off + quarter * 32, o);
            tmem_st_wait();
          }
        }
        // zero V slots at or past the sequence end inside this tile's last
        // page (threads 0..127: value row d = thread)
        if (threadIdx.x < 128 && t == zero_t) {
          const int vb = j % NV;
          if (!mbar_wait(&v_full[vb], ((uint32_t)j / NV) & 1u, p.status, abort_flag)) { ok = false; break; }
          uint8_t* vblk = smem + OFF_V + vb * TILE_BYTES + zero_off;
          const int d = threadIdx.x;
          for (int slot = tail; slot < PAGE; ++slot) {
            const uint32_t off = (uint32_t)(d >> 3) * 256u + (uint32_t)(slot >> 3) * 128u +
                                 (uint32_t)(d & 7) * 16u + (uint32_t)(slot & 7) * 2u;
            *reinterpret_cast<uint16_t*>(vblk + off) = 0;
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_ready[j % L::NP]);
      }
      if (!ok) break;
      // end of the split: unnormalised O, m, l of every valid row
      if (!pv_done(j - 1)) { ok = false; break; }
      if (warp_valid) {
        // the row's sum: its four quarter sums, in quarter order
        float xl[4];
        if (!exchange(l, xl)) { ok = false; break; }
        const float lrow = __fadd_rn(__fadd_rn(__fadd_rn(xl[0], xl[1]), xl[2]), xl[3]);
        uint32_t o[32];
        tmem_ld32(tmem + TMEM_O + lane_off + quarter * 32, o);
        tmem_ld_wait();
        if (row_valid && quarter == 0) *reinterpret_cast<float2*>(p.ws_ml + widx * 2) = make_float2(m, lrow);
        if constexpr (decode) {
          if (row_valid) st_global_f32x32(p.ws_o + widx * HD + quarter * 32, o, p.ws_wide != 0);
        } else {
          // The warp's 32 rows go out as 128-byte row pieces, four lanes per
          // row: within each group of four lanes the 8-column chunks are
          // transposed (two exchange stages, lanes i ^ 2 then i ^ 1), after
          // which lane 4a + c holds chunk c of rows 4a .. 4a + 3 in its slots
          // 0 .. 3 (o[8k .. 8k + 7] = row 4a + k). Store k then writes row
          // 4a + k whole from its four lanes (same bytes as one row per lane,
          // a quarter of the memory requests).
          const int i4 = lane & 3;
#pragma unroll
          for (int e = 0; e < 16; ++e) {  // lanes i, i ^ 2 swap chunks {2, 3} / {0, 1}
            const bool hi = (i4 & 2) != 0;
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, hi ? o[e] : o[16 + e], 2);
            if (hi) o[e] = recv; else o[16 + e] = recv;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {  // lanes i, i ^ 1 swap slots {1, 3} / {0, 2}
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const bool odd = (i4 & 1) != 0;
              const int even_slot = h * 16 + e, odd_slot = h * 16 + 8 + e;
              const uint32_t recv = __shfl_xor_sync(0xffffffffu, odd ? o[even_slot] : o[odd_slot], 1);
              if (odd) o[even_slot] = recv; else o[odd_slot] = recv;
            }
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int rk = rg * 32 + (lane & ~3) + k;  // the row this store writes
            const int qk = it.q_lo + rk / p.G, hk = rk % p.G;
            if (qk < it.q_hi && it.L - it.nb + qk >= it.key_lo) {
              const size_t wk = ((size_t)(it.r0 + qk) * p.Hq + (size_t)(it.g * p.G + hk)) * p.n_split_max + it.s;
              float* dst = p.ws_o + wk * HD + quarter * 32 + i4 * 8;
              if (p.ws_wide) {
                asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst),
                             "r"(o[8 * k]), "r"(o[8 * k + 1]), "r"(o[8 * k + 2]), "r"(o[8 * k + 3]),
                             "r"(o[8 * k + 4]), "r"(o[8 * k + 5]), "r"(o[8 * k + 6]), "r"(o[8 * k + 7])
                             : "memory");
              } else {
                asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(o[8 * k]),
                             "r"(o[8 * k + 1]), "r"(o[8 * k + 2]), "r"(o[8 * k + 3])
                             : "memory");
                asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 4), "r"(o[8 * k + 4]),
                             "r"(o[8 * k + 5]), "r"(o[8 * k + 6]), "r"(o[8 * k + 7])
                             : "memory");
              }
            }
          }
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == L::PRODUCER_WARP + 1) {
    __syncwarp();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Finishing pass: a (query token, q head) row is merged by one warp, lane
// owning 4 of the 128 output elements. Splits merged strictly in order s = 0
// .. n-1.
struct CombineParams {
  const float* ws_o;
  const float* ws_ml;
  const int32_t* seq_lens;
  const int32_t* cu_q;  // null: decode
  void* out;  // 16-bit rows (the element type of the kernel)
  int64_t ldo;
  int32_t n_tok, B, Hq, n_split_max, max_kv_len;
  int32_t max_rows;  // rows per sequence the split kernel covers (qblocks x rows per block)
  int32_t hpu;       // heads of one query token per unit of work (1 .. 16)
};

// One (token, head) row, by one warp.
template <typename ET>
__device__ __forceinline__ void combine_row(const CombineParams& p, int tok, int h, int lane) {
  int b, nb, qidx;
  if (p.cu_q) {
    if (tok < p.cu_q[0] || tok >= p.cu_q[p.B]) return;  // a row this call does not cover
    int lo = 0, hi = p.B;  // find b with cu_q[b] <= tok < cu_q[b+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_q[mid] <= tok) lo = mid; else hi = mid;
    }
    b = lo;
    nb = p.cu_q[b + 1] - p.cu_q[b];
    qidx = tok - p.cu_q[b];
    if (p.cu_q[b] < 0 || p.cu_q[b + 1] > p.n_tok) nb = 0;  // malformed cu_q: zeros
  } else {
    b = tok;
    nb = 1;
    qidx = 0;
  }
  const int L = p.seq_lens[b];
  uint16_t* dst = static_cast<uint16_t*>(p.out) + (size_t)tok * p.ldo + (size_t)h * HD + lane * 4;
  if (L < nb || L > p.max_kv_len || nb <= 0 || qidx >= p.max_rows) {  // flagged by the split kernel; zeros
    *reinterpret_cast<uint2*>(dst) = make_uint2(0u, 0u);
    return;
  }
  const int pos = L - nb + qidx;
  const int n = pos / SPLIT + 1;
  const size_t base = ((size_t)tok * p.Hq + h) * p.n_split_max;
  // Lane s holds split s's (m, l) (splits 32 at a time); M is their maximum
  // (exact in any order), taken across the warp by shuffles.
  float2 ml0 = make_float2(-INFINITY, 0.0f);  // splits 0 .. 31, kept for the sums
  if (lane < n) ml0 = *reinterpret_cast<const float2*>(p.ws_ml + (base + lane) * 2);
  float M = ml0.x;
  for (int c = 32; c < n; c += 32)
    if (c + lane < n) M = fmaxf(M, p.ws_ml[(base + c + lane) * 2]);
#pragma unroll
  for (int d = 16; d; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
  // The sums in split order s = 0 .. n-1; the O rows of four splits are
  // loaded before their four fused multiply-adds, so the loads overlap.
  float Lsum = 0.0f;
  float o0 = 0.0f, o1 = 0.0f, o2 = 0.0f, o3 = 0.0f;
  for (int c = 0; c < n; c += 32) {
    float2 ml = ml0;
    if (c > 0) ml = c + lane < n ? *reinterpret_cast<const float2*>(p.ws_ml + (base + c + lane) * 2)
                                 : make_float2(-INFINITY, 0.0f);
    const float w_lane = c + lane < n ? exp2f(__fsub_rn(ml.x, M)) : 0.0f;  // split c + lane's weight
    const int cn = min(32, n - c);
    for (int k0 = 0; k0 < cn; k0 += 4) {
      float4 ov[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (k0 + k < cn) ov[k] = *reinterpret_cast<const float4*>(p.ws_o + (base + c + k0 + k) * HD + lane * 4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k0 + k < cn) {  // the same for the whole warp
          const float w = __shfl_sync(0xffffffffu, w_lane, k0 + k);
          const float l = __shfl_sync(0xffffffffu, ml.y, k0 + k);
          Lsum = __fmaf_rn(w, l, Lsum);
          o0 = __fmaf_rn(w, ov[k].x, o0);
          o1 = __fmaf_rn(w, ov[k].y, o1);
          o2 = __fmaf_rn(w, ov[k].z, o2);
          o3 = __fmaf_rn(w, ov[k].w, o3);
        }
      }
    }
  }
  // + 0.0f turns a -0 into +0, so a zero's sign cannot depend on the split path
  const float y0 = __fadd_rn(__fdiv_rn(o0, Lsum), 0.0f), y1 = __fadd_rn(__fdiv_rn(o1, Lsum), 0.0f);
  const float y2 = __fadd_rn(__fdiv_rn(o2, Lsum), 0.0f), y3 = __fadd_rn(__fdiv_rn(o3, Lsum), 0.0f);
  *reinterpret_cast<uint2*>(dst) = make_uint2(E16<ET>::pack2(y0, y1), E16<ET>::pack2(y2, y3));
}

// A query token's place in the finishing pass (every head of a token is the
// same case): 0 nothing to do (not covered by this call), 1 zeros (flagged by
// the split kernel), 2 n <= 4 splits, 3 more.
struct CombTok {
  int kind, n, tok;
};

__device__ __forceinline__ CombTok comb_token(const CombineParams& p, int tok) {
  CombTok t;
  t.tok = tok;
  t.kind = 0;
  t.n = 0;
  int b, nb, qidx;
  if (p.cu_q) {
    if (tok < p.cu_q[0] || tok >= p.cu_q[p.B]) return t;  // a token this call does not cover
    int lo = 0, hi = p.B;  // find b with cu_q[b] <= tok < cu_q[b+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_q[mid] <= tok) lo = mid; else hi = mid;
    }
    b = lo;
    nb = p.cu_q[b + 1] - p.cu_q[b];
    qidx = tok - p.cu_q[b];
    if (p.cu_q[b] < 0 || p.cu_q[b + 1] > p.n_tok) nb = 0;  // malformed cu_q: zeros
  } else {
    b = tok;
    nb = 1;
    qidx = 0;
  }
  const int L = p.seq_lens[b];
  if (L < nb || L > p.max_kv_len || nb <= 0 || qidx >= p.max_rows) {
    t.kind = 1;
    return t;
  }
  t.n = (L - nb + qidx) / SPLIT + 1;
  t.kind = t.n <= 4 ? 2 : 3;
  return t;
}

// One (token, head) row of the finishing pass and its token's case.
struct CombRow {
  int kind, n, tok, h;
};

__device__ __forceinline__ CombRow comb_row(const CombTok& t, int h) {
  CombRow r;
  r.kind = t.kind;
  r.n = t.n;
  r.tok = t.tok;
  r.h = h;
  return r;
}

// The row's first partial (split 0) in the workspace, and this lane's 4
// output elements.
__device__ __forceinline__ size_t comb_base(const CombineParams& p, const CombRow& r) {
  return ((size_t)r.tok * p.Hq + r.h) * p.n_split_max;
}
__device__ __forceinline__ uint16_t* comb_dst(const CombineParams& p, const CombRow& r, int lane) {
  return static_cast<uint16_t*>(p.out) + (size_t)r.tok * p.ldo + (size_t)r.h * HD + lane * 4;
}

// A short row's loads, issued asynchronously (cp.async) into this lane's own
// shared-memory slots: its 16 bytes of each split's O row, and (lane s < n)
// split s's (m, l). One commit group per row.
__device__ __forceinline__ void comb_issue(const CombineParams& p, const CombRow& r, int lane, float4* so,
                                           float2* sml) {
  if (r.kind == 2) {
    const size_t base = comb_base(p, r);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < r.n)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_u32(so + k * 32 + lane)),
                     "l"(p.ws_o + (base + k) * HD + lane * 4)
                     : "memory");
    if (lane < r.n)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(sml + lane)),
                   "l"(p.ws_ml + (base + lane) * 2)
                   : "memory");
  }
  cp_async_commit();
}

// The merge of a short row from the lane's own slots: the same operations as
// combine_row (M over the splits' m by shuffles, weights 2^(m_s - M), sums in
// split order, y = o / L + 0).
template <typename ET>
__device__ __forceinline__ void comb_short(const CombineParams& p, const CombRow& r, int lane, const float4* so,
                                           const float2* sml) {
  const float2 ml = lane < r.n ? sml[lane] : make_float2(-INFINITY, 0.0f);
  float M = ml.x;
#pragma unroll
  for (int d = 16; d; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
  const float w_lane = lane < r.n ? exp2f(__fsub_rn(ml.x, M)) : 0.0f;
  float Lsum = 0.0f;
  float o0 = 0.0f, o1 = 0.0f, o2 = 0.0f, o3 = 0.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (k < r.n) {  // the same for the whole warp
      const float w = __shfl_sync(0xffffffffu, w_lane, k);
      const float l = __shfl_sync(0xffffffffu, ml.y, k);
      const float4 o = so[k * 32 + lane];
      Lsum = __fmaf_rn(w, l, Lsum);
      o0 = __fmaf_rn(w, o.x, o0);
      o1 = __fmaf_rn(w, o.y, o1);
      o2 = __fmaf_rn(w, o.z, o2);
      o3 = __fmaf_rn(w, o.w, o3);
    }
  }
  const float y0 = __fadd_rn(__fdiv_rn(o0, Lsum), 0.0f), y1 = __fadd_rn(__fdiv_rn(o1, Lsum), 0.0f);
  const float y2 = __fadd_rn(__fdiv_rn(o2, Lsum), 0.0f), y3 = __fadd_rn(__fdiv_rn(o3, Lsum), 0.0f);
  *reinterpret_cast<uint2*>(comb_dst(p, r, lane)) = make_uint2(E16<ET>::pack2(y0, y1), E16<ET>::pack2(y2, y3));
}

// A grid of a few CTAs per SM whose warps stride over units of one query
// token and up to p.hpu of its heads (tens of thousands of one-row CTAs
// cost more in scheduling than the rows); the token's sequence and split
// count are looked up once per unit. A warp walks its rows (the heads of a
// unit, then the next unit's) and issues the next row's loads (cp.async into
// its own shared-memory slots, double-buffered) before merging the current
// row, so two rows' loads are in flight per warp without holding them in
// registers. Rows with more than four splits are merged from global memory
// (combine_row).
template <typename ET>
__global__ void __launch_bounds__(256, 4) attn_combine_kernel(const CombineParams p) {
  __shared__ __align__(16) float4 s_o[8][2][4 * 32];  // [warp][buffer][split * 32 + lane]
  __shared__ __align__(16) float2 s_ml[8][2][32];     // [warp][buffer][lane = split]
  // launched as a programmatic dependent of the split kernel: wait until that
  // grid has completed and its writes are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int hch = (p.Hq + p.hpu - 1) / p.hpu;  // units per token
  const int64_t units = (int64_t)p.n_tok * hch;
  const int64_t step = (int64_t)gridDim.x * (blockDim.x >> 5);
  int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + w;
  if (u >= units) return;
  // row cursor: unit u, head h of [h .. h_end)
  CombTok t = comb_token(p, (int)(u / hch));
  int h = (int)(u % hch) * p.hpu;
  int h_end = min(h + p.hpu, p.Hq);
  auto advance = [&]() -> bool {  // to the next row; false past the last
    if (++h < h_end) return true;
    u += step;
    if (u >= units) return false;
    t = comb_token(p, (int)(u / hch));
    h = (int)(u % hch) * p.hpu;
    h_end = min(h + p.hpu, p.Hq);
    return true;
  };
  CombRow cur = comb_row(t, h);
  int buf = 0;
  comb_issue(p, cur, lane, s_o[w][0], s_ml[w][0]);
  // every pass merges the current row; the loop ends after the row at which
  // the cursor (advance) ran past this warp's last unit
  bool more = advance(), last = false;
  do {
    CombRow nxt;
    nxt.kind = 0;
    if (more) nxt = comb_row(t, h);
    comb_issue(p, nxt, lane, s_o[w][buf ^ 1], s_ml[w][buf ^ 1]);
    cp_async_wait<1>();  // this lane's copies of the current row have landed
    if (cur.kind == 1) {
      *reinterpret_cast<uint2*>(comb_dst(p, cur, lane)) = make_uint2(0u, 0u);
    } else if (cur.kind == 2) {
      comb_short<ET>(p, cur, lane, s_o[w][buf], s_ml[w][buf]);
    } else if (cur.kind == 3) {
      combine_row<ET>(p, cur.tok, cur.h, lane);
    }
    last = !more;
    cur = nxt;
    buf ^= 1;
    if (more) more = advance();
  } while (!last);
  cp_async_wait<0>();
}

// partial O [n_tok][Hq][n_split][128] fp32, then (m, l) pairs, then (256-byte
// aligned) the work-item counter of the split kernel
static size_t ws_counter_offset(int64_t n_tok, int Hq, int n_split) {
  const size_t o = (size_t)n_tok * Hq * n_split * HD * sizeof(float);
  const size_t ml = (size_t)n_tok * Hq * n_split * 2 * sizeof(float);
  return (o + ml + 255) & ~(size_t)255;
}

static size_t ws_bytes_for(int64_t n_tok, int Hq, int n_split) {
  return ws_counter_offset(n_tok, Hq, n_split) + 256;
}

static bi_status check_shape(const bi_attn_shape* sh) {
  if (!sh) return fail(BI_ERR_INVALID_ARG, "attention: shape is null");
  if (sh->head_dim != HD) return fail(BI_ERR_SHAPE, "attention: head_dim must be %d", HD);
  if (sh->page_size != PAGE) return fail(BI_ERR_SHAPE, "attention: page_size must be %d", PAGE);
  if (sh->num_q_heads <= 0 || sh->num_kv_heads <= 0 || sh->num_q_heads % sh->num_kv_heads)
    return fail(BI_ERR_SHAPE, "attention: num_q_heads must be a positive multiple of num_kv_heads");
  const int G = sh->num_q_heads / sh->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(BI_ERR_SHAPE, "attention: q heads per kv head must be 1, 2, 4 or 8 (got %d)", G);
  if (sh->num_pages <= 0 || sh->max_pages_per_seq <= 0 || sh->max_kv_len <= 0)
    return fail(BI_ERR_SHAPE, "attention: num_pages, max_pages_per_seq and max_kv_len must be positive");
  if ((int64_t)sh->num_pages * sh->num_kv_heads > 0x7fffffffll / PAGE)
    return fail(BI_ERR_SHAPE, "attention: cache too large");
  if (!(sh->scale > 0.0f)) return fail(BI_ERR_INVALID_ARG, "attention: scale must be > 0");
  return BI_OK;
}

template <typename ET>
static bi_status run(const void* q, int64_t ldq, const int32_t* cu_q, int32_t max_q_len,
                     int64_t n_tok, const void* k_cache, const void* v_cache,
                     const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                     const bi_attn_shape* sh, void* out, int64_t ldo, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
  bi_status st = check_shape(sh);
  if (st != BI_OK) return st;
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !out)
    return fail(BI_ERR_INVALID_ARG, "attention: null pointer");
  if (B < 0 || n_tok < 0 || max_q_len < 0) return fail(BI_ERR_INVALID_ARG, "attention: negative size");
  const int Hq = sh->num_q_heads, G = sh->num_q_heads / sh->num_kv_heads;
  if (ldq < (int64_t)Hq * HD || ldo < (int64_t)Hq * HD) return fail(BI_ERR_SHAPE, "attention: ldq/ldo smaller than num_q_heads*128");
  if (ldq % 8 || ldo % 8) return fail(BI_ERR_ALIGN, "attention: ldq and ldo must be multiples of 8");
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache) || (ws && !aligned16(ws)))
    return fail(BI_ERR_ALIGN, "attention: pointers must be 16-byte aligned");
  if (B == 0 || n_tok == 0) return BI_OK;
  const int n_split = (sh->max_kv_len + SPLIT - 1) / SPLIT;
  const int QR = 128 / G;
  const int qblocks = cu_q ? (max_q_len + QR - 1) / QR : 1;
  if (cu_q && max_q_len <= 0) return fail(BI_ERR_SHAPE, "attention: max_q_len must be positive");
  const int64_t total_items = (int64_t)n_split * B * qblocks * sh->num_kv_heads;
  if (total_items > 0x7fffffffll) return fail(BI_ERR_SHAPE, "attention: too many work items");
  if (n_tok > 0x7fffffffll / Hq) return fail(BI_ERR_SHAPE, "attention: too many tokens");
  const size_t need = ws_bytes_for(n_tok, Hq, n_split);
  if (!ws || ws_bytes < need) return fail(BI_ERR_WORKSPACE, "attention: workspace %zu bytes < %zu needed", ws_bytes, need);
  if ((st = require_sm100()) != BI_OK) return st;

  CUtensorMap tmQ;
  {
    uint64_t dims[3] = {(uint64_t)HD, (uint64_t)Hq, (uint64_t)n_tok};
    uint64_t strides[2] = {(uint64_t)HD * 2, (uint64_t)ldq * 2};
    uint32_t box[3] = {64, (uint32_t)G, cu_q ? (uint32_t)QR : 1u};
    if ((st = encode_tmap(&tmQ, E16<ET>::kTmap, 3, const_cast<void*>(q), dims,
                          strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != BI_OK)
      return st;
  }
  Params p;
  p.kc = static_cast<const uint8_t*>(k_cache);
  p.vc = static_cast<const uint8_t*>(v_cache);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.cu_q = cu_q;
  p.ws_o = static_cast<float*>(ws);
  p.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + (size_t)n_tok * Hq * n_split * HD * sizeof(float));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = sh->num_kv_heads;
  p.G = G;
  p.QR = QR;
  p.qblocks = qblocks;
  p.q_box = cu_q ? QR : 1;
  p.n_tok = (int32_t)n_tok;
  p.num_pages = sh->num_pages;
  p.max_pages = sh->max_pages_per_seq;
  p.max_kv_len = sh->max_kv_len;
  p.n_split_max = n_split;
  p.total_items = (int32_t)total_items;
  p.work_counter = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + ws_counter_offset(n_tok, Hq, n_split));
  p.scale_log2 = (float)((double)sh->scale * 1.4426950408889634);  // scale * log2(e)
  p.status = status_word();
  p.ws_wide = (reinterpret_cast<uintptr_t>(p.ws_o) & 31) == 0;

  {
    // once per device, under a lock (calls may come from several host threads)
    static bool attr_set[64] = {false};
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return fail(BI_ERR_UNSUPPORTED, "attention: device id %d out of range", dev);
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_set[dev]) {
      cudaError_t e = cudaFuncSetAttribute(attn_split_kernel<true, ET>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)Lay<true>::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(attn_split_kernel<false, ET>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Lay<false>::SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail(e, "attention: smem attribute");
      attr_set[dev] = true;
    }
  }
  const int sms = num_sms();
  const int grid = (int)(total_items < sms ? total_items : sms);
  cudaError_t me = cudaMemsetAsync(p.work_counter, 0, sizeof(int32_t), stream);
  if (me != cudaSuccess) return cuda_fail(me, "attention: work counter reset");
  if (cu_q)
    attn_split_kernel<false, ET><<<grid, Lay<false>::THREADS, Lay<false>::SMEM_BYTES, stream>>>(tmQ, p);
  else
    attn_split_kernel<true, ET><<<grid, Lay<true>::THREADS, Lay<true>::SMEM_BYTES, stream>>>(tmQ, p);
  BI_CHECK_LAUNCH("attention split launch");

  CombineParams c;
  c.ws_o = p.ws_o;
  c.ws_ml = p.ws_ml;
  c.seq_lens = seq_lens;
  c.cu_q = cu_q;
  c.out = out;
  c.ldo = ldo;
  c.n_tok = (int32_t)n_tok;
  c.B = B;
  c.Hq = Hq;
  c.n_split_max = n_split;
  c.max_kv_len = sh->max_kv_len;
  c.max_rows = qblocks * QR;
  // Heads per unit: the largest of 16, 8, 4, 2 that still leaves a unit for
  // every warp of the grid (four CTAs of eight warps per SM), else 1. Units
  // decide only which warp merges a row, never how.
  const int64_t grid_warps = (int64_t)sms * 4 * 8;
  c.hpu = 1;
  for (int hpu = 16; hpu > 1; hpu >>= 1) {
    if (n_tok * ((Hq + hpu - 1) / hpu) >= grid_warps) {
      c.hpu = hpu;
      break;
    }
  }
  const int64_t warps = n_tok * ((Hq + c.hpu - 1) / c.hpu);  // one per (token, head unit)
  const int64_t want = (warps + 7) / 8;
  const int blocks = (int)(want < (int64_t)num_sms() * 4 ? want : (int64_t)num_sms() * 4);
  // programmatic dependent launch: the combine is launched as the split
  // kernel's CTAs exit (no explicit trigger: an early one measured slower for
  // prefill) and starts its work only once the split grid is done
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t ce = cudaLaunchKernelEx(&cfg, attn_combine_kernel<ET>, c);
  if (ce != cudaSuccess) return cuda_fail(ce, "attention combine launch");
  BI_CHECK_LAUNCH("attention combine launch");
  return BI_OK;
}

}  // namespace attn

// The FP16 variant (fp16 Q, caches, P and output) for the forward's FP16
// precision mode; the same kernels as bi_attn_decode / bi_attn_prefill.
bi_status attn_decode_f16(const void* q, int64_t ldq, const void* k_cache, const void* v_cache,
                          const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                          const bi_attn_shape* shape, void* out, int64_t ldo, void* ws, size_t ws_bytes,
                          cudaStream_t s) {
  return attn::run<f16>(q, ldq, nullptr, 1, B, k_cache, v_cache, block_table, seq_lens, B, shape, out, ldo,
                        ws, ws_bytes, s);
}

bi_status attn_prefill_f16(const void* q, int64_t ldq, const int32_t* cu_q, int32_t max_q_len, int64_t n_tok,
                           const void* k_cache, const void* v_cache, const int32_t* block_table,
                           const int32_t* seq_lens, int32_t B, const bi_attn_shape* shape, void* out,
                           int64_t ldo, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (!cu_q) return fail(BI_ERR_INVALID_ARG, "attn_prefill: cu_q is null");
  return attn::run<f16>(q, ldq, cu_q, max_q_len, n_tok, k_cache, v_cache, block_table, seq_lens, B, shape, out,
                        ldo, ws, ws_bytes, s);
}
}  // namespace bi

using namespace bi;

extern "C" bi_status bi_attn_workspace_size(const bi_attn_shape* shape, int64_t max_tokens,
                                            size_t* bytes) {
  bi_status st = attn::check_shape(shape);
  if (st != BI_OK) return st;
  if (!bytes || max_tokens < 0) return fail(BI_ERR_INVALID_ARG, "attn_workspace_size: bad arguments");
  const int n_split = (shape->max_kv_len + attn::SPLIT - 1) / attn::SPLIT;
  *bytes = attn::ws_bytes_for(max_tokens, shape->num_q_heads, n_split);
  return BI_OK;
}

extern "C" bi_status bi_attn_decode(const void* q, int64_t ldq, const void* k_cache,
                                    const void* v_cache, const int32_t* block_table,
                                    const int32_t* seq_lens, int32_t B, const bi_attn_shape* shape,
                                    void* out, int64_t ldo, void* ws, size_t ws_bytes,
                                    void* stream) {
  return attn::run<bf16>(q, ldq, nullptr, 1, B, k_cache, v_cache, block_table, seq_lens, B, shape, out,
                   ldo, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" bi_status bi_attn_prefill(const void* q, int64_t ldq, const int32_t* cu_q,
                                     int32_t max_q_len, int64_t n_tok, const void* k_cache,
                                     const void* v_cache, const int32_t* block_table,
                                     const int32_t* seq_lens, int32_t B,
                                     const bi_attn_shape* shape, void* out, int64_t ldo, void* ws,
                                     size_t ws_bytes, void* stream) {
  if (!cu_q) return fail(BI_ERR_INVALID_ARG, "attn_prefill: cu_q is null");
  return attn::run<bf16>(q, ldq, cu_q, max_q_len, n_tok, k_cache, v_cache, block_table, seq_lens, B,
                   shape, out, ldo, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}
