// Persistent grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes (SwiGLU equation of the Sparse MoE FFN note, "How it
// works": FFN(u) = W2 (SiLU(W1 u) * W3 u), W1, W3 in R^{f x d}, W2 in
// R^{d x f}; the router logits have their own kernel, umma_router.cu):
//
//   kUmmaSwiGLU: h[r][m] = SiLU(sum_c W1_e[m][c] x[r][c]) * (sum_c W3_e[m][c] x[r][c])
//   kUmmaSwiGLUSave: the same, also storing both sums (the pre-activations a
//                training forward keeps for the backward pass)
//   kUmmaDown:   y[r][m] = sum_c W2_e[m][c] h[r][c]
//   kUmmaBiasAct: o[r][m] = act(sum_c W_e[m][c] u[r][c] + b_e[m]), act = GELU or
//                identity (the generic expert of "Lesson 2 - From the Dense FFN
//                to a Layer of Experts", section 2: W2 phi(W1 u + b1) + b2)
//   kUmmaDgrad:  o[r][m] = sum_c W_e[c][m] g[r][c]   (the transposed weight:
//                input gradients of the backward pass; W_e is read with m
//                contiguous, an MN-major operand; the contraction may run
//                over two stacked weights, W for c < k_split blocks, W' after)
//
// for every packed row r of every segment. Segment e < n_routed is expert e
// over packed rows [offsets[e], offsets[e+1]); segment n_routed is the dense
// segment (the shared expert over all T tokens, or a dense weight such as the
// router's in the backward pass).
//
// Orientation ("swap AB"): weight rows are the MMA's M side (128 per MMA) and
// tokens its N side (16..256 per tile, a multiple of 16). A DeepSeek-V3 expert
// sees a few dozen to a few hundred tokens; putting tokens on N pads them to
// 16, not to a 128-row M tile, and each weight tile is read from HBM once per
// token tile. Each tile pairs two 128-row weight blocks with one token block
// (SwiGLU: the W1 and W3 rows of the same f range; down: 256 consecutive W2
// rows), so two MMAs share every token tile that is staged.
//
// Roles (one CTA per SM, persistent over a static tile list):
//   warp 0 lane 0 : TMA producer into a ring of variable-size slots
//   warp 1        : TMEM allocator; lane 0 issues tcgen05.mma (kind::f16,
//                   bf16 x bf16 -> fp32 in TMEM) and tcgen05.commit; in a
//                   pair's peer CTA lane 0 forwards gathered rows' arrivals
//   warps 2..9    : epilogue, EPI_WPQ warps per 32-lane TMEM quarter (each
//                   takes every EPI_WPQ-th 16-column chunk); tcgen05.ld, SiLU
//                   * up in fp32, one rounding to the output type, masked
//                   stores
//   warps 10..11  : launched for CTA pairs and gathered rows: lane 0 of warp
//                   10 issues each slot's second weight block and packed token
//                   rows, or both warps gather token rows with cp.async
//
// TMEM (512 columns) holds a tile's two accumulators. Tiles of at most 128
// token columns alternate between the two 256-column halves, so the MMAs of
// the next tile do not wait for the epilogue to drain this one; wider tiles
// take all 512 columns.
//
// The slot ring: a k-step needs (weights) + (its token rows, rounded to 32)
// bytes, so slots are sized per tile and packed into one shared-memory ring
// (wrapping to the start when the tail is too short), with at most
// max_inflight slots loading or waiting at a time. Slot addresses depend
// only on the sequence of slot sizes, so the producer and the MMA issuer
// compute them independently; the producer reuses bytes only after the MMA
// released (tcgen05.commit) every slot that overlaps them. Narrow token
// tiles thus buy more weight bytes in flight, the quantity that bounds a
// weight-streaming GEMM.
//
// Shared-memory tiles use the 128-byte swizzle written by TMA and read by the
// MMA through K-major SW128 descriptors (8-row atoms 1024 B apart). TMA loads
// past a segment's end read neighbouring rows or zero fill; such columns
// (tokens) and rows (weights past m_rows) are never stored.
//
// Every wait is bounded; on expiry the CTA records kErrTimeoutWait in the
// error word, raises a shared abort flag, drains its in-flight copies and
// MMAs (again bounded), frees TMEM and returns.
#include "umma_common.cuh"

namespace moe {
namespace {

constexpr int BM = 128;          // weight rows per MMA (M)
constexpr int BK = 64;           // K per slot: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;       // K per tcgen05.mma for 16-bit inputs
constexpr int BN_MAX = 256;      // token columns per tile (MMA N), upper bound
constexpr int BOX_N_MAX = 128;   // token rows per TMA box, at most
constexpr int kSplitB = 1;       // CTA pairs: a second thread issues part of each slot's copies
constexpr int A_BYTES = BM * BK * 2;
constexpr int EPI_WPQ = 2;                  // epilogue warps per 32-lane TMEM quarter
constexpr int EPI_WARPS = 4 * EPI_WPQ;      // warps 2 .. 1 + EPI_WARPS
constexpr int EPI_CPW = (16 + EPI_WPQ - 1) / EPI_WPQ;   // 16-column chunks per warp and accumulator (256 / 16 = 16 in all)
constexpr int GATHER_WARPS = 2;   // warps 10..11, launched only when B is gathered
constexpr int NUM_THREADS = 32 * (2 + EPI_WARPS);                   // without gather warps
constexpr int NUM_THREADS_GATHER = 32 * (2 + EPI_WARPS + GATHER_WARPS);
constexpr int TMEM_COLS = 512;
constexpr int NSLOT = 8;            // barrier pairs of the slot ring
constexpr int SMEM_LIMIT = 232448;  // 227 KB of dynamic shared memory per block
// Gathered token rows per gather lane and tile: a CTA stages at most 128
// rows, each gather warp half of them, four rows per 32 lanes at a time.
constexpr int kGatherRowsPerLane = 128 / GATHER_WARPS / 4;
// barriers, TMEM slot, slot records (first 1 KB); per gather warp the source
// offsets of its token rows, [kGatherRowsPerLane][32 lanes] words
constexpr int HDR_BYTES = 1024 + GATHER_WARPS * kGatherRowsPerLane * 32 * 4;

// Shared-memory plan of one launch: [header (barriers, gathered token rows) |
// tile tables | slot ring],
// the ring 1024-byte aligned (128-byte swizzle atoms).
struct SmemPlan {
  int table_bytes, ring_bytes, total;
};

__host__ __device__ inline SmemPlan smem_plan(int n_routed, int nseg) {
  SmemPlan sp;
  sp.table_bytes = ((nseg + 1 + n_routed + 1) * 4 + 1023) / 1024 * 1024;
  sp.ring_bytes = (SMEM_LIMIT - 1024 - HDR_BYTES - sp.table_bytes) / 1024 * 1024;
  sp.total = 1024 + HDR_BYTES + sp.table_bytes + sp.ring_bytes;
  return sp;
}

// Deterministic slot allocation shared by producer and MMA issuer.
struct RingCursor {
  uint32_t head = 0;    // next free byte (before wrap check)
  uint32_t count = 0;   // slots allocated so far
  __device__ __forceinline__ uint32_t peek(uint32_t size, uint32_t cap) const {
    return head + size > cap ? 0u : head;
  }
  __device__ __forceinline__ void take(uint32_t size, uint32_t cap, uint32_t& off, uint32_t& slot,
                                       uint32_t& parity) {
    off = peek(size, cap);
    head = off + size;
    slot = count % NSLOT;
    parity = (count / NSLOT) & 1u;
    ++count;
  }
};

// ---- CTA-pair (cluster of 2) forms used by the two-SM MMA path.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA into this CTA's shared memory, completing on a barrier that may sit in
// the peer CTA (the pair leader's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* tm, int c0, int c1,
                                                 uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(cluster_bar)
      : "memory");
}
// 16 bytes from global memory into shared memory (cp.async, L2 only);
// bytes past src_bytes (0..16) are zero.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// One arrival on the barrier once this thread's earlier cp.async copies have
// landed; the arrival is not added to the barrier's expected count.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (M=256 across the pair) (+)= A * B^T; each CTA holds 128 rows of A and
// half of B's rows at the same shared-memory offsets, and 128 lanes of D.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at this offset in every CTA of `mask` once the pair
// MMAs issued so far complete.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

// ------------------------------------------------------------ tile list
// Per mode: weight blocks (128 rows each) per CTA. With PAIR the two CTAs of
// a cluster run one M=256 MMA: each holds 128 rows of every weight block and
// half of the token tile.
template <int MODE> struct Kind;
template <> struct Kind<kUmmaSwiGLU> { static constexpr int A_TILES = 2; };
template <> struct Kind<kUmmaSwiGLUSave> { static constexpr int A_TILES = 2; };

// Modes whose tile pairs the W1 and W3 rows of one range (SwiGLU).
__host__ __device__ constexpr bool dual_a(int mode) { return mode == kUmmaSwiGLU || mode == kUmmaSwiGLUSave; }
template <> struct Kind<kUmmaDown>   { static constexpr int A_TILES = 2; };
template <> struct Kind<kUmmaBiasAct> { static constexpr int A_TILES = 2; };
template <> struct Kind<kUmmaDgrad> { static constexpr int A_TILES = 2; };

// Where a tile's two accumulators sit in the 512 TMEM columns. Half h is
// columns [128h, 128h + 128) and [256 + 128h, 256 + 128h + 128). A tile of at
// most 128 token columns takes one half (first accumulator at 128h, second
// at 256 + 128h), alternating halves, so the next such tile accumulates
// while the epilogue drains this one. A wider tile takes both halves (first
// accumulator at 0, second at 256): its token columns 0..127 are half 0, so
// its epilogue can hand half 0 back as soon as it has drained those columns
// of both accumulators, and a following narrow tile starts while the rest
// drains. The MMA issuer and the epilogue walk the same tile sequence, so
// they derive the same placement.
struct AccPlace {
  uint32_t next = 0;   // half the next narrow tile takes
  __device__ __forceinline__ void take(int n_mma, bool& wide, uint32_t& half) {
    wide = n_mma > BN_MAX / 2;
    half = wide ? 0u : next;
    next = wide ? 0u : (next ^ 1u);
  }
  __device__ __forceinline__ static uint32_t col0(bool wide, uint32_t half) { return wide ? 0u : half * (BN_MAX / 2); }
  __device__ __forceinline__ static uint32_t second(bool) { return BN_MAX; }
};

// Modes whose tile is two consecutive 128-row blocks of one weight matrix.
__host__ __device__ constexpr bool two_blocks(int mode) {
  return mode == kUmmaDown || mode == kUmmaBiasAct || mode == kUmmaDgrad;
}

// Weight rows covered by one tile (all CTAs of the group together).
__host__ __device__ constexpr int tile_rows(int mode, bool pair) {
  return (two_blocks(mode) ? 256 : 128) * (pair ? 2 : 1);
}

// The parameters as launched: the caller's, plus what the launcher derives.
// Each TMA copy costs the issuing thread and the copy engine a fixed
// overhead whatever its size, and a slot completes only when all of its
// copies have, so a CTA's token rows of a slot come in one copy.
struct UmmaLaunch : UmmaGemmParams {
  int box_n;     // token rows per copy of B: a multiple of 8, at most 128
  int split_b;   // a second thread (warp 2 + EPI_WARPS, lane 0) issues each slot's second
                 // weight block and its packed token rows (CTA pairs only)
};

struct Tile {
  int seg, wt, tt;
  int rows;      // tokens in the segment
  int mrows;     // weight rows of the segment
  int K;
  int b_row0;    // first packed row (token) of the segment in the B tensor
  bool dense;
};

__device__ __forceinline__ void seg_dims(const UmmaGemmParams& p, const int* s_off, int s, int& rows,
                                         int& mrows) {
  if (s < p.n_routed) {
    rows = s_off[s + 1] - s_off[s];
    mrows = p.m_rows;
  } else {
    rows = p.shared_rows;
    mrows = p.m_rows_s;
  }
}

__device__ __forceinline__ Tile decode_tile(const UmmaGemmParams& p, const int* s_off,
                                            const int* s_start, int nseg, int tile, int wrows) {
  int lo = 0, hi = nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  Tile t;
  t.seg = lo;
  seg_dims(p, s_off, lo, t.rows, t.mrows);
  t.dense = lo >= p.n_routed;
  t.K = t.dense ? p.K_s : p.K;
  t.b_row0 = t.dense ? 0 : s_off[lo];
  const int nwt = ceil_div(t.mrows, wrows), ntt = ceil_div(t.rows, p.bn_max);
  const int local = tile - s_start[lo];
  if (t.rows <= t.mrows) {   // weights dominate: keep one weight tile's token tiles together
    t.wt = local / ntt;
    t.tt = local - t.wt * ntt;
  } else {                   // tokens dominate: sweep the expert's weights per token tile
    t.tt = local / nwt;
    t.wt = local - t.tt * nwt;
  }
  return t;
}

// Token rows this CTA stages for a tile, and how many TMA boxes that takes.
struct TokenSlice {
  int n_valid, n_mma, row, nbox;
  uint32_t box_bytes;   // bytes of one copy of B
  int rows_gather;      // rows staged by gather4 (routed tiles of a gathered B), else 0
  __device__ __forceinline__ uint32_t bytes() const {
    return rows_gather > 0 ? (uint32_t)rows_gather * (BK * 2) : (uint32_t)nbox * box_bytes;
  }
};
template <bool PAIR>
__device__ __forceinline__ TokenSlice token_slice(const UmmaLaunch& p, const Tile& t, uint32_t rank) {
  TokenSlice ts;
  ts.n_valid = min(p.bn_max, t.rows - t.tt * p.bn_max);
  ts.n_mma = (ts.n_valid + 15) & ~15;
  const int mine = PAIR ? ts.n_mma / 2 : ts.n_valid;
  ts.row = t.b_row0 + t.tt * p.bn_max + (PAIR ? (int)rank * (ts.n_mma / 2) : 0);
  ts.nbox = (mine + p.box_n - 1) / p.box_n;
  ts.box_bytes = (uint32_t)p.box_n * (BK * 2);
  // Gathered tiles stage exactly the rows the MMA reads (a multiple of 8).
  ts.rows_gather = (p.b_gather && !t.dense) ? (PAIR ? ts.n_mma / 2 : ts.n_mma) : 0;
  return ts;
}

// The warps after the epilogue's gather the SwiGLU forward's token rows,
// or (split_b) the first of them issues the packed token rows' copies.
template <int MODE> constexpr int max_threads() { return NUM_THREADS_GATHER; }

template <int MODE, bool PAIR>
__global__ void __launch_bounds__(max_threads<MODE>(), 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA3,
                     const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmAs,
                     const __grid_constant__ CUtensorMap tmA3s, const __grid_constant__ CUtensorMap tmBs,
                     const UmmaLaunch p) {
  using KD = Kind<MODE>;
  constexpr int A_TILES = KD::A_TILES;
  constexpr int WROWS = tile_rows(MODE, PAIR);
  // Row offset of weight block a (0 or 1) inside a tile, for CTA rank r.
  constexpr int BLOCK_STEP = two_blocks(MODE) ? (PAIR ? 256 : 128) : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int nseg = p.n_routed + (p.shared_rows > 0 ? 1 : 0);
  const SmemPlan sp = smem_plan(p.n_routed, nseg);
  const uint32_t cap = (uint32_t)sp.ring_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + NSLOT;
  uint64_t* accf_bar = bars + 2 * NSLOT;
  uint64_t* acce_bar = accf_bar + 2;
  uint64_t* drain_bar = acce_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  uint32_t* fl_off = tmem_slot + 2;             // producer's record of slots in flight
  uint32_t* fl_size = fl_off + NSLOT;
  uint64_t* gbar = reinterpret_cast<uint64_t*>(smem + 256);   // peer CTA: its gathered rows landed
  uint64_t* acq_bar = gbar + NSLOT;                            // slot claimed by the TMA issuer
  uint32_t* s_goff = reinterpret_cast<uint32_t*>(smem + 1024);   // gathered rows' byte offsets in the source
  int* s_start = reinterpret_cast<int*>(smem + HDR_BYTES);
  int* s_off = s_start + (nseg + 1);
  uint8_t* ring = smem + HDR_BYTES + sp.table_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const bool gather = p.b_gather != nullptr;
  const int group = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int ngroups = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  // Segment offsets come from the caller: each is clamped into the packed
  // rows (and a decreasing pair makes an empty segment), so no tile can reach
  // past them; CTA 0 records any offset that was out of range.
  for (int s = threadIdx.x; s <= p.n_routed; s += blockDim.x)
    s_off[s] = p.n_routed > 0 ? clamp_offset(p.offsets[s], p.max_routed_rows, blockIdx.x == 0 ? p.err : nullptr)
                              : 0;
  if (threadIdx.x == 64) {
    // Full barrier arrivals per slot: the arming TMA issuer; with a gathered
    // B also every gather lane, and on a pair the peer's forwarder.
    constexpr uint32_t kGatherLanes = 32 * GATHER_WARPS;
    const uint32_t full_count = gather ? (PAIR ? (leader ? 2u + kGatherLanes : 1u) : 1u + kGatherLanes) : 1u;
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(smem_u32(&full_bar[i]), full_count);
      mbar_init(smem_u32(&empty_bar[i]), 1);
      mbar_init(smem_u32(&gbar[i]), kGatherLanes);
      mbar_init(smem_u32(&acq_bar[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&accf_bar[i]), 1);
      mbar_init(smem_u32(&acce_bar[i]), (PAIR ? 2 : 1) * EPI_WARPS);   // one arrival per epilogue warp
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  if (threadIdx.x == 0) {
    tmap_prefetch(&tmA); tmap_prefetch(&tmB); tmap_prefetch(&tmAs); tmap_prefetch(&tmBs);
    if (dual_a(MODE)) { tmap_prefetch(&tmA3); tmap_prefetch(&tmA3s); }
  }
  __syncthreads();
  // Tiles per segment -> exclusive prefix s_start[0..nseg] (warp 0).
  if (warp == 0) {
    const int per = ceil_div(nseg, 32);
    const int s0 = min(nseg, lane * per), s1 = min(nseg, s0 + per);
    int sum = 0;
    for (int s = s0; s < s1; ++s) {
      int rows, mrows;
      seg_dims(p, s_off, s, rows, mrows);
      sum += rows > 0 ? ceil_div(mrows, WROWS) * ceil_div(rows, p.bn_max) : 0;
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    int run = incl - sum;
    for (int s = s0; s < s1; ++s) {
      s_start[s] = run;
      int rows, mrows;
      seg_dims(p, s_off, s, rows, mrows);
      run += rows > 0 ? ceil_div(mrows, WROWS) * ceil_div(rows, p.bn_max) : 0;
    }
    if (lane == 31) s_start[nseg] = incl;
  }
  if (blockIdx.x == 0 && p.err)
    for (int s = threadIdx.x; s < p.n_routed; s += blockDim.x)
      if (s_off[s + 1] < s_off[s]) atomicOr(p.err, kErrBadIndex);
  tc_fence_before();
  if (PAIR) cluster_sync_all(); else __syncthreads();   // barriers of both CTAs exist from here on
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = s_start[nseg];

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    // Claims ring slots and issues the TMA copies. A gathered B (routed
    // token rows read from the source activations through b_gather) is
    // copied by the gather warps: each claimed slot is announced on its
    // acq_bar.
    RingCursor cur;
    uint32_t inflight = 0;
    const uint32_t max_inflight = (uint32_t)min(max(p.max_inflight, 2), NSLOT);
    bool ok = true;
    for (int tile = group; tile < total_tiles && ok; tile += ngroups) {
      const Tile t = decode_tile(p, s_off, s_start, nseg, tile, WROWS);
      const TokenSlice ts = token_slice<PAIR>(p, t, rank);
      const CUtensorMap* mA = t.dense ? &tmAs : &tmA;
      const CUtensorMap* mA3 = t.dense ? &tmA3s : &tmA3;
      const CUtensorMap* mB = t.dense ? &tmBs : &tmB;
      const int a_row = (t.dense ? 0 : t.seg * p.m_rows) + t.wt * WROWS + (int)rank * BM;
      // kUmmaDgrad: output rows m of the stored weight's columns, contraction
      // rows c of the stored weight (this segment's block of them).
      const int m_row0 = t.wt * WROWS + (int)rank * BM;
      const int c_row0 = t.dense ? 0 : t.seg * p.a_k_rows;
      const int ksplit = t.dense ? p.k_split_s : p.k_split;
      const uint32_t bytes = A_TILES * A_BYTES + ts.bytes();
      // Bytes the TMA delivers: the weights, and B unless it is gathered.
      const uint32_t tx = A_TILES * A_BYTES + (ts.rows_gather > 0 ? 0u : ts.bytes());
      const int nk = ceil_div(t.K, BK);
      for (int kb = 0; kb < nk && ok; ++kb) {
        // Make room: the barrier pair and the bytes of the new slot must be free.
        const uint32_t off_new = cur.peek(bytes, cap);
        while (true) {
          bool clash = inflight >= max_inflight;
          for (uint32_t i = 0; i < inflight && !clash; ++i) {
            const uint32_t j = (cur.count - inflight + i) % NSLOT;
            clash = off_new < fl_off[j] + fl_size[j] && fl_off[j] < off_new + bytes;
          }
          if (!clash) break;
          const uint32_t oldest = cur.count - inflight;
          if (!wait_bounded(smem_u32(&empty_bar[oldest % NSLOT]), (oldest / NSLOT) & 1u, abort_flag,
                            p.err, p.timeout_ns, true)) {
            ok = false;
            break;
          }
          --inflight;
        }
        if (!ok) break;
        uint32_t off, slot, parity;
        cur.take(bytes, cap, off, slot, parity);
        fl_off[slot] = off;
        fl_size[slot] = bytes;
        ++inflight;
        if (gather || p.split_b) mbar_arrive(smem_u32(&acq_bar[slot]));
        const uint32_t fb_local = smem_u32(&full_bar[slot]);
        const uint32_t sb = smem_u32(ring + off);
        const uint32_t bb = sb + A_TILES * A_BYTES;
        if (PAIR) {
          // Both CTAs' copies complete on the leader's barrier, which the
          // leader arms for both halves (the halves are the same size).
          const uint32_t fb = map_to_cta(fb_local, 0);
          if (leader) mbar_expect_tx(fb_local, 2 * tx);
          if (MODE == kUmmaDgrad) {
            const bool second = kb >= ksplit;
            const int crow = c_row0 + (second ? kb - ksplit : kb) * BK;
            const CUtensorMap* mk = second ? mA3 : mA;
#pragma unroll
            for (int blk = 0; blk < 2; ++blk)
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_2d_pair(sb + blk * A_BYTES + h * MN_BOX_BYTES, mk, m_row0 + blk * BLOCK_STEP + h * 64,
                                 crow, fb);
          } else {
            tma_load_2d_pair(sb, mA, kb * BK, a_row, fb);
            if (dual_a(MODE) && !p.split_b) tma_load_2d_pair(sb + A_BYTES, mA3, kb * BK, a_row, fb);
            if (two_blocks(MODE) && !p.split_b) tma_load_2d_pair(sb + A_BYTES, mA, kb * BK, a_row + BLOCK_STEP, fb);
          }
          if (ts.rows_gather == 0 && !p.split_b)
            for (int bx = 0; bx < ts.nbox; ++bx)
              tma_load_2d_pair(bb + bx * ts.box_bytes, mB, kb * BK, ts.row + bx * p.box_n, fb);
        } else {
          mbar_expect_tx(fb_local, tx);
          if (MODE == kUmmaDgrad) {
            const bool second = kb >= ksplit;
            const int crow = c_row0 + (second ? kb - ksplit : kb) * BK;
            const CUtensorMap* mk = second ? mA3 : mA;
#pragma unroll
            for (int blk = 0; blk < 2; ++blk)
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_2d(sb + blk * A_BYTES + h * MN_BOX_BYTES, mk, m_row0 + blk * BLOCK_STEP + h * 64, crow,
                            fb_local);
          } else {
            tma_load_2d(sb, mA, kb * BK, a_row, fb_local);
            if (dual_a(MODE)) tma_load_2d(sb + A_BYTES, mA3, kb * BK, a_row, fb_local);
            if (two_blocks(MODE)) tma_load_2d(sb + A_BYTES, mA, kb * BK, a_row + BLOCK_STEP, fb_local);
          }
          if (ts.rows_gather == 0 && !p.split_b)
            for (int bx = 0; bx < ts.nbox; ++bx)
              tma_load_2d(bb + bx * ts.box_bytes, mB, kb * BK, ts.row + bx * p.box_n, fb_local);
        }
      }
    }
    // Let every copy this thread started land before the CTA can exit: its
    // slot is released only after the MMA consumed it.
    for (uint32_t i = 0; i < inflight; ++i) {
      const uint32_t u = cur.count - inflight + i;
      if (PAIR)
        wait_bounded(smem_u32(&empty_bar[u % NSLOT]), (u / NSLOT) & 1u, abort_flag, p.err,
                     p.timeout_ns, false);
      else
        wait_bounded(smem_u32(&full_bar[u % NSLOT]), (u / NSLOT) & 1u, abort_flag, p.err,
                     p.timeout_ns, false);
    }
  } else if (p.split_b && warp == 2 + EPI_WARPS && lane == 0) {
    // ------------------------------------------------------------ second issuer
    // One thread's copy issue paces the weight stream (each copy costs its
    // issuer a fixed time, whatever the size), so on CTA pairs a second
    // thread takes the slot's second weight block (W3, or down's block a
    // block step further) and its packed token rows, once the producer has
    // claimed the slot (same ring walk, so the same offsets). The copies
    // complete on the slot's full barrier, which the producer armed for all.
    RingCursor cur;
    bool ok = true;
    for (int tile = group; tile < total_tiles && ok; tile += ngroups) {
      const Tile t = decode_tile(p, s_off, s_start, nseg, tile, WROWS);
      const TokenSlice ts = token_slice<PAIR>(p, t, rank);
      const CUtensorMap* mB = t.dense ? &tmBs : &tmB;
      const uint32_t bytes = A_TILES * A_BYTES + ts.bytes();
      const int nk = ceil_div(t.K, BK);
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t u = cur.count;
        uint32_t off, slot, parity;
        cur.take(bytes, cap, off, slot, parity);
        if (!wait_bounded(smem_u32(&acq_bar[slot]), (u / NSLOT) & 1u, abort_flag, p.err, p.timeout_ns, true)) {
          ok = false;
          break;
        }
        const uint32_t bb = smem_u32(ring + off) + A_TILES * A_BYTES;
        const uint32_t fb_local = smem_u32(&full_bar[slot]);
        if (PAIR && MODE != kUmmaDgrad) {   // the slot's second weight block
          const int a_row = (t.dense ? 0 : t.seg * p.m_rows) + t.wt * WROWS + (int)rank * BM;
          const CUtensorMap* mA = t.dense ? &tmAs : &tmA;
          const CUtensorMap* mA3 = t.dense ? &tmA3s : &tmA3;
          const uint32_t sb = smem_u32(ring + off);
          if (dual_a(MODE)) tma_load_2d_pair(sb + A_BYTES, mA3, kb * BK, a_row, map_to_cta(fb_local, 0));
          if (two_blocks(MODE)) tma_load_2d_pair(sb + A_BYTES, mA, kb * BK, a_row + BLOCK_STEP, map_to_cta(fb_local, 0));
        }
        for (int bx = 0; bx < ts.nbox; ++bx) {
          if (PAIR)
            tma_load_2d_pair(bb + bx * ts.box_bytes, mB, kb * BK, ts.row + bx * p.box_n, map_to_cta(fb_local, 0));
          else
            tma_load_2d(bb + bx * ts.box_bytes, mB, kb * BK, ts.row + bx * p.box_n, fb_local);
        }
      }
    }
  } else if (gather && warp >= 2 + EPI_WARPS) {
    // ------------------------------------------------------------ gather
    // Gather warp g copies rows [g R/2, (g+1) R/2) of the CTA's R gathered
    // token rows into each slot the issuer claims (same ring walk, so the
    // same offsets): lane l takes 16-byte column chunk l % 8 of rows
    // l / 8 + 4i, whose source offsets are fixed per tile. Each lane's
    // completion is one arrival on the slot's full barrier (in a pair's peer
    // CTA on its gather barrier, which the forwarder passes on).
    const int gw = warp - (2 + EPI_WARPS);
    uint32_t* goff = s_goff + gw * kGatherRowsPerLane * 32;
    const char* src = static_cast<const char*>(p.b_gather_src);
    RingCursor cur;
    bool ok = true;
    for (int tile = group; tile < total_tiles && ok; tile += ngroups) {
      const Tile t = decode_tile(p, s_off, s_start, nseg, tile, WROWS);
      const TokenSlice ts = token_slice<PAIR>(p, t, rank);
      const uint32_t bytes = A_TILES * A_BYTES + ts.bytes();
      const int nk = ceil_div(t.K, BK);
      const int half_rows = ts.rows_gather / GATHER_WARPS;   // a multiple of 4
      const int g_n = half_rows / 4;                          // rows per lane, at most kGatherRowsPerLane
      if (g_n > 0) {
        // Packed rows map to source tokens through b_gather; rows past the
        // segment reuse its first token. A source row outside
        // [0, b_gather_rows) is recorded and replaced by row 0.
        const int r_base = t.b_row0 + t.tt * p.bn_max + (PAIR ? (int)rank * ts.rows_gather : 0) + gw * half_rows;
        const int r_end = t.b_row0 + t.rows;
        for (int i = 0; i < g_n; ++i) {
          const int r = r_base + (lane >> 3) + 4 * i;
          int tok = p.b_gather[r < r_end ? r : t.b_row0];
          if (tok < 0 || (long long)tok >= p.b_gather_rows) {
            if (p.err) atomicOr(p.err, kErrBadIndex);
            tok = 0;
          }
          goff[i * 32 + lane] = (uint32_t)(((long long)tok * t.K + (lane & 7) * 8) * 2);
        }
        __syncwarp();
      }
      // Row r = gw R/2 + lane / 8 + 4i lands at r * 128 in the 128-byte
      // swizzle, its chunk c at (c ^ (r % 8)) * 16.
      const int c = lane & 7;
      const int rb = gw * half_rows + (lane >> 3);
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t u = cur.count;
        uint32_t off, slot, parity;
        cur.take(bytes, cap, off, slot, parity);
        if (!wait_bounded(smem_u32(&acq_bar[slot]), (u / NSLOT) & 1u, abort_flag, p.err, p.timeout_ns, true)) {
          ok = false;
          break;
        }
        if (g_n > 0) {
          const uint32_t bb = smem_u32(ring + off) + A_TILES * A_BYTES;
          const bool in_k = kb * BK + c * 8 < t.K;   // K is a multiple of 8
          const long long koff = in_k ? (long long)kb * BK * 2 : 0;
          const uint32_t src_bytes = in_k ? 16u : 0u;
#pragma unroll
          for (int i = 0; i < kGatherRowsPerLane; ++i)
            if (i < g_n) {
              const int r = rb + 4 * i;
              cp_async_16(bb + (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)), src + goff[i * 32 + lane] + koff,
                          src_bytes);
            }
        }
        cp_async_arrive_noinc(PAIR && !leader ? smem_u32(&gbar[slot]) : smem_u32(&full_bar[slot]));
      }
    }
    cp_async_wait_all();
  } else if (PAIR && gather && warp == 1 && lane == 0 && !leader) {
    // ------------------------------------------------------------ forwarder
    // The peer CTA's gathered rows land in its own shared memory; once all
    // 32 lanes' copies of a slot are done, make them visible to the tensor
    // core's (async) proxy and count them on the leader's full barrier.
    uint32_t u = 0;
    bool ok = true;
    for (int tile = group; tile < total_tiles && ok; tile += ngroups) {
      const Tile t = decode_tile(p, s_off, s_start, nseg, tile, WROWS);
      const int nk = ceil_div(t.K, BK);
      for (int kb = 0; kb < nk; ++kb, ++u) {
        if (!wait_bounded(smem_u32(&gbar[u % NSLOT]), (u / NSLOT) & 1u, abort_flag, p.err, p.timeout_ns,
                          true)) {
          ok = false;
          break;
        }
        fence_proxy_async_smem();
        mbar_arrive_cluster(map_to_cta(smem_u32(&full_bar[u % NSLOT]), 0));
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer
    RingCursor cur;
    AccPlace place;
    uint32_t uses0 = 0, uses1 = 0;   // tiles placed in each TMEM half so far
    bool issued = false;
    for (int tile = group; tile < total_tiles; tile += ngroups) {
      const Tile t = decode_tile(p, s_off, s_start, nseg, tile, WROWS);
      const TokenSlice ts = token_slice<PAIR>(p, t, 0);
      const uint32_t bytes = A_TILES * A_BYTES + ts.bytes();
      const int nk = ceil_div(t.K, BK);
      bool wide;
      uint32_t half;
      place.take(ts.n_mma, wide, half);
      // The half (both for a wide tile) must have been drained by the epilogue.
      bool ok = true;
      if (wide || half == 0u) {
        ok = wait_bounded(smem_u32(&acce_bar[0]), (uses0 & 1u) ^ 1u, abort_flag, p.err, p.timeout_ns, true);
        ++uses0;
      }
      if (ok && (wide || half == 1u)) {
        ok = wait_bounded(smem_u32(&acce_bar[1]), (uses1 & 1u) ^ 1u, abort_flag, p.err, p.timeout_ns, true);
        ++uses1;
      }
      if (!ok) break;
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(PAIR ? 2 * BM : BM, ts.n_mma) | (MODE == kUmmaDgrad ? (1u << 15) : 0u);
      const uint32_t d1 = tmem_base + AccPlace::col0(wide, half);
      const uint32_t d3 = d1 + AccPlace::second(wide);
      for (int kb = 0; kb < nk; ++kb) {
        uint32_t off, slot, parity;
        cur.take(bytes, cap, off, slot, parity);
        if (!wait_bounded(smem_u32(&full_bar[slot]), parity, abort_flag, p.err, p.timeout_ns, true)) {
          ok = false;
          break;
        }
        // Rows gathered with cp.async were written through the generic proxy;
        // the tensor core reads shared memory through the async proxy.
        if (gather) fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t sb = smem_u32(ring + off);
        constexpr bool MN_A = MODE == kUmmaDgrad;
        const uint64_t a_desc = MN_A ? sw128_mn_desc(sb) : sw128_desc(sb);
        const uint64_t a3_desc = MN_A ? sw128_mn_desc(sb + A_BYTES) : sw128_desc(sb + A_BYTES);
        const uint64_t b_desc = sw128_desc(sb + A_TILES * A_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk) {
          const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
          // K-major: the next 16 k are 32 bytes along the row; MN-major: two
          // 8-row k groups (2 x 1024 bytes) further on.
          const uint64_t koff = (uint64_t)((kk * UMMA_K * 2) >> 4);
          const uint64_t koff_a = MN_A ? (uint64_t)((kk * 2 * 1024) >> 4) : koff;
          if (PAIR) {
            umma_bf16_pair(d1, a_desc + koff_a, b_desc + koff, idesc, accum);
            if (A_TILES == 2) umma_bf16_pair(d3, a3_desc + koff_a, b_desc + koff, idesc, accum);
          } else {
            umma_bf16(d1, a_desc + koff_a, b_desc + koff, idesc, accum);
            if (A_TILES == 2) umma_bf16(d3, a3_desc + koff_a, b_desc + koff, idesc, accum);
          }
        }
        issued = true;
        if (PAIR) umma_commit_pair(smem_u32(&empty_bar[slot]), 0x3);
        else umma_commit(smem_u32(&empty_bar[slot]));
      }
      if (!ok) break;
      if (PAIR) umma_commit_pair(smem_u32(&accf_bar[half]), 0x3);
      else umma_commit(smem_u32(&accf_bar[half]));
    }
    if (issued) {   // every MMA this thread issued completes before TMEM is freed
      if (PAIR) umma_commit_pair(smem_u32(drain_bar), 0x1);
      else umma_commit(smem_u32(drain_bar));
      wait_bounded(smem_u32(drain_bar), 0u, abort_flag, p.err, p.timeout_ns, false);
    }
  } else if (warp >= 2 && warp < 2 + EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                  // TMEM lane quarter this warp may read
    const int ch = (warp - 2) >> 2;          // which 16-column chunks: ch, ch + EPI_WPQ, ch + 2 EPI_WPQ, ...
    const int row = q * 32 + lane;
    // The accumulator is released to the leader's barrier (remote for the peer).
    const uint32_t acce0 = PAIR ? map_to_cta(smem_u32(&acce_bar[0]), 0) : smem_u32(&acce_bar[0]);
    AccPlace place;
    uint32_t fills0 = 0, fills1 = 0;   // accumulators consumed from each half so far
    for (int tile = group; tile < total_tiles; tile += ngroups) {
      const Tile t = decode_tile(p, s_off, s_start, nseg, tile, WROWS);
      const TokenSlice ts = token_slice<PAIR>(p, t, 0);
      const int n_valid = ts.n_valid, n_mma = ts.n_mma;
      bool wide;
      uint32_t half;
      place.take(n_mma, wide, half);
      const uint32_t fill_parity = (half ? fills1 : fills0) & 1u;
      if (!wait_bounded(smem_u32(&accf_bar[half]), fill_parity, abort_flag, p.err, p.timeout_ns, true))
        break;
      if (half) ++fills1; else ++fills0;
      tc_fence_after();
      const int m = t.wt * WROWS + (int)rank * BM + row;
      const bool m_ok = m < t.mrows;
      const long long ld = t.dense ? p.out_s_ld : p.out_ld;
      void* out = t.dense ? p.out_s : p.out;
      const long long r0 = (long long)t.b_row0 + (long long)t.tt * p.bn_max;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + AccPlace::col0(wide, half);
      const uint32_t off2 = AccPlace::second(wide);   // second accumulator's column offset
      // Hand TMEM half h back to the MMA warp (after this warp's last read of it).
      auto release_half = [&](uint32_t h) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR) mbar_arrive_cluster(acce0 + h * 8u);
          else mbar_arrive(acce0 + h * 8u);
        }
      };
      // Hand the tile's TMEM back: its half, or both halves for a wide tile.
      auto release = [&]() {
        release_half(half);
        if (wide) release_half(1u);
      };
      // The same for epilogues that already handed half 0 of a wide tile back
      // once its token columns 0..127 (chunks 0..7) were drained.
      auto release_rest = [&]() { release_half(wide ? 1u : half); };
      // Chunk cc of this warp is its last one among chunks 0..7.
      auto last_low_chunk = [&](int cc) { return EPI_WPQ * cc + ch < 8 && EPI_WPQ * (cc + 1) + ch >= 8; };
      if (dual_a(MODE)) {
        // Drain both accumulators into registers as packed bf16 h, hand TMEM
        // back to the MMA warp, then store while the next tile accumulates.
        __nv_bfloat16* pre_a = nullptr;
        __nv_bfloat16* pre_b = nullptr;
        if (MODE == kUmmaSwiGLUSave) {
          pre_a = static_cast<__nv_bfloat16*>(t.dense ? p.pre_a_s : p.pre_a) + r0 * ld;
          pre_b = static_cast<__nv_bfloat16*>(t.dense ? p.pre_b_s : p.pre_b) + r0 * ld;
        }
        uint32_t hp[EPI_CPW * 8];
#pragma unroll
        for (int cc = 0; cc < EPI_CPW; ++cc) {
          const int c = EPI_WPQ * cc + ch;
          if (c < 16 && c * 16 < n_mma) {
            uint32_t r1[16], r3[16];
            tmem_ld16x2_wait(taddr + c * 16, taddr + off2 + c * 16, r1, r3);
            if (MODE == kUmmaSwiGLUSave && m_ok) {
              // Training forward: keep W1 u and W3 u (bf16) for the backward.
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int col = c * 16 + j;
                if (col < n_valid) {
                  pre_a[(long long)col * ld + m] = __float2bfloat16_rn(__uint_as_float(r1[j]));
                  pre_b[(long long)col * ld + m] = __float2bfloat16_rn(__uint_as_float(r3[j]));
                }
              }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float g0 = __uint_as_float(r1[2 * j]), g1 = __uint_as_float(r1[2 * j + 1]);
              // SiLU(g) = g / (1 + e^-g), element by element (a token's h
              // depends on nothing but its own accumulators); the fast divide
              // returns 0 once the denominator passes 2^126, where the exact
              // quotient is below 1e-36.
              const float h0 = __fdividef(g0, 1.0f + __expf(-g0)) * __uint_as_float(r3[2 * j]);
              const float h1 = __fdividef(g1, 1.0f + __expf(-g1)) * __uint_as_float(r3[2 * j + 1]);
              const __nv_bfloat162 hb = __floats2bfloat162_rn(h0, h1);
              hp[cc * 8 + j] = *reinterpret_cast<const uint32_t*>(&hb);
            }
          }
          if (wide && last_low_chunk(cc)) release_half(0u);   // token columns 0..127 drained
        }
        release_rest();
        if (m_ok) {
          unsigned short* o = reinterpret_cast<unsigned short*>(out) + r0 * ld + m;
#pragma unroll
          for (int cc = 0; cc < EPI_CPW; ++cc) {
            const int c = EPI_WPQ * cc + ch;
            if (c < 16 && c * 16 < n_valid) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int col = c * 16 + j;
                if (col < n_valid)
                  o[(long long)col * ld] = (unsigned short)(hp[cc * 8 + (j >> 1)] >> ((j & 1) * 16));
              }
            }
          }
        }
      } else if (MODE == kUmmaDgrad && p.out_f32) {
        // Two 128-row blocks, BLOCK_STEP apart; fp32 output.
        const int m2 = m + BLOCK_STEP;
        const bool m2_ok = m2 < t.mrows;
        float* o = reinterpret_cast<float*>(out) + r0 * ld;
        for (int c0 = ch * 16; c0 < n_mma; c0 += 16 * EPI_WPQ) {
          uint32_t r1[16], r3[16];
          tmem_ld16x2_wait(taddr + c0, taddr + off2 + c0, r1, r3);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c0 + j;
            if (col < n_valid) {
              if (m_ok) o[(long long)col * ld + m] = __uint_as_float(r1[j]);
              if (m2_ok) o[(long long)col * ld + m2] = __uint_as_float(r3[j]);
            }
          }
        }
        release();
      } else if (MODE == kUmmaDown) {
        // Two 128-row blocks of W2, BLOCK_STEP apart. Both accumulators are
        // drained into packed bf16 registers first, TMEM goes back to the MMA
        // warp, and the stores run while the next tile accumulates (down
        // tiles are short, 32 k-steps at f = 2048, so a TMEM hold over the
        // stores would stop the weight stream for a large share of a tile).
        const int m2 = m + BLOCK_STEP;
        const bool m2_ok = m2 < t.mrows;
        uint32_t q1[EPI_CPW * 8], q2[EPI_CPW * 8];
#pragma unroll
        for (int cc = 0; cc < EPI_CPW; ++cc) {
          const int c = EPI_WPQ * cc + ch;
          if (c < 16 && c * 16 < n_mma) {
            uint32_t r1[16], r3[16];
            tmem_ld16x2_wait(taddr + c * 16, taddr + off2 + c * 16, r1, r3);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const __nv_bfloat162 pa = __floats2bfloat162_rn(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
              const __nv_bfloat162 pb = __floats2bfloat162_rn(__uint_as_float(r3[2 * j]), __uint_as_float(r3[2 * j + 1]));
              q1[cc * 8 + j] = *reinterpret_cast<const uint32_t*>(&pa);
              q2[cc * 8 + j] = *reinterpret_cast<const uint32_t*>(&pb);
            }
          }
          if (wide && last_low_chunk(cc)) release_half(0u);   // token columns 0..127 drained
        }
        release_rest();
        unsigned short* o = reinterpret_cast<unsigned short*>(out) + r0 * ld;
#pragma unroll
        for (int cc = 0; cc < EPI_CPW; ++cc) {
          const int c = EPI_WPQ * cc + ch;
          if (c < 16 && c * 16 < n_valid) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int col = c * 16 + j;
              if (col < n_valid) {
                const int sh = (j & 1) * 16;
                if (m_ok) o[(long long)col * ld + m] = (unsigned short)(q1[cc * 8 + (j >> 1)] >> sh);
                if (m2_ok) o[(long long)col * ld + m2] = (unsigned short)(q2[cc * 8 + (j >> 1)] >> sh);
              }
            }
          }
        }
      } else if (MODE == kUmmaDgrad) {
        // Two 128-row blocks, BLOCK_STEP apart; bf16 output.
        const int m2 = m + BLOCK_STEP;
        const bool m2_ok = m2 < t.mrows;
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + r0 * ld;
        for (int c0 = ch * 16; c0 < n_mma; c0 += 16 * EPI_WPQ) {
          uint32_t r1[16], r3[16];
          tmem_ld16x2_wait(taddr + c0, taddr + off2 + c0, r1, r3);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c0 + j;
            if (col < n_valid) {
              if (m_ok) o[(long long)col * ld + m] = __float2bfloat16_rn(__uint_as_float(r1[j]));
              if (m2_ok) o[(long long)col * ld + m2] = __float2bfloat16_rn(__uint_as_float(r3[j]));
            }
          }
        }
        release();
      } else if (MODE == kUmmaBiasAct) {
        // As the bf16 input gradients, with the weight row's bias added and the
        // activation applied in fp32 before the one rounding to bf16.
        const int m2 = m + BLOCK_STEP;
        const bool m2_ok = m2 < t.mrows;
        const float* rb = t.dense ? p.row_bias_s : p.row_bias;
        const long long boff = t.dense ? 0 : (long long)t.seg * p.m_rows;
        const float bias1 = (rb && m_ok) ? rb[boff + m] : 0.0f;
        const float bias2 = (rb && m2_ok) ? rb[boff + m2] : 0.0f;
        const bool gelu = p.act == kActGelu;
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + r0 * ld;
        for (int c0 = ch * 16; c0 < n_mma; c0 += 16 * EPI_WPQ) {
          uint32_t r1[16], r3[16];
          tmem_ld16x2_wait(taddr + c0, taddr + off2 + c0, r1, r3);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c0 + j;
            if (col < n_valid) {
              float v1 = __uint_as_float(r1[j]) + bias1;
              float v2 = __uint_as_float(r3[j]) + bias2;
              if (gelu) { v1 = gelu_erf(v1); v2 = gelu_erf(v2); }
              if (m_ok) o[(long long)col * ld + m] = __float2bfloat16_rn(v1);
              if (m2_ok) o[(long long)col * ld + m2] = __float2bfloat16_rn(v2);
            }
          }
        }
        release();
      }
    }
  }
  tc_fence_before();
  if (PAIR) cluster_sync_all(); else __syncthreads();   // peer smem and TMEM stay live until here
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

__global__ void wait_timeout_selftest_kernel(uint32_t* err, long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: phase 0 never completes, the wait runs out.
  if (threadIdx.x == 0)
    wait_bounded(smem_u32(&bar), 0u, &abort_flag, err, timeout_ns, false);
  __syncthreads();
}

// ------------------------------------------------------------ host side
template <int MODE, bool PAIR>
cudaError_t ensure_smem_attr() {
  static int done_mask = 0;   // one bit per device ordinal (< 32)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 32 && ((done_mask >> dev) & 1)) return cudaSuccess;
  e = cudaFuncSetAttribute(umma_gemm_kernel<MODE, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           SMEM_LIMIT);
  if (e == cudaSuccess && dev < 32) done_mask |= 1 << dev;
  return e;
}

template <int MODE, bool PAIR>
cudaError_t launch_mode(const CUtensorMap& tA, const CUtensorMap& tA3, const CUtensorMap& tB,
                        const CUtensorMap& tAs, const CUtensorMap& tA3s, const CUtensorMap& tBs,
                        const UmmaLaunch& p, int grid, int smem,
                        cudaStream_t s) {
  cudaError_t e = ensure_smem_attr<MODE, PAIR>();
  if (e != cudaSuccess) return e;
  const int threads = (p.b_gather || p.split_b) ? NUM_THREADS_GATHER : NUM_THREADS;
  if (!PAIR) {
    umma_gemm_kernel<MODE, false><<<grid, threads, smem, s>>>(tA, tA3, tB, tAs, tA3s, tBs, p);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, umma_gemm_kernel<MODE, true>, tA, tA3, tB, tAs, tA3s, tBs, p);
}

}  // namespace

cudaError_t launch_umma_gemm(const UmmaGemmParams& p, int num_sms, cudaStream_t s) {
  const bool has_dense = p.shared_rows > 0;
  if (p.n_routed == 0 && !has_dense) return cudaSuccess;
  if (p.bn_max < 16 || p.bn_max > BN_MAX || p.bn_max % 16) return cudaErrorInvalidValue;
  const int nseg = p.n_routed + (has_dense ? 1 : 0);
  const SmemPlan sp = smem_plan(p.n_routed, nseg);
  const int a_tiles = 2;
  // Wide token tiles run on CTA pairs (M=256 MMAs: each CTA stages half the
  // token tile, halving token traffic per weight byte). Narrow tiles (decode)
  // stay on single CTAs.
  const bool pair = p.bn_max >= 128 && num_sms >= 2;
  const int wrows = tile_rows(p.mode, pair);
  UmmaLaunch q;
  static_cast<UmmaGemmParams&>(q) = p;
  // One copy of B per CTA and slot: a box as tall as the most token rows a
  // CTA stages (rounded to the 8-row swizzle atom), at most 128 rows.
  const int mine_max = pair ? p.bn_max / 2 : p.bn_max;
  q.box_n = ((mine_max + 7) & ~7) < BOX_N_MAX ? ((mine_max + 7) & ~7) : BOX_N_MAX;
  // Second issuing thread on CTA pairs (wide token tiles), where a slot's
  // copies are many bytes and the issuing thread paces the stream; single
  // CTAs (decode) stage a few token rows per slot and keep one issuer.
  q.split_b = (p.b_gather || !pair) ? 0 : kSplitB;
  if (sp.ring_bytes < 2 * (a_tiles * A_BYTES + ceil_div(mine_max, q.box_n) * q.box_n * BK * 2))
    return cudaErrorInvalidValue;
  const bool swiglu = dual_a(p.mode);
  const bool dgrad = p.mode == kUmmaDgrad;
  CUtensorMap tA, tA3, tB, tAs, tA3s, tBs;
  if (has_dense) {
    if (dgrad) {   // stored weight [a_k_rows_s][m_rows_s], m contiguous: 64 x 64 boxes
      if (!make_tmap(&tAs, p.a_s, p.m_rows_s, p.a_k_rows_s, 64)) return cudaErrorInvalidValue;
      if (!make_tmap(&tA3s, p.a3_s ? p.a3_s : p.a_s, p.m_rows_s, p.a_k_rows_s, 64)) return cudaErrorInvalidValue;
    } else {
      if (!make_tmap(&tAs, p.a_s, p.K_s, p.m_rows_s, BM)) return cudaErrorInvalidValue;
      if (swiglu && !make_tmap(&tA3s, p.a3_s, p.K_s, p.m_rows_s, BM)) return cudaErrorInvalidValue;
      if (!swiglu) tA3s = tAs;
    }
    if (!make_tmap(&tBs, p.b_s, p.K_s, p.shared_rows, q.box_n)) return cudaErrorInvalidValue;
  }
  if (p.n_routed > 0) {
    if (dgrad) {   // stacked weights [n_routed * a_k_rows][m_rows], m contiguous
      if (!make_tmap(&tA, p.a, p.m_rows, p.a_rows_total, 64)) return cudaErrorInvalidValue;
      if (!make_tmap(&tA3, p.a3 ? p.a3 : p.a, p.m_rows, p.a_rows_total, 64)) return cudaErrorInvalidValue;
    } else {
      if (!make_tmap(&tA, p.a, p.K, p.a_rows_total, BM)) return cudaErrorInvalidValue;
      if (swiglu && !make_tmap(&tA3, p.a3, p.K, p.a_rows_total, BM)) return cudaErrorInvalidValue;
      if (!swiglu) tA3 = tA;
    }
    if (!make_tmap(&tB, p.b, p.K, p.b_rows_total, q.box_n)) return cudaErrorInvalidValue;
  } else {
    tA = tAs; tA3 = tA3s; tB = tBs;
  }
  if (!has_dense) { tAs = tA; tA3s = tA3; tBs = tB; }
  // Gathered token rows are copied with cp.async: the source rows must be
  // 16-byte aligned.
  if (p.b_gather && (p.mode != kUmmaSwiGLU || !p.b_gather_src || p.b_gather_rows <= 0 ||
                     (reinterpret_cast<uintptr_t>(p.b_gather_src) & 15u) || (p.K * 2) % 16 ||
                     mine_max > GATHER_WARPS * 4 * kGatherRowsPerLane || p.b_gather_rows * p.K * 2 > 0xffffffffll))
    return cudaErrorInvalidValue;

  long long tiles = 0;
  if (p.n_routed > 0)
    tiles += (long long)ceil_div(p.m_rows, wrows) * (ceil_div(p.max_routed_rows, p.bn_max) + p.n_routed);
  if (has_dense) tiles += (long long)ceil_div(p.m_rows_s, wrows) * ceil_div(p.shared_rows, p.bn_max);
  const int groups = pair ? num_sms / 2 : num_sms;
  const int ngroup = (int)(tiles < groups ? tiles : groups);
  if (ngroup <= 0) return cudaSuccess;
  const int grid = pair ? 2 * ngroup : ngroup;
  switch (p.mode) {
    case kUmmaSwiGLU:
      return pair ? launch_mode<kUmmaSwiGLU, true>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s)
                  : launch_mode<kUmmaSwiGLU, false>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s);
    case kUmmaSwiGLUSave:
      return pair ? launch_mode<kUmmaSwiGLUSave, true>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s)
                  : launch_mode<kUmmaSwiGLUSave, false>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s);
    case kUmmaDown:
      return pair ? launch_mode<kUmmaDown, true>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s)
                  : launch_mode<kUmmaDown, false>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s);
    case kUmmaBiasAct:
      return pair ? launch_mode<kUmmaBiasAct, true>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s)
                  : launch_mode<kUmmaBiasAct, false>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s);
    case kUmmaDgrad:
      return pair ? launch_mode<kUmmaDgrad, true>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s)
                  : launch_mode<kUmmaDgrad, false>(tA, tA3, tB, tAs, tA3s, tBs, q, grid, sp.total, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_wait_timeout_selftest(uint32_t* err, long long timeout_ns, cudaStream_t s) {
  wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace moe
