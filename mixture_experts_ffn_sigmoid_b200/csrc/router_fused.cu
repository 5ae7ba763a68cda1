// The router of the block in one kernel (bf16 inputs, up to 256 experts):
// logits, affinities, biased group-limited top-k, gates, per-expert counts
// and packing offsets.
//
//   l[t][e] = sum_c x[t][c] w_router[e][c]         (the router linear: the
//     Sparse MoE FFN note's Routing paragraph, u_t . e_i; the MoE cheat
//     sheet's "The router in code": one dot product per router row)
//   then per token the biased, group-limited top-k and the gates of
//   route_topk.cuh, and the counts and offsets that pack every token's rows
//   expert by expert, tokens in order (the note's "Packed forward
//   (official)": each expert gathers the tokens that chose it).
//
// One 128-token tile per cluster of S CTAs (S = 1, 2, 4 or 8). CTA r of the
// cluster runs its share of the contraction on the tensor cores: TMA stages
// x and w_router tiles (128-byte swizzle) into a 4-stage ring, one lane
// issues tcgen05.mma (kind::f16, M = 128 tokens, N = the expert count
// rounded up to 16, fp32 accumulator in TMEM). The 32 warps then copy the
// partial logits from TMEM into the CTA's shared memory (over the ring,
// which is no longer needed), and after a cluster barrier the CTAs add the
// S partial sums through distributed shared memory in rank order (a fixed
// order: the logits are the same bits on every run). The tile's tokens are
// shared among the CTAs' warps (one warp per token, token tl on CTA tl % S),
// and per-expert bit masks record which tokens of each 32-token chunk chose
// each expert. CTA 0 ORs the CTAs' masks and turns them into each chunk's
// base within the tile and the tile's histogram. The last tile to finish (a device-wide counter)
// scans the tile histograms into each tile's base, the per-expert counts
// and the offsets. A token's packed row is then
//   offsets[e] + tile_base[tile][e] + chunk_base[chunk][e] + (earlier tokens
//   of its chunk that chose e),
// which the permute kernel computes.
//
// No fp32 partial logits go through HBM; the summed logits are written once
// ([T][E], kept for the backward pass). Every mbarrier wait is bounded; on
// expiry the CTA records the timeout in the error word and still reaches
// every cluster barrier, so no CTA waits for an aborted peer.
#include "route_topk.cuh"
#include "umma_common.cuh"

namespace moe {
namespace {

constexpr int FR_BM = 128;                        // tokens per tile (one cluster)
constexpr int FR_BK = 64;
constexpr int FR_STAGES = 4;
constexpr int FR_THREADS = 1024;                  // 32 warps: one token each when routing
constexpr int FR_BN_MAX = 256;
constexpr int FR_A_BYTES = FR_BM * FR_BK * 2;     // 16 KB of x per stage
constexpr int FR_HDR = 1024;
constexpr int FR_TMEM_COLS = 256;

static_assert(FR_BM == kTileChunks * kChunk, "a tile is kTileChunks chunks");

struct FusedRouterArgs {
  int T, E, K;
  int n_pad;          // MMA N: E rounded up to 16
  int kb_per_split;   // 64-wide k blocks per CTA of a cluster
  int ntiles;
  TopkArgs topk;
  float* logits;      // [T][E] summed router logits
  int* topk_idx;      // [T][k]
  float* topk_gate;   // [T][k]
  int* chunk_base;    // [ceil(T/32)][E]: base of each chunk within its tile
  int* tile_hist;     // [ntiles][E]
  int* tile_base;     // [ntiles][E]: base of each tile
  int* counts;        // [E]
  int* offsets;       // [E + 1]
  uint32_t* err;
  uint32_t* done_count;   // zero before the launch; the last tile sets it back to zero
  long long timeout_ns;
  // With one tile (T <= 128) and these set, the row maps of the permute as
  // well: inv_row [T][k] (each token's packed rows) and perm_src [T * k]
  // (each packed row's token).
  int* inv_row;
  int* perm_src;
};

__host__ __device__ inline int fr_stage_bytes(int n_pad) { return FR_A_BYTES + n_pad * FR_BK * 2; }
__host__ __device__ inline int fr_smem_bytes(int n_pad) {
  // alignment slack, header, ring (also the partial-logit buffer), the tile's
  // chunk masks [kTileChunks][256], the scan's partial sums [4][256], the
  // selection bias [256] and the tile's chunk bases [kTileChunks][256]
  return 1024 + FR_HDR + FR_STAGES * fr_stage_bytes(n_pad) + kTileChunks * 256 * 4 + 4 * 256 * 4 + 256 * 4 +
         kTileChunks * 256 * 4 + 256;
}

// NPL consecutive fp32 values (NPL = 1, 2, 4 or 8) from the shared memory of
// a CTA of the cluster; the address is aligned to min(NPL, 4) * 4 bytes.
template <int NPL>
__device__ __forceinline__ void ld_cluster_vec(uint32_t a, float (&v)[NPL]) {
  if constexpr (NPL == 1) {
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v[0]) : "r"(a) : "memory");
  } else if constexpr (NPL == 2) {
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v[0]), "=f"(v[1]) : "r"(a) : "memory");
  } else {
#pragma unroll
    for (int h = 0; h < NPL / 4; ++h)
      asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                   : "=f"(v[4 * h]), "=f"(v[4 * h + 1]), "=f"(v[4 * h + 2]), "=f"(v[4 * h + 3])
                   : "r"(a + 16u * h) : "memory");
  }
}
// The same number of values to this CTA's shared memory, same alignment.
template <int NPL>
__device__ __forceinline__ void st_shared_vec(float* dst, const float (&v)[NPL]) {
  if constexpr (NPL == 1) {
    dst[0] = v[0];
  } else if constexpr (NPL == 2) {
    *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
  } else {
#pragma unroll
    for (int h = 0; h < NPL / 4; ++h)
      reinterpret_cast<float4*>(dst)[h] = make_float4(v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]);
  }
}

template <int NPL>
__global__ void __launch_bounds__(FR_THREADS, 1)
    router_fused_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                        const FusedRouterArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty_bar = full_bar + FR_STAGES;
  uint64_t* done_bar = empty_bar + FR_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* s_ok = reinterpret_cast<volatile int*>(tmem_slot + 3);
  int* s_warp = reinterpret_cast<int*>(tmem_slot + 4);          // [32]
  uint8_t* ring = smem + FR_HDR;
  const int stage_bytes = fr_stage_bytes(p.n_pad);
  float* s_log = reinterpret_cast<float*>(ring);                // [128][ld_log] after the MMAs
  const int ld_log = p.n_pad + 4;                               // 16-byte rows, conflict-free float4 stores
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(ring + FR_STAGES * stage_bytes);   // [kTileChunks][256]
  int* s_part = reinterpret_cast<int*>(s_mask + kTileChunks * 256);                 // [4][256]
  float* s_bias = reinterpret_cast<float*>(s_part + 4 * 256);                       // [256]
  int* s_cbase = reinterpret_cast<int*>(s_bias + 256);                               // [kTileChunks][256]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t S = cluster_ncta();
  const int tile = (int)(blockIdx.x / S);
  const int t0 = tile * FR_BM;
  const int E = p.E;
  const int nkb = ceil_div(p.K, FR_BK);
  const int kb0 = (int)rank * p.kb_per_split;
  const int kb1 = min(nkb, kb0 + p.kb_per_split);
  const int nk = max(0, kb1 - kb0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < FR_STAGES; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    mbar_init(smem_u32(done_bar), 1);
    *abort_flag = 0u;
    fence_mbar_init();
    tmap_prefetch(&tmX);
    tmap_prefetch(&tmW);
  }
  for (int i = threadIdx.x; i < kTileChunks * 256; i += blockDim.x) s_mask[i] = 0u;
  if (p.topk.bias)   // every token of the tile reads all of it
    for (int i = threadIdx.x; i < E; i += blockDim.x) s_bias[i] = p.topk.bias[i];
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), FR_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // ------------------------------------------------------------ partial logits
  if (warp == 0 && lane == 0) {
    // producer: x [128 tokens][64] and w_router [n_pad experts][64] per k block
    int n_issued = 0;
    for (int i = 0; i < nk; ++i) {
      const int stage = i % FR_STAGES;
      const uint32_t parity = ((i / FR_STAGES) & 1u) ^ 1u;
      if (!wait_bounded(smem_u32(&empty_bar[stage]), parity, abort_flag, p.err, p.timeout_ns, true)) break;
      const uint32_t fb = smem_u32(&full_bar[stage]);
      const uint32_t sa = smem_u32(ring + stage * stage_bytes);
      mbar_expect_tx(fb, (uint32_t)stage_bytes);   // whole boxes; rows past T or E read as zeros
      tma_load_2d(sa, &tmX, (kb0 + i) * FR_BK, t0, fb);
      tma_load_2d(sa + FR_A_BYTES, &tmW, (kb0 + i) * FR_BK, 0, fb);
      n_issued = i + 1;
    }
    // Every copy this thread started has landed before the ring is reused
    // for the partial logits (on an abort some may not have been consumed).
    for (int i = max(0, n_issued - FR_STAGES); i < n_issued; ++i)
      wait_bounded(smem_u32(&full_bar[i % FR_STAGES]), (i / FR_STAGES) & 1u, abort_flag, p.err, p.timeout_ns,
                   false);
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer
      bool issued = false;
      const uint32_t idesc = idesc_bf16_f32(FR_BM, p.n_pad);
      for (int i = 0; i < nk; ++i) {
        const int stage = i % FR_STAGES;
        if (!wait_bounded(smem_u32(&full_bar[stage]), (i / FR_STAGES) & 1u, abort_flag, p.err, p.timeout_ns,
                          true))
          break;
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + stage * stage_bytes);
        const uint64_t a_desc = sw128_desc(sa);
        const uint64_t b_desc = sw128_desc(sa + FR_A_BYTES);
#pragma unroll
        for (int kk = 0; kk < FR_BK / 16; ++kk) {
          const uint64_t koff = (uint64_t)((kk * 32) >> 4);
          umma_bf16(tmem_base, a_desc + koff, b_desc + koff, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&empty_bar[stage]));
        issued = true;
      }
      if (issued) umma_commit(smem_u32(done_bar));   // completion of every MMA releases the drain
      else mbar_arrive(smem_u32(done_bar));
    }
    __syncwarp();
  } else if (warp == 2 && lane == 0) {
    // One thread waits for the MMAs; the other threads wait in the block
    // barrier below instead of polling the mbarrier.
    *s_ok = wait_bounded(smem_u32(done_bar), 0u, abort_flag, p.err, p.timeout_ns, false) ? 1 : 0;
  }
  __syncthreads();      // MMAs complete, and the producer's copies have landed: the ring may be overwritten
  tc_fence_after();
  const bool ok = *s_ok != 0;
  // TMEM -> shared memory: warp w reads lane quarter w & 3 (32 tokens) and
  // 32 columns starting at 32 * (w >> 2).
  {
    const int q = warp & 3, c0 = (warp >> 2) * 32;
    if (c0 < p.n_pad) {
      uint32_t ra[16], rb[16];
      if (ok && nk > 0) {
        const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c0;
        tmem_ld16x2_wait(ta, ta + 16, ra, rb);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) { ra[j] = 0u; rb[j] = 0u; }   // empty share (or a failed wait): zeros
      }
      float* row = s_log + (q * 32 + lane) * ld_log + c0;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        reinterpret_cast<float4*>(row)[j] = make_float4(__uint_as_float(ra[4 * j]), __uint_as_float(ra[4 * j + 1]),
                                                        __uint_as_float(ra[4 * j + 2]), __uint_as_float(ra[4 * j + 3]));
      if (c0 + 16 < p.n_pad) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          reinterpret_cast<float4*>(row + 16)[j] =
              make_float4(__uint_as_float(rb[4 * j]), __uint_as_float(rb[4 * j + 1]), __uint_as_float(rb[4 * j + 2]),
                          __uint_as_float(rb[4 * j + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, FR_TMEM_COLS);
  }
  cluster_sync_all();   // every CTA's partial logits are in its shared memory

  // ------------------------------------------------------------ routing
  // Token tl of the tile is routed by CTA tl % S, warp (tl / S) % 32, so a
  // short tile (decode) spreads its tokens over every CTA of the cluster
  // rather than queueing them on one SM. Each CTA records, per chunk, which
  // of the tokens it routed chose each expert; CTA 0 ORs those masks below.
  const int nch_tile = min(kTileChunks, ceil_div(p.T - t0, kChunk));
  const int tile_tokens = min(FR_BM, p.T - t0);
  const int k = p.topk.k;
  TopkArgs tk = p.topk;
  if (tk.bias) tk.bias = s_bias;
  // route_token takes lane l's experts l*NPL .. l*NPL + NPL - 1 (its blocked
  // layout); columns past n_pad are not there, and columns E .. n_pad - 1
  // hold zeros the routing ignores.
  for (int tl = (int)rank + (int)S * warp; tl < tile_tokens; tl += (int)S * 32) {
    const int t = t0 + tl;
    const int j = tl / kChunk;
    {   // one warp, one token
      // Partial sums, CTA by CTA in rank order; the shares of up to QB CTAs
      // are requested before the first of them is added (QB * NPL values in
      // registers). Each load instruction of the warp reads one contiguous
      // run of the row (lane l: columns 4l .. 4l + 3 of each 128-column
      // half with eight per lane), so no two lanes share a bank; with eight
      // per lane the sums then go through this CTA's row into the blocked
      // layout.
      constexpr uint32_t QB = NPL >= 8 ? 4 : 8;
      constexpr int VW = NPL >= 4 ? 4 : NPL;       // values per vector
      float lg[NPL];
      float* own = s_log + tl * ld_log;
      auto col = [&](int h) { return NPL >= 8 ? 128 * h + 4 * lane : lane * NPL; };
      bool hv[NPL / VW];
#pragma unroll
      for (int h = 0; h < NPL / VW; ++h) hv[h] = col(h) < p.n_pad;
#pragma unroll
      for (int i = 0; i < NPL; ++i) lg[i] = 0.0f;
#pragma unroll
      for (uint32_t q0 = 0; q0 < 8; q0 += QB) {
        if (q0 < S) {
          float part[QB][NPL];
#pragma unroll
          for (uint32_t b = 0; b < QB; ++b) {
#pragma unroll
            for (int h = 0; h < NPL / VW; ++h) {
              float* dst = &part[b][h * VW];
              if (hv[h] && q0 + b < S) {
                ld_cluster_vec<VW>(map_to_cta(smem_u32(own + col(h)), q0 + b),
                                   *reinterpret_cast<float(*)[VW]>(dst));
              } else {
#pragma unroll
                for (int i = 0; i < VW; ++i) dst[i] = 0.0f;
              }
            }
          }
#pragma unroll
          for (uint32_t b = 0; b < QB; ++b) {
            if (q0 + b < S) {
#pragma unroll
              for (int i = 0; i < NPL; ++i) lg[i] = q0 + b == 0 ? part[b][i] : lg[i] + part[b][i];
            }
          }
        }
      }
      // The sums replace this CTA's own partials of the token (a token's
      // rows are read only by the CTA that routes it), to be copied out after
      // the handshake.
#pragma unroll
      for (int h = 0; h < NPL / VW; ++h)
        if (hv[h]) st_shared_vec<VW>(own + col(h), *reinterpret_cast<const float(*)[VW]>(&lg[h * VW]));
      if constexpr (NPL >= 8) {   // into the blocked layout
        __syncwarp();
        const bool have = lane * NPL < p.n_pad;
#pragma unroll
        for (int h = 0; h < NPL / 4; ++h) {
          const float4 v = have ? reinterpret_cast<const float4*>(own + lane * NPL)[h] : make_float4(0.f, 0.f, 0.f, 0.f);
          lg[4 * h] = v.x; lg[4 * h + 1] = v.y; lg[4 * h + 2] = v.z; lg[4 * h + 3] = v.w;
        }
      }
      int my_e, pos;
      float gate;
      route_token<NPL>(lg, lane, tk, my_e, pos, gate, own);
      if (lane < k) {
        p.topk_idx[(size_t)t * k + pos] = my_e;
        p.topk_gate[(size_t)t * k + pos] = gate;
        atomicOr(&s_mask[j * 256 + my_e], 1u << (tl % kChunk));
      }
    }
  }
  __syncthreads();
  cluster_sync_all();   // chunk masks complete; no CTA reads a peer's logits any more

  // ------------------------------------------------------------ tile histogram (CTA 0)
  if (rank == 0) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      // every CTA's masks of every chunk requested before any is used
      uint32_t m[kTileChunks];
#pragma unroll
      for (int j = 0; j < kTileChunks; ++j) m[j] = 0u;
#pragma unroll
      for (uint32_t q = 0; q < 8; ++q) {
        if (q < S) {
#pragma unroll
          for (int j = 0; j < kTileChunks; ++j)
            if (j < nch_tile) m[j] |= ld_cluster_u32(map_to_cta(smem_u32(&s_mask[j * 256 + e]), q));
        }
      }
      int run = 0;
#pragma unroll
      for (int j = 0; j < kTileChunks; ++j) {
        if (j < nch_tile) {
          p.chunk_base[(size_t)(tile * kTileChunks + j) * E + e] = run;
          if (p.inv_row) {   // kept for the row maps: this thread's own entries
            s_mask[j * 256 + e] = m[j];
            s_cbase[j * 256 + e] = run;
          }
          run += __popc(m[j]);
        }
      }
      p.tile_hist[(size_t)tile * E + e] = run;
    }
  }
  cluster_sync_all();   // CTA 0 has read its peers' masks: they may exit

  // The summed logits of the tokens this CTA routed ([T][E] fp32, kept for
  // the backward pass), one warp per token row. CTA 0 first publishes its
  // tile histogram (and, on the last tile, runs the scan), so neither waits
  // on these stores.
  auto store_logits = [&]() {
    for (int tl = (int)rank + (int)S * warp; tl < tile_tokens; tl += (int)S * 32)
      for (int e = lane; e < E; e += 32) p.logits[(size_t)(t0 + tl) * E + e] = s_log[tl * ld_log + e];
  };
  if (rank != 0) {
    store_logits();
    return;
  }

  // ------------------------------------------------------------ last tile: scan
  // The block barrier orders every thread's chunk bases and tile-histogram
  // stores before thread 0's fence (a cumulative gpu-scope fence), which
  // orders them before the counter increment that publishes them. On the
  // last tile thread 0 fences again after reading the counter, and the block
  // barrier after it passes that ordering on to every thread, so the other
  // tiles' histograms are visible to the scan. (One fence per CTA: a fence
  // in each of the 1024 threads costs microseconds.)
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(p.done_count, 1u);
    const bool last = prev == (uint32_t)(p.ntiles - 1);
    if (last) __threadfence();
    *s_last = last ? 1 : 0;
  }
  __syncthreads();
  if (!*s_last) {
    store_logits();
    return;
  }
  // Four groups of 256 threads, each over a quarter of the tiles: its partial
  // per-expert sums, then each tile's base from the groups before it.
  const int g = threadIdx.x >> 8, e = threadIdx.x & 255;
  // Loads go out eight at a time before any is added; with at most eight
  // tiles per group (up to 32 tiles) they stay in registers for the bases.
  constexpr int kBatch = 8;
  const int per = ceil_div(p.ntiles, 4);
  const int i0 = min(p.ntiles, g * per), i1 = min(p.ntiles, i0 + per);
  int h[kBatch];
  int part = 0;
  if (e < E)
    for (int i = i0; i < i1; i += kBatch) {
#pragma unroll
      for (int u = 0; u < kBatch; ++u) h[u] = i + u < i1 ? __ldcg(&p.tile_hist[(size_t)(i + u) * E + e]) : 0;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) part += h[u];
    }
  s_part[g * 256 + e] = part;
  __syncthreads();
  if (e < E) {
    int run = 0;
    for (int gg = 0; gg < g; ++gg) run += s_part[gg * 256 + e];
    for (int i = i0; i < i1; i += kBatch) {
      if (per > kBatch) {   // the registers hold the last batch only: reload
#pragma unroll
        for (int u = 0; u < kBatch; ++u) h[u] = i + u < i1 ? __ldcg(&p.tile_hist[(size_t)(i + u) * E + e]) : 0;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (i + u < i1) p.tile_base[(size_t)(i + u) * E + e] = run;
        run += h[u];
      }
    }
  }
  // Counts, then offsets = exclusive scan of the counts over experts (threads 0..255).
  int cnt = 0;
  if (g == 0 && e < E) {
    cnt = s_part[e] + s_part[256 + e] + s_part[512 + e] + s_part[768 + e];
    p.counts[e] = cnt;
  }
  int incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (g == 0 && lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (g == 0) {
    int before = 0;
    for (int w = 0; w < warp; ++w) before += s_warp[w];
    if (e < E) {
      p.offsets[e] = before + incl - cnt;
      s_part[e] = before + incl - cnt;   // the partial sums are no longer read
    }
    if (e == 0) {
      int total = 0;
      for (int w = 0; w < 8; ++w) total += s_warp[w];
      p.offsets[E] = total;
      *p.done_count = 0u;   // ready for the next launch
    }
  }
  if (p.inv_row) {
    // One tile: the rows of token t, j-th choice e = offsets[e] + its chunk's
    // base for e + the earlier tokens of its chunk that chose e (the tile's
    // base is zero). The other CTAs' index stores are visible after the
    // cluster barriers; read them from L2.
    __syncthreads();
    for (int i = threadIdx.x; i < tile_tokens * k; i += blockDim.x) {
      const int tl = i / k;
      const int e = __ldcg(&p.topk_idx[(size_t)(t0 + tl) * k + (i - tl * k)]);
      const int c = tl / kChunk;
      const int row = s_part[e] + s_cbase[c * 256 + e] + __popc(s_mask[c * 256 + e] & ((1u << (tl % kChunk)) - 1u));
      p.inv_row[(size_t)(t0 + tl) * k + (i - tl * k)] = row;
      p.perm_src[row] = t0 + tl;
    }
  }
  store_logits();
}

}  // namespace

bool router_fused_supported(int dtype, int E) { return dtype == MOE_DTYPE_BF16 && E >= 1 && E <= FR_BN_MAX; }

// CTAs per tile: the largest of 8, 4, 2, 1 that keeps every CTA at least one
// k block and the grid within B200's 148 SMs (one CTA per SM). A function of
// the shape only.
int router_fused_cluster(int T, int K) {
  constexpr int num_sms = 148;
  const int ntiles = ceil_div(T, FR_BM);
  const int nkb = ceil_div(K, FR_BK);
  int s = 8;
  while (s > 1 && (s > nkb || ntiles * s > num_sms)) s >>= 1;
  return s;
}

cudaError_t launch_router_fused(const FusedRouterLaunch& a, cudaStream_t s) {
  if (a.T <= 0) return cudaSuccess;
  if (!router_fused_supported(MOE_DTYPE_BF16, a.E)) return cudaErrorInvalidValue;
  const int n_pad = (a.E + 15) / 16 * 16;
  CUtensorMap tX, tW;
  if (!make_tmap(&tX, a.x, a.K, a.T, FR_BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&tW, a.w_router, a.K, a.E, n_pad)) return cudaErrorInvalidValue;
  const int smem = fr_smem_bytes(n_pad);
  const int npl = ceil_div(a.E, 32);
  auto kernel = npl <= 1 ? router_fused_kernel<1>
              : npl <= 2 ? router_fused_kernel<2>
              : npl <= 4 ? router_fused_kernel<4>
                         : router_fused_kernel<8>;
  static int attr_done[4] = {0, 0, 0, 0};   // one bit per device ordinal (< 32), per instantiation
  const int which = npl <= 1 ? 0 : npl <= 2 ? 1 : npl <= 4 ? 2 : 3;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!(dev < 32 && ((attr_done[which] >> dev) & 1))) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fr_smem_bytes(FR_BN_MAX));
    if (e != cudaSuccess) return e;
    if (dev < 32) attr_done[which] |= 1 << dev;
  }
  FusedRouterArgs p = {};
  p.T = a.T; p.E = a.E; p.K = a.K;
  p.n_pad = n_pad;
  const int S = router_fused_cluster(a.T, a.K);
  p.kb_per_split = ceil_div(ceil_div(a.K, FR_BK), S);
  p.ntiles = ceil_div(a.T, FR_BM);
  p.topk = a.topk;
  p.logits = a.logits;
  p.topk_idx = a.topk_idx; p.topk_gate = a.topk_gate;
  p.chunk_base = a.chunk_base; p.tile_hist = a.tile_hist; p.tile_base = a.tile_base;
  p.counts = a.counts; p.offsets = a.offsets;
  p.err = a.err; p.done_count = a.done_count;
  p.timeout_ns = kDefaultTimeoutNs;
  if (a.inv_row || a.perm_src) {
    if (!(a.inv_row && a.perm_src) || p.ntiles != 1) return cudaErrorInvalidValue;
    p.inv_row = a.inv_row;
    p.perm_src = a.perm_src;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.ntiles * S);
  cfg.blockDim = dim3(FR_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, tX, tW, p);
}

}  // namespace moe
