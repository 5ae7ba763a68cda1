// Router logits on the tensor cores: l[t][e] = sum_c x[t][c] w_router[e][c]
// (the router linear of the Sparse MoE FFN note's "Routing" paragraph,
// u_t . e_i; the MoE cheat sheet's "The router in code": one dot product of
// the hidden state with each router row).
//
// Tokens sit on the MMA's M side (128 per CTA) and experts on N (up to 256
// per CTA), so each token row is read from HBM once and the small router
// matrix is re-read from L2 once per 128 tokens. A few dozen token tiles do
// not fill the GPU, so the contraction is split into n_split chunks of
// whole 64-wide k blocks; CTA (token tile, chunk, expert tile) writes its
// fp32 partial sums to partial[chunk][t][e]. The top-k kernel adds the
// partials in chunk order (a fixed order: the logits are the same bits on
// every run) and stores the sum in partial 0.
//
// One tile per CTA, 128 threads: warp 0 lane 0 issues TMA into a 4-stage
// ring, warp 1 allocates TMEM and lane 0 issues tcgen05.mma (kind::f16,
// M = 128, N = 256 max, both operands K-major, 128-byte swizzle); then all
// four warps read their TMEM lane quarter (one token each) and store the
// token's partial logits. Waits are bounded like the other tcgen05 kernels.
#include "umma_common.cuh"

namespace moe {
namespace {

constexpr int RT_BM = 128;                 // tokens per CTA
constexpr int RT_BN = 256;                 // experts per CTA (max)
constexpr int RT_BK = 64;
constexpr int RT_STAGES = 4;
constexpr int RT_A_BYTES = RT_BM * RT_BK * 2;
constexpr int RT_B_BYTES = RT_BN * RT_BK * 2;
constexpr int RT_STAGE_BYTES = RT_A_BYTES + RT_B_BYTES;
constexpr int RT_THREADS = 128;
constexpr int RT_SMEM = 1024 + 1024 + RT_STAGES * RT_STAGE_BYTES;
constexpr int RT_TMEM_COLS = 256;

struct RouterGemmArgs {
  int T, E, K;
  int n_split, kb_per_split;   // k blocks per chunk
  float* partial;              // [n_split][T][E]
  uint32_t* err;
  long long timeout_ns;
};

__global__ void __launch_bounds__(RT_THREADS, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const RouterGemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty_bar = full_bar + RT_STAGES;
  uint64_t* done_bar = empty_bar + RT_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  uint8_t* ring = smem + 1024;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * RT_BM;
  const int split = blockIdx.y;
  const int e0 = blockIdx.z * RT_BN;
  const int n_e = min(RT_BN, p.E - e0);
  const int n_mma = (n_e + 15) & ~15;
  const int nkb_total = ceil_div(p.K, RT_BK);
  const int kb0 = split * p.kb_per_split;
  const int kb1 = min(nkb_total, kb0 + p.kb_per_split);
  const int nk = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < RT_STAGES; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    mbar_init(smem_u32(done_bar), 1);
    *abort_flag = 0u;
    fence_mbar_init();
    tmap_prefetch(&tmX);
    tmap_prefetch(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), RT_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    for (int i = 0; i < nk; ++i) {
      const int stage = i % RT_STAGES;
      const uint32_t parity = ((i / RT_STAGES) & 1u) ^ 1u;
      if (!wait_bounded(smem_u32(&empty_bar[stage]), parity, abort_flag, p.err, p.timeout_ns, true)) break;
      const uint32_t fb = smem_u32(&full_bar[stage]);
      const uint32_t sa = smem_u32(ring + stage * RT_STAGE_BYTES);
      mbar_expect_tx(fb, RT_STAGE_BYTES);   // whole boxes, zero fill past T or E included
      tma_load_2d(sa, &tmX, (kb0 + i) * RT_BK, t0, fb);
      tma_load_2d(sa + RT_A_BYTES, &tmW, (kb0 + i) * RT_BK, e0, fb);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool issued = false;
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(RT_BM, n_mma);
      for (int i = 0; i < nk; ++i) {
        const int stage = i % RT_STAGES;
        if (!wait_bounded(smem_u32(&full_bar[stage]), (i / RT_STAGES) & 1u, abort_flag, p.err, p.timeout_ns, true))
          break;
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + stage * RT_STAGE_BYTES);
        const uint64_t a_desc = sw128_desc(sa);
        const uint64_t b_desc = sw128_desc(sa + RT_A_BYTES);
#pragma unroll
        for (int kk = 0; kk < RT_BK / 16; ++kk) {
          const uint64_t koff = (uint64_t)((kk * 32) >> 4);
          umma_bf16(tmem_base, a_desc + koff, b_desc + koff, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&empty_bar[stage]));
        issued = true;
      }
      // Completion of every MMA (or nothing to wait for) releases the epilogue.
      if (issued) umma_commit(smem_u32(done_bar));
      else mbar_arrive(smem_u32(done_bar));
    }
    __syncwarp();
  }
  // ------------------------------------------------------------ epilogue (all warps)
  __syncwarp();   // lane 0 of warps 0 and 1 rejoins its warp before the aligned TMEM loads
  const bool ok = __all_sync(0xffffffffu,
                             wait_bounded(smem_u32(done_bar), 0u, abort_flag, p.err, p.timeout_ns, false));
  tc_fence_after();
  const int t = t0 + warp * 32 + lane;
  float* orow = p.partial + ((size_t)split * p.T + (t < p.T ? t : 0)) * p.E + e0;
  const uint32_t taddr = tmem_base + ((uint32_t)(warp * 32) << 16);
  for (int c0 = 0; c0 < n_mma; c0 += 64) {
    uint32_t r[64];
    if (ok && nk > 0) {
      tmem_ld64_wait(taddr + c0, r);
    } else {
#pragma unroll
      for (int j = 0; j < 64; ++j) r[j] = 0u;   // empty chunk (or a failed wait): zeros
    }
    if (t < p.T) {
      if ((p.E & 3) == 0 && c0 + 64 <= n_e) {   // rows 16-byte aligned: vector stores
        float4* o4 = reinterpret_cast<float4*>(orow + c0);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          o4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                              __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j)
          if (c0 + j < n_e) orow[c0 + j] = __uint_as_float(r[j]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, RT_TMEM_COLS);
  }
}

}  // namespace

// Chunks of the contraction: enough CTAs to cover B200's 148 SMs, at most
// 8, never more than there are 64-wide k blocks. A function of the shape
// only, so the workspace size does not depend on the device.
int router_gemm_splits(int T, int E, int K) {
  constexpr int num_sms = 148;
  const int tiles = ceil_div(T, RT_BM) * ceil_div(E, RT_BN);
  const int nkb = ceil_div(K, RT_BK);
  int s = num_sms / (tiles > 0 ? tiles : 1);
  if (s < 1) s = 1;
  if (s > 8) s = 8;
  if (s > nkb) s = nkb;
  return s;
}

cudaError_t launch_router_gemm(const void* x, const void* w_router, int T, int E, int K, float* partial,
                               int n_split, uint32_t* err, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  CUtensorMap tX, tW;
  if (!make_tmap(&tX, x, K, T, RT_BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&tW, w_router, K, E, RT_BN)) return cudaErrorInvalidValue;
  static int attr_done_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!(dev < 32 && ((attr_done_mask >> dev) & 1))) {
    e = cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, RT_SMEM);
    if (e != cudaSuccess) return e;
    if (dev < 32) attr_done_mask |= 1 << dev;
  }
  RouterGemmArgs a;
  a.T = T; a.E = E; a.K = K;
  a.n_split = n_split;
  a.kb_per_split = ceil_div(ceil_div(K, RT_BK), n_split);
  a.partial = partial;
  a.err = err;
  a.timeout_ns = kDefaultTimeoutNs;
  dim3 grid(ceil_div(T, RT_BM), n_split, ceil_div(E, RT_BN));
  router_gemm_kernel<<<grid, RT_THREADS, RT_SMEM, s>>>(tX, tW, a);
  return cudaGetLastError();
}

}  // namespace moe
