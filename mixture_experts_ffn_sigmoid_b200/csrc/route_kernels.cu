// Routing kernels: biased, optionally group-limited top-k over router logits
// held in memory (the per-token logic of route_topk.cuh: the Sparse MoE FFN
// note's Routing paragraph and the MoE cheat sheet's "The router in code"),
// gates from the unbiased affinities, and the deterministic packing offsets.
// Used for fp32 inputs and for more than 256 experts; the bf16 router of up
// to 256 experts runs fused with its GEMM (router_fused.cu).
//
// Layout: one warp per token, each lane holding the experts route_expert
// gives it (NPL consecutive experts up to 256, else l, l+32, ...); a
// block of 32 warps is one chunk of 32 tokens, so the same block can also
// emit the chunk's per-expert histogram (a bit mask per expert: bit w set
// when token w of the chunk chose the expert). Histograms are exact and the
// scan below gives every (token, expert) pair the packed row
// offsets[e] + #{earlier tokens that chose e}: deterministic, atomic-free.
#include <math.h>

#include "route_topk.cuh"

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

template <int NPL>
__global__ void __launch_bounds__(1024, 1) router_topk_kernel(RouteParams p) {
  __shared__ uint32_t s_mask[kMaxExperts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int t = chunk * kChunk + warp;
  const int E = p.E, k = p.k;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_mask[e] = 0u;
  __syncthreads();

  if (t < p.T) {                       // warp-uniform
    float* lrow = p.logits + (size_t)t * E;
    float lg[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = route_expert<NPL>(lane, i);
      float l = 0.0f;
      if (e < E) {
        // Router partial sums (a split contraction) add up in a fixed order;
        // the total replaces partial 0, where later readers find the logit.
        l = lrow[e];
        for (int q = 1; q < p.n_partials; ++q) l += lrow[(size_t)q * p.partial_stride + e];
        if (p.n_partials > 1) lrow[e] = l;
      }
      lg[i] = l;
    }
    const TopkArgs a = {E, k, p.gate_mode, p.n_groups, p.topk_groups, p.route_scale, p.bias};
    int my_e, pos;
    float gate;
    route_token<NPL>(lg, lane, a, my_e, pos, gate, NPL > 8 ? lrow : nullptr);
    if (lane < k) {
      p.topk_idx[(size_t)t * k + pos] = my_e;
      p.topk_gate[(size_t)t * k + pos] = gate;
      atomicOr(&s_mask[my_e], 1u << warp);
    }
  }
  if (p.chunk_counts) {
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      p.chunk_counts[(size_t)chunk * E + e] = __popc(s_mask[e]);
  }
}

// Per-chunk histograms from a caller-supplied topk_idx (used by the
// stand-alone permute entry point). Out-of-range ids are skipped.
__global__ void __launch_bounds__(256) chunk_count_kernel(const int* __restrict__ idx, int T, int k,
                                                          int E, int* __restrict__ chunk_counts) {
  __shared__ uint32_t s_mask[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_mask[e] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kChunk + threadIdx.x;
  if (threadIdx.x < kChunk && t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e >= 0 && e < E) atomicOr(&s_mask[e], 1u << threadIdx.x);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_counts[(size_t)blockIdx.x * E + e] = __popc(s_mask[e]);
}

// Inclusive block scan of one int per thread (blockDim a multiple of 32, <= 1024).
__device__ int block_inclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(kFull, v, off);
    if (lane >= off) v += o;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(kFull, w, off);
      if (lane >= off) w += o;
    }
    if (lane < nwarps) s_warp[lane] = w;
  }
  __syncthreads();
  const int before = warp > 0 ? s_warp[warp - 1] : 0;
  *total = s_warp[nwarps - 1];
  __syncthreads();
  return v + before;
}

// One block per expert: exclusive scan of its per-chunk counts over chunks.
__global__ void __launch_bounds__(256) chunk_scan_kernel(const int* __restrict__ cc, int nch, int E,
                                                         int* __restrict__ base, int* __restrict__ counts) {
  __shared__ int s_warp[32];
  const int e = blockIdx.x;
  int carry = 0;
  for (int c0 = 0; c0 < nch; c0 += blockDim.x) {
    const int c = c0 + threadIdx.x;
    const int v = c < nch ? cc[(size_t)c * E + e] : 0;
    int total;
    const int incl = block_inclusive_scan(v, s_warp, &total);
    if (c < nch) base[(size_t)c * E + e] = carry + incl - v;
    carry += total;
  }
  if (threadIdx.x == 0) counts[e] = carry;
}

// Exclusive scan of counts over experts: offsets[0..E].
__global__ void __launch_bounds__(1024) offsets_kernel(const int* __restrict__ counts, int E,
                                                       int* __restrict__ offsets) {
  __shared__ int s_warp[32];
  const int e = threadIdx.x;
  const int v = e < E ? counts[e] : 0;
  int total;
  const int incl = block_inclusive_scan(v, s_warp, &total);
  if (e < E) offsets[e] = incl - v;
  if (e == 0) offsets[E] = total;
}

// Aux-loss-free balancing step (MoE cheat sheet, "Aux-loss-free balance
// loop"): target = T*k/E; an expert over target loses gamma of bias, one
// under target gains gamma, one on target keeps its bias (decided in exact
// integer arithmetic, count*E vs T*k). Also the entropy (nats) of the usage
// distribution counts/sum, accumulated in fp64.
__global__ void __launch_bounds__(1024) balance_update_kernel(const int* __restrict__ counts, int E,
                                                              long long tk, float gamma,
                                                              float* __restrict__ bias,
                                                              float* __restrict__ entropy) {
  __shared__ double s_red[32];
  __shared__ long long s_tot[32];
  const int e = threadIdx.x;
  const int lane = e & 31, warp = e >> 5, nwarps = blockDim.x >> 5;
  const long long c = e < E ? (long long)counts[e] : 0;
  if (e < E && bias) {
    const long long scaled = c * E;
    if (scaled > tk) bias[e] -= gamma;
    else if (scaled < tk) bias[e] += gamma;
  }
  if (!entropy) return;
  // Total count, then -sum p ln p.
  long long tot = c;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(kFull, tot, off);
  if (lane == 0) s_tot[warp] = tot;
  __syncthreads();
  long long all = 0;
  for (int w = 0; w < nwarps; ++w) all += s_tot[w];
  double h = 0.0;
  if (c > 0 && all > 0) {
    const double pr = (double)c / (double)all;
    h = -pr * log(pr);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) h += __shfl_xor_sync(kFull, h, off);
  if (lane == 0) s_red[warp] = h;
  __syncthreads();
  if (e == 0) {
    double sum = 0.0;
    for (int w = 0; w < nwarps; ++w) sum += s_red[w];
    *entropy = (float)sum;
  }
}

}  // namespace

cudaError_t launch_balance_update(const int* counts, int E, long long tk, float gamma, float* bias,
                                  float* entropy, cudaStream_t s) {
  const int threads = ceil_div(E, 32) * 32;
  balance_update_kernel<<<1, threads, 0, s>>>(counts, E, tk, gamma, bias, entropy);
  return cudaGetLastError();
}

cudaError_t launch_router_topk(const RouteParams& p, cudaStream_t s) {
  if (p.T <= 0) return cudaSuccess;
  const int nch = ceil_div(p.T, kChunk);
  const int per_lane = ceil_div(p.E, 32);
  dim3 grid(nch), block(1024);
  if (per_lane <= 1) router_topk_kernel<1><<<grid, block, 0, s>>>(p);
  else if (per_lane <= 2) router_topk_kernel<2><<<grid, block, 0, s>>>(p);
  else if (per_lane <= 4) router_topk_kernel<4><<<grid, block, 0, s>>>(p);
  else if (per_lane <= 8) router_topk_kernel<8><<<grid, block, 0, s>>>(p);
  else if (per_lane <= 16) router_topk_kernel<16><<<grid, block, 0, s>>>(p);
  else router_topk_kernel<32><<<grid, block, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_chunk_counts(const int* topk_idx, int T, int k, int E, int* chunk_counts,
                                cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  chunk_count_kernel<<<ceil_div(T, kChunk), 256, 0, s>>>(topk_idx, T, k, E, chunk_counts);
  return cudaGetLastError();
}

cudaError_t launch_chunk_scan(const int* chunk_counts, int nchunks, int E, int* chunk_base,
                              int* counts, cudaStream_t s) {
  chunk_scan_kernel<<<E, 256, 0, s>>>(chunk_counts, nchunks, E, chunk_base, counts);
  return cudaGetLastError();
}

cudaError_t launch_offsets(const int* counts, int E, int* offsets, cudaStream_t s) {
  const int threads = ceil_div(E, 32) * 32;
  offsets_kernel<<<1, threads, 0, s>>>(counts, E, offsets);
  return cudaGetLastError();
}

}  // namespace moe
