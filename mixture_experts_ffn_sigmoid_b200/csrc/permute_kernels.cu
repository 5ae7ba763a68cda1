// Permute (gather into expert-contiguous order) and combine (gate-weighted
// sum plus the shared row).
//
// Sparse MoE FFN (DeepSeek-V3 note), "How it works", "Packed forward
// (official)": for each expert, gather the tokens whose indices equal it,
// run the SwiGLU, scale by the matching weights and scatter-add into a zero
// buffer; add the shared FFN computed on all tokens.
// MoE knowledge-base page, "The router and load balancing": out[rows] +=
// w * expert(x[rows]).
//
// Both kernels move whole rows with 16-byte vector loads and stores; rows
// are d * sizeof(T) bytes, a multiple of 16 (checked by the C ABI).
#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ uint4 ld16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void st16(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// grid = (chunks of 32 tokens, column splits). Each block recomputes its
// chunk's packed rows (cheap: offsets[e] + the chunk's base for e, plus the
// base of its 128-token tile when the chunk bases count from the tile's
// start, + the token's rank in the chunk), then copies a column slice of the
// 32 rows to their k destinations. Split 0 also writes inv_row / perm_src. Without
// `copy` only the maps are written (the GEMM then gathers rows from x).
template <typename T>
__global__ void __launch_bounds__(256) permute_kernel(
    const T* __restrict__ x, const int* __restrict__ idx, const int* __restrict__ offsets,
    const int* __restrict__ chunk_base, const int* __restrict__ tile_base, int n_tok, int d, int E, int k,
    T* __restrict__ x_perm,
    int* __restrict__ perm_src, int* __restrict__ inv_row, int rows_total, int vec_per_split,
    int copy, uint32_t* __restrict__ err) {
  constexpr int V = Vec16<T>::N;
  __shared__ uint32_t s_mask[kMaxExperts];
  __shared__ int s_row[kChunk * kMaxTopK];
  const int c = blockIdx.x;
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) s_mask[e] = 0u;
  __syncthreads();
  const int t = c * kChunk + tid;
  const bool tok = tid < kChunk && t < n_tok;
  if (tok) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e >= 0 && e < E) atomicOr(&s_mask[e], 1u << tid);
    }
  }
  __syncthreads();
  if (tok) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      int row = -1;
      if (e >= 0 && e < E) {
        const int rank = __popc(s_mask[e] & ((1u << tid) - 1u));
        row = offsets[e] + chunk_base[(size_t)c * E + e] + rank;
        if (tile_base) row += tile_base[(size_t)(c / kTileChunks) * E + e];
        if (row < 0 || row >= rows_total) row = -1;
      }
      if (row < 0 && err && blockIdx.y == 0) atomicOr(err, kErrBadIndex);
      s_row[tid * k + j] = row;
      if (blockIdx.y == 0) {
        inv_row[(size_t)t * k + j] = row;
        if (row >= 0) perm_src[row] = t;
      }
    }
  }
  if (!copy) return;
  __syncthreads();
  const int nvec = d / V;
  const int v0 = blockIdx.y * vec_per_split;
  const int v1 = min(nvec, v0 + vec_per_split);
  const int nv = v1 - v0;
  const int ntok = min(kChunk, n_tok - c * kChunk);
  if (nv <= 0) return;
  // Four independent 16-byte loads in flight per thread before their stores
  // (each load feeds k stores, so the copy is bound by how many loads wait).
  constexpr int U = 4;
  const int n_items = ntok * nv;
  for (int base = tid; base < n_items; base += U * blockDim.x) {
    uint4 val[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int item = base + u * blockDim.x;
      if (item < n_items) {
        const int tl = item / nv;
        val[u] = ld16(x + (size_t)(c * kChunk + tl) * d + (size_t)(v0 + item - tl * nv) * V);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int item = base + u * blockDim.x;
      if (item < n_items) {
        const int tl = item / nv;
        const int v = v0 + item - tl * nv;
        for (int j = 0; j < k; ++j) {
          const int row = s_row[tl * k + j];
          if (row >= 0) st16(x_perm + (size_t)row * d + (size_t)v * V, val[u]);
        }
      }
    }
  }
}

template <typename T>
__device__ __forceinline__ void unpack_add(float* acc, uint4 raw, float g);
template <>
__device__ __forceinline__ void unpack_add<float>(float* acc, uint4 raw, float g) {
  acc[0] = fmaf(g, __uint_as_float(raw.x), acc[0]);
  acc[1] = fmaf(g, __uint_as_float(raw.y), acc[1]);
  acc[2] = fmaf(g, __uint_as_float(raw.z), acc[2]);
  acc[3] = fmaf(g, __uint_as_float(raw.w), acc[3]);
}
template <>
__device__ __forceinline__ void unpack_add<__nv_bfloat16>(float* acc, uint4 raw, float g) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16);
    const float hi = __uint_as_float(w[i] & 0xffff0000u);
    acc[2 * i] = fmaf(g, lo, acc[2 * i]);
    acc[2 * i + 1] = fmaf(g, hi, acc[2 * i + 1]);
  }
}
template <typename T> __device__ __forceinline__ uint4 pack(const float* acc);
template <> __device__ __forceinline__ uint4 pack<float>(const float* acc) {
  return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                    __float_as_uint(acc[3]));
}
template <> __device__ __forceinline__ uint4 pack<__nv_bfloat16>(const float* acc) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// grid = (T, column splits). y[t] = sum_j g[t,j] * y_perm[inv_row[t,j]] (+ y_shared[t]),
// accumulated in fp32 in slot order, then the shared row, rounded once.
template <typename T>
__global__ void __launch_bounds__(128) combine_kernel(
    const T* __restrict__ y_perm, const int* __restrict__ inv_row, const float* __restrict__ gate,
    const T* __restrict__ y_shared, T* __restrict__ y, int d, int k, int vec_per_split, int rows_total) {
  constexpr int V = Vec16<T>::N;
  __shared__ int s_row[kMaxTopK];
  __shared__ float s_g[kMaxTopK];
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    const int r = inv_row[(size_t)t * k + threadIdx.x];
    s_row[threadIdx.x] = r < rows_total ? r : -1;   // a caller row past the packed rows is skipped
    s_g[threadIdx.x] = gate[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
  const int nvec = d / V;
  const int v0 = blockIdx.y * vec_per_split;
  const int v1 = min(nvec, v0 + vec_per_split);
  for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int row = s_row[j];
      if (row >= 0) unpack_add<T>(acc, ld16(y_perm + (size_t)row * d + (size_t)v * V), s_g[j]);
    }
    if (y_shared) unpack_add<T>(acc, ld16(y_shared + (size_t)t * d + (size_t)v * V), 1.0f);
    st16(y + (size_t)t * d + (size_t)v * V, pack<T>(acc));
  }
}

}  // namespace

cudaError_t launch_permute(int dtype, const void* x, const int* topk_idx, const int* offsets,
                           const int* chunk_base, const int* tile_base, int T, int d, int E, int k,
                           void* x_perm, int* perm_src, int* inv_row, int num_sms, cudaStream_t s, bool copy,
                           uint32_t* err) {
  if (T <= 0) return cudaSuccess;
  const int V = dtype == MOE_DTYPE_F32 ? 4 : 8;
  const int nvec = d / V;
  const int nch = ceil_div(T, kChunk);
  int nsplit = copy ? ceil_div(4 * num_sms, nch) : 1;
  if (nsplit < 1) nsplit = 1;
  if (nsplit > nvec) nsplit = nvec;
  const int vps = ceil_div(nvec, nsplit);
  nsplit = ceil_div(nvec, vps);
  dim3 grid(nch, nsplit);
  if (dtype == MOE_DTYPE_F32)
    permute_kernel<float><<<grid, 256, 0, s>>>((const float*)x, topk_idx, offsets, chunk_base, tile_base, T,
                                                d, E, k, (float*)x_perm, perm_src, inv_row, T * k, vps,
                                                copy ? 1 : 0, err);
  else
    permute_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        (const __nv_bfloat16*)x, topk_idx, offsets, chunk_base, tile_base, T, d, E, k,
        (__nv_bfloat16*)x_perm, perm_src, inv_row, T * k, vps, copy ? 1 : 0, err);
  return cudaGetLastError();
}

cudaError_t launch_combine(int dtype, const void* y_perm, const int* inv_row, const float* gate,
                           const void* y_shared, void* y, int T, int d, int k, int num_sms,
                           cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int V = dtype == MOE_DTYPE_F32 ? 4 : 8;
  const int nvec = d / V;
  int nsplit = ceil_div(2 * num_sms, T);
  const int max_split = ceil_div(nvec, 32);
  if (nsplit > max_split) nsplit = max_split;
  if (nsplit < 1) nsplit = 1;
  const int vps = ceil_div(nvec, nsplit);
  nsplit = ceil_div(nvec, vps);
  dim3 grid(T, nsplit);
  if (dtype == MOE_DTYPE_F32)
    combine_kernel<float><<<grid, 128, 0, s>>>((const float*)y_perm, inv_row, gate,
                                               (const float*)y_shared, (float*)y, d, k, vps, T * k);
  else
    combine_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(
        (const __nv_bfloat16*)y_perm, inv_row, gate, (const __nv_bfloat16*)y_shared,
        (__nv_bfloat16*)y, d, k, vps, T * k);
  return cudaGetLastError();
}

}  // namespace moe
