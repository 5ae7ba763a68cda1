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
#include <algorithm>

#include "umma_common.cuh"

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
// Packed rows of chunk c's tokens into s_row[token * k + j] (-1 for an id
// outside [0, E) or a row outside [0, rows_total), recorded in err); with
// write_maps also inv_row and perm_src. Called by every thread of the block;
// ends with the block synchronised.
__device__ void chunk_rows(int c, const int* __restrict__ idx, const int* __restrict__ offsets,
                           const int* __restrict__ chunk_base, const int* __restrict__ tile_base, int n_tok, int E,
                           int k, int rows_total, bool write_maps, int* __restrict__ perm_src,
                           int* __restrict__ inv_row, uint32_t* __restrict__ err, uint32_t* s_mask, int* s_row) {
  // A token's ids go out kB at a time, and so do the loads of each batch's
  // offsets and bases, before any is used: a few memory round trips per
  // chunk rather than a few per id.
  constexpr int kB = 8;
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) s_mask[e] = 0u;
  __syncthreads();
  const int t = c * kChunk + tid;
  const bool tok = tid < kChunk && t < n_tok;
  int ids[kB];
  if (tok) {
    for (int j0 = 0; j0 < k; j0 += kB) {
#pragma unroll
      for (int u = 0; u < kB; ++u) ids[u] = j0 + u < k ? idx[(size_t)t * k + j0 + u] : -1;
#pragma unroll
      for (int u = 0; u < kB; ++u)
        if (ids[u] >= 0 && ids[u] < E) atomicOr(&s_mask[ids[u]], 1u << tid);
    }
  }
  __syncthreads();
  if (tok) {
    const int* tb_row = tile_base ? tile_base + (size_t)(c / kTileChunks) * E : nullptr;
    for (int j0 = 0; j0 < k; j0 += kB) {
      if (k > kB) {   // the registers hold the last batch only: reload
#pragma unroll
        for (int u = 0; u < kB; ++u) ids[u] = j0 + u < k ? idx[(size_t)t * k + j0 + u] : -1;
      }
      int base[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int e = ids[u];
        base[u] = 0;
        if (e >= 0 && e < E) {
          base[u] = offsets[e] + chunk_base[(size_t)c * E + e];
          if (tb_row) base[u] += tb_row[e];
        }
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int j = j0 + u;
        if (j >= k) break;
        const int e = ids[u];
        int row = -1;
        if (e >= 0 && e < E) {
          row = base[u] + __popc(s_mask[e] & ((1u << tid) - 1u));
          if (row < 0 || row >= rows_total) row = -1;
        }
        if (row < 0 && err && write_maps) atomicOr(err, kErrBadIndex);
        s_row[tid * k + j] = row;
        if (write_maps) {
          inv_row[(size_t)t * k + j] = row;
          if (row >= 0) perm_src[row] = t;
        }
      }
    }
  }
  __syncthreads();
}

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
  chunk_rows(c, idx, offsets, chunk_base, tile_base, n_tok, E, k, rows_total, blockIdx.y == 0, perm_src, inv_row,
             err, s_mask, s_row);
  if (!copy) return;
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

constexpr int kMaxBulkBufs = 8;

__device__ __forceinline__ void bulk_load_row(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void bulk_store_row(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
// All but the newest committed group have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// The same permute moving whole rows with bulk copies: grid = tok_split
// blocks per chunk of 32 tokens, block b taking the chunk's tokens
// i = b % tok_split, i + tok_split, ... (smaller blocks spread the rows
// over every SM). After the chunk's row maps (written by the first of its
// blocks), one thread streams the block's rows through a ring of nbuf
// shared-memory buffers: one copy brings a row (row_bytes, a multiple of
// 16) in, k copies write it to its packed rows. A row's buffer is refilled
// once the copies out of it have read it, so up to nbuf - 1 rows are on
// their way in while one goes out. Every wait is bounded; on expiry the
// block records kErrTimeoutWait, waits (bounded) for the rows it still has
// coming in, and stops.
__global__ void __launch_bounds__(128) permute_bulk_kernel(
    const char* __restrict__ x, const int* __restrict__ idx, const int* __restrict__ offsets,
    const int* __restrict__ chunk_base, const int* __restrict__ tile_base, int n_tok, int E, int k,
    uint32_t row_bytes, int nbuf, int tok_split, char* __restrict__ x_perm, int* __restrict__ perm_src,
    int* __restrict__ inv_row, int rows_total, uint32_t* __restrict__ err, long long timeout_ns) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint32_t s_mask[kMaxExperts];
  __shared__ int s_row[kChunk * kMaxTopK];
  __shared__ __align__(8) uint64_t bars[kMaxBulkBufs];
  __shared__ uint32_t s_abort;
  const int c = blockIdx.x / tok_split, part = blockIdx.x % tok_split;
  // this block's tokens of the chunk: part, part + tok_split, ...
  const int ntok = max(0, ceil_div(min(kChunk, n_tok - c * kChunk) - part, tok_split));
  const uint32_t ring0 = smem_u32(ring);
  auto tok = [&](int i) { return part + i * tok_split; };
  auto load = [&](int i) {
    const int b = i % nbuf;
    mbar_expect_tx(smem_u32(&bars[b]), row_bytes);
    bulk_load_row(ring0 + (uint32_t)b * row_bytes, x + (size_t)(c * kChunk + tok(i)) * row_bytes, row_bytes,
                  smem_u32(&bars[b]));
  };
  // The first rows come in while the block works out the row maps (the
  // loads need no map; only the copies out do).
  int issued = min(nbuf, ntok);
  if (threadIdx.x == 0) {
    for (int b = 0; b < nbuf; ++b) mbar_init(smem_u32(&bars[b]), 1);
    s_abort = 0u;
    fence_mbar_init();
    for (int i = 0; i < issued; ++i) load(i);
  }
  chunk_rows(c, idx, offsets, chunk_base, tile_base, n_tok, E, k, rows_total, part == 0, perm_src, inv_row, err,
             s_mask, s_row);
  if (threadIdx.x != 0) return;
  int done = 0;   // rows whose load has been waited for
  for (int i = 0; i < ntok; ++i) {
    const int b = i % nbuf;
    if (!wait_bounded(smem_u32(&bars[b]), (uint32_t)(i / nbuf) & 1u, (volatile uint32_t*)&s_abort, err, timeout_ns,
                      true))
      break;
    done = i + 1;
    for (int j = 0; j < k; ++j) {
      const int row = s_row[tok(i) * k + j];
      if (row >= 0) bulk_store_row(x_perm + (size_t)row * row_bytes, ring0 + (uint32_t)b * row_bytes, row_bytes);
    }
    bulk_commit();
    // Refill the previous row's buffer once its copies out have read it.
    if (i >= 1 && issued < ntok) {
      bulk_wait_read_but_one();
      load(issued++);
    }
  }
  for (int i = done; i < issued; ++i)   // only after a timeout: let the rows in flight land
    wait_bounded(smem_u32(&bars[i % nbuf]), (uint32_t)(i / nbuf) & 1u, (volatile uint32_t*)&s_abort, err,
                 timeout_ns, false);
  bulk_wait_all();
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
    // The k expert rows' loads go out eight at a time before any is summed
    // (the sum itself keeps slot order), so eight wait in parallel.
    for (int j0 = 0; j0 < k; j0 += 8) {
      uint4 raw[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = j0 + jj;
        const int row = j < k ? s_row[j] : -1;
        raw[jj] = row >= 0 ? ld16(y_perm + (size_t)row * d + (size_t)v * V) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = j0 + jj;
        if (j < k && s_row[j] >= 0) unpack_add<T>(acc, raw[jj], s_g[j]);
      }
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
  // Whole rows by bulk copies when each row goes to at least four packed
  // rows and there are at least 64 chunks (measured on B200: 12% faster at
  // k = 8 with 128 or 512 chunks, slower at k = 2 or with a handful of
  // chunks, where one thread's per-row chain dominates), a ring of at least
  // two rows fits in kBulkRingBytes and both row arrays are 16-byte aligned.
  // With more chunks than SMs the chunks run in waves whose last one leaves
  // SMs idle; blocks of four tokens (eight per chunk) even that out
  // (measured on B200: 8% faster at 512 chunks, 4% slower at 128).
  constexpr int kBulkRingBytes = 96 * 1024;
  const int tok_split = nch > num_sms ? 8 : 1;
  const long long row_bytes = (long long)d * (dtype == MOE_DTYPE_F32 ? 4 : 2);
  const int nbuf = (int)std::min<long long>(std::min(kMaxBulkBufs, ceil_div(kChunk, tok_split) + 1),
                                            kBulkRingBytes / row_bytes);
  if (copy && k >= 4 && nch >= 64 && nbuf >= 2 && row_bytes % 16 == 0 &&
      ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(x_perm)) & 15u) == 0) {
    static int attr_done = 0;   // one bit per device ordinal (< 32)
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!(dev < 32 && ((attr_done >> dev) & 1))) {
      e = cudaFuncSetAttribute(permute_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBulkRingBytes);
      if (e != cudaSuccess) return e;
      if (dev < 32) attr_done |= 1 << dev;
    }
    permute_bulk_kernel<<<nch * tok_split, 128, nbuf * row_bytes, s>>>(
        static_cast<const char*>(x), topk_idx, offsets, chunk_base, tile_base, T, E, k, (uint32_t)row_bytes, nbuf,
        tok_split, static_cast<char*>(x_perm), perm_src, inv_row, T * k, err, kDefaultTimeoutNs);
    return cudaGetLastError();
  }
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
