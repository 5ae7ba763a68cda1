// Internal declarations shared by the kernels and the C-ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kChunk = 32;            // tokens per routing chunk (one warp's worth)
constexpr int kTileChunks = 4;        // chunks per 128-token tile of the fused router
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kMaxGroups = 32;
constexpr long long kDefaultTimeoutNs = 2000000000LL;   // 2 s per device wait

// Error word codes written by kernels (bit flags, OR-ed together).
constexpr uint32_t kErrTimeoutWait = 1u << 0;
constexpr uint32_t kErrBadIndex = 1u << 1;

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// A caller-supplied segment offset, clamped into [0, hi] so that every row a
// kernel derives from it stays inside the packed arrays; a value that needed
// clamping is recorded in the error word (when there is one).
__device__ __forceinline__ int clamp_offset(int v, int hi, uint32_t* err) {
  if (v < 0 || v > hi) {
    if (err) atomicOr(err, kErrBadIndex);
    return v < 0 ? 0 : hi;
  }
  return v;
}
__host__ __device__ inline long long ceil_div_ll(long long a, long long b) { return (a + b - 1) / b; }

template <typename T> struct Vec16;            // 16-byte vector of T
template <> struct Vec16<float> { static constexpr int N = 4; };
template <> struct Vec16<__nv_bfloat16> { static constexpr int N = 8; };

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Expert nonlinearities after a biased linear map (generic experts).
constexpr int kActNone = 0;
constexpr int kActGelu = 1;
// GELU(v) = v * Phi(v), Phi the standard normal CDF, through erf.
__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

// ---------------------------------------------------------------- launchers
// Per-token routing settings (route_topk.cuh).
struct TopkArgs {
  int E, k, gate_mode, n_groups, topk_groups;
  float route_scale;
  const float* bias;   // [E] or null
};

// Routing (route_kernels.cu)
struct RouteParams {
  int T, E, k, gate_mode, n_groups, topk_groups;
  float route_scale;
  float* logits;           // [T][E]; with n_partials > 1, partial 0 of n_partials
  int n_partials;          // router partial sums to add (in order) per logit, >= 1
  long long partial_stride;  // elements between partials (T * E)
  const float* bias;       // [E] or null
  int* topk_idx;           // [T][k]
  float* topk_gate;        // [T][k]
  int* chunk_counts;       // [nchunks][E] or null
};
cudaError_t launch_router_topk(const RouteParams& p, cudaStream_t s);
cudaError_t launch_chunk_counts(const int* topk_idx, int T, int k, int E, int* chunk_counts,
                                cudaStream_t s);
cudaError_t launch_chunk_scan(const int* chunk_counts, int nchunks, int E, int* chunk_base,
                              int* counts, cudaStream_t s);
cudaError_t launch_offsets(const int* counts, int E, int* offsets, cudaStream_t s);
cudaError_t launch_balance_update(const int* counts, int E, long long tk, float gamma, float* bias,
                                  float* entropy, cudaStream_t s);

// Permute / combine (permute_kernels.cu)
// A token's packed row: offsets[e] + tile_base[chunk / kTileChunks][e] (null:
// 0) + chunk_base[chunk][e] + its rank among the chunk's tokens that chose e.
// Ids outside [0, E) and rows outside [0, T*k) are skipped (row -1) and
// recorded in `err` (nullable).
cudaError_t launch_permute(int dtype, const void* x, const int* topk_idx, const int* offsets,
                           const int* chunk_base, const int* tile_base, int T, int d, int E, int k,
                           void* x_perm, int* perm_src, int* inv_row, int num_sms, cudaStream_t s, bool copy,
                           uint32_t* err);
cudaError_t launch_combine(int dtype, const void* y_perm, const int* inv_row, const float* gate,
                           const void* y_shared, void* y, int T, int d, int k, int num_sms,
                           cudaStream_t s);

// SIMT grouped GEMM (simt_gemm.cu): fp32 experts and fp32 router logits.
struct SimtGemmParams {
  int dual;                 // 1: out = SiLU(A B1^T) * (A B3^T); 0: out = A B1^T
  int n_routed;             // routed segments (E), 0 for a single dense segment
  const int* offsets;       // [n_routed+1] packed-row offsets
  const void* a;            // routed A rows [rows][K]
  const void* b1;           // routed B1 [n_routed][N][K]
  const void* b3;           // routed B3 (dual)
  void* out;                // routed out [rows][N]
  int N, K;
  int shared_rows;          // rows of the dense (shared) segment, 0 = none
  const void* a_s; const void* b1_s; const void* b3_s; void* out_s;
  int N_s, K_s;
  int max_rows;             // routed rows (T*k): grid size, and the bound offsets are clamped to
  uint32_t* err;            // error word for out-of-range offsets, or null
  // Dual GEMM, optional: also store A B1^T and A B3^T (pre-activations).
  void* pre_a; void* pre_b; void* pre_a_s; void* pre_b_s;
  // Single GEMM only: out = act(A B1^T + bias), bias fp32 [n_routed][N] / [N_s] or null.
  const float* bias1; const float* bias1_s;
  int act;                  // kActNone or kActGelu
};
cudaError_t launch_simt_gemm(int in_dtype, int out_f32, const SimtGemmParams& p, cudaStream_t s);

// Strided grouped GEMM for the backward pass (grad_gemm.cu), fp32 FMA.
enum GradSegMode { kSegRows = 0, kSegK = 1 };
struct GradGemmParams {
  int dtype;                // MOE_DTYPE_*: type of B and of A/C unless a_f32 / c_f32
  int a_f32, c_f32;         // A / C held in fp32 regardless of dtype
  int seg_mode;             // kSegRows or kSegK
  int n_seg;
  const int* offsets;       // [n_seg+1] row or reduction offsets (null: one segment)
  int M, N, K;              // kSegK: output M x N per segment; kSegRows: N columns, K reduction
  int max_rows;             // kSegRows: upper bound on rows (grid sizing / dense segment)
  const void* a; long long a_si, a_sk;
  const void* b; long long b_seg, b_sj, b_sk;
  void* c; long long c_seg, c_si;
  int accumulate;           // C += product instead of C = product
};
cudaError_t launch_grad_gemm(const GradGemmParams& p, cudaStream_t s);

// Backward elementwise / per-token kernels (backward_kernels.cu)
cudaError_t launch_swiglu_bwd(int dtype, const void* a, const void* b, const float* dhp,
                              const int* inv_row, const float* gate, float* dgate, void* hg, void* dadb,
                              int n_rows, int f, int f_pad, cudaStream_t s);
cudaError_t launch_gate_bwd(const float* logits, const int* idx, const float* gate, const float* dgate,
                            float* dl, void* dl_bf16, int e_pad, int T, int E, int k, int gate_mode,
                            float route_scale, cudaStream_t s);
cudaError_t launch_unpermute_sum(int dtype, const float* dxp, const int* inv_row, const float* dxs,
                                 const float* dxr, void* dx, int T, int d, int k, cudaStream_t s);

// tcgen05 grouped GEMM (umma_gemm.cu)
enum UmmaMode { kUmmaSwiGLU = 1, kUmmaDown = 2, kUmmaBiasAct = 3, kUmmaDgrad = 4, kUmmaSwiGLUSave = 5 };
struct UmmaGemmParams {
  int mode;
  int n_routed;             // routed segments
  const int* offsets;       // [n_routed+1]
  int m_rows;               // weight rows per routed expert
  int K;                    // reduction length of routed segments
  int shared_rows;          // tokens of the dense segment (0 = none)
  int m_rows_s;             // weight rows of the dense segment
  int K_s;
  int bn_max;               // token tile cap, multiple of 16, <= 256
  int max_inflight;         // slots a CTA keeps loading at once (2..8)
  // tensor sources (bf16, row-major)
  const void* a; const void* a3; const void* b;        // routed: [n_routed*m_rows][K], ..., [rows][K]
  long long a_rows_total, b_rows_total;
  const void* a_s; const void* a3_s; const void* b_s;  // dense: [m_rows_s][K_s], ..., [shared_rows][K_s]
  void* out; long long out_ld;                          // routed out [rows][out_ld]
  void* out_s; long long out_s_ld;                      // dense out
  uint32_t* err;
  long long timeout_ns;
  int max_routed_rows;      // upper bound on routed rows (T*k) for the grid
  // Optional gather of routed token rows: packed row r reads source row
  // b_gather[r] of b_gather_src ([b_gather_rows][K]) instead of row r of b.
  const int* b_gather;
  const void* b_gather_src;
  long long b_gather_rows;
  // kUmmaBiasAct: out = act(acc + bias[weight row]); fp32 bias per segment
  // ([n_routed][m_rows] routed, [m_rows_s] dense), null = no bias.
  const float* row_bias; const float* row_bias_s;
  int act;                  // kActNone or kActGelu
  // kUmmaDgrad: a / a3 (a_s / a3_s) are stored [rows c][m_rows] with m
  // contiguous; a_k_rows (a_k_rows_s) rows of c per segment; the first
  // k_split (k_split_s) 64-wide k blocks read a, the rest read a3 from row 0.
  int a_k_rows, a_k_rows_s;
  int k_split, k_split_s;
  int out_f32;              // kUmmaDgrad: fp32 output instead of bf16
  // kUmmaSwiGLUSave: also store the pre-activations W1 u, W3 u (bf16, laid
  // out like out / out_s) for a later backward pass.
  void* pre_a; void* pre_b; void* pre_a_s; void* pre_b_s;
};
cudaError_t launch_umma_gemm(const UmmaGemmParams& p, int num_sms, cudaStream_t s);

// tcgen05 weight-gradient GEMM (umma_wgrad.cu): D_s[m][n] = sum over the
// rows r of segment s of P[r][m] Q[r][n], bf16 in, fp32 accumulate, bf16 out.
struct WgradParams {
  int n_seg;
  const int* offsets;       // [n_seg+1] row offsets; null: one segment of k_total rows
  int k_total;
  int M, N;
  const void* P; long long ldP, p_rows;   // [p_rows][ldP] bf16, columns [0, M) used
  const void* Q; long long ldQ, q_rows;   // [q_rows][ldQ] bf16, columns [0, N) used
  void* out;                // bf16 [n_seg][M][N]
  uint32_t* err;
  long long timeout_ns;
};
cudaError_t launch_wgrad(const WgradParams& p, int num_sms, cudaStream_t s);
cudaError_t launch_wait_timeout_selftest(uint32_t* err, long long timeout_ns, cudaStream_t s);

// The whole router in one kernel (router_fused.cu), bf16 and E <= 256:
// logits, top-k, gates, chunk bases within 128-token tiles, tile bases,
// counts and offsets. `done_count` must be zero before the launch.
struct FusedRouterLaunch {
  const void* x; const void* w_router;
  int T, E, K;
  TopkArgs topk;
  float* logits; int* topk_idx; float* topk_gate;
  int* chunk_base; int* tile_hist; int* tile_base; int* counts; int* offsets;
  uint32_t* err; uint32_t* done_count;
  int* inv_row = nullptr;    // with perm_src: the permute's row maps too (T <= 128 only)
  int* perm_src = nullptr;
};
bool router_fused_supported(int dtype, int E);
int router_fused_cluster(int T, int K);
cudaError_t launch_router_fused(const FusedRouterLaunch& a, cudaStream_t s);

// tcgen05 router logits with a split contraction (umma_router.cu): partial
// [n_split][T][E] fp32, summed by the top-k kernel.
int router_gemm_splits(int T, int E, int K);
cudaError_t launch_router_gemm(const void* x, const void* w_router, int T, int E, int K, float* partial,
                               int n_split, uint32_t* err, cudaStream_t s);

int device_sm_count();

}  // namespace moe
