// Elementwise and per-token kernels of the backward pass.
//
// The block's forward (Sparse MoE FFN note, "How it works": SwiGLU equation,
// "Routing", "Packed forward"):
//   y_t = sum_j g_tj W2_e (SiLU(a) * b) + shared,  a = W1_e x_t, b = W3_e x_t
//   sigmoid gates g_j = rs * s_j / sum_i s_i (s = sigmoid(l));
//   softmax gates g_j = rs * softmax over the selected logits (the MoE cheat
//   sheet's "The router in code").
// The expert choice is piecewise constant, so gradients flow through the
// gates and the experts only.
#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float sigmoid_f(float v) { return 1.0f / (1.0f + expf(-v)); }

template <typename T> __device__ __forceinline__ void st(T* p, float v) { *p = from_f32<T>(v); }

// One block per (token, slot) of the routed rows, or per shared row. With
// dh' = W2^T dy_t (the down projection's input gradient, gate not applied):
//   h = SiLU(a) * b,  dgate = <dh', h>,  dh = g dh',
//   da = dh * b * SiLU'(a),  db = dh * SiLU(a),
// and hg = g h (the down projection's weight-gradient operand). da and db go
// side by side in one row of 2 * f_pad (zero past f in each half).
template <typename T>
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(
    const T* __restrict__ a, const T* __restrict__ b, const float* __restrict__ dhp,
    const int* __restrict__ inv_row, const float* __restrict__ gate, float* __restrict__ dgate,
    T* __restrict__ hg, T* __restrict__ dadb, int f, int f_pad) {
  const int pair = blockIdx.x;                 // t * k + j, or the shared row when inv_row is null
  const int r = inv_row ? inv_row[pair] : pair;
  if (r < 0) {                                 // no packed row (never for valid routing)
    if (dgate && threadIdx.x == 0) dgate[pair] = 0.0f;
    return;
  }
  const float g = gate ? gate[pair] : 1.0f;
  const size_t ro = (size_t)r * f;
  const size_t rd = (size_t)r * 2 * f_pad;
  float dot = 0.0f;
  for (int m = threadIdx.x; m < f_pad; m += blockDim.x) {
    if (m < f) {
      const float av = to_f32(a[ro + m]), bv = to_f32(b[ro + m]);
      const float dv = dhp[ro + m];
      const float sg = sigmoid_f(av);
      const float silu = av * sg;
      const float h = silu * bv;
      dot = fmaf(dv, h, dot);
      const float dh = g * dv;
      st(hg + ro + m, g * h);
      st(dadb + rd + m, dh * bv * sg * (1.0f + av * (1.0f - sg)));
      st(dadb + rd + f_pad + m, dh * silu);
    } else {
      st(dadb + rd + m, 0.0f);
      st(dadb + rd + f_pad + m, 0.0f);
    }
  }
  if (!dgate) return;
  __shared__ float red[32];
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dot;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) dgate[pair] = v;
  }
}

// Gate gradients -> logit gradients, one warp per token (lanes over slots).
// dl is [T][E], zero outside the token's k experts (written here for every
// expert, so no separate clear is needed); the optional bf16 copy is
// [T][e_pad] with zero columns past E.
__global__ void __launch_bounds__(256) gate_bwd_kernel(
    const float* __restrict__ logits, const int* __restrict__ idx, const float* __restrict__ gate,
    const float* __restrict__ dgate, float* __restrict__ dl, void* __restrict__ dl_bf16, int e_pad, int T,
    int E, int k, int gate_mode, float route_scale) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= T) return;
  const int t = warp;
  float* row = dl + (size_t)t * E;
  __nv_bfloat16* rowb = dl_bf16 ? static_cast<__nv_bfloat16*>(dl_bf16) + (size_t)t * e_pad : nullptr;
  for (int e = lane; e < E; e += 32) row[e] = 0.0f;
  if (rowb)
    for (int e = lane; e < e_pad; e += 32) rowb[e] = __float2bfloat16_rn(0.0f);
  __syncwarp();
  // Lanes j < k hold slot j (k <= 32). A slot whose id lies outside [0, E)
  // (a caller-supplied topk_idx) is skipped before anything is read through it.
  const int e_in = lane < k ? idx[(size_t)t * k + lane] : -1;
  const bool act = lane < k && e_in >= 0 && e_in < E;
  const int e = act ? e_in : 0;
  const float dg = act ? dgate[(size_t)t * k + lane] : 0.0f;
  float out = 0.0f;
  if (gate_mode == MOE_GATE_SIGMOID) {
    const float s = act ? sigmoid_f(logits[(size_t)t * E + e]) : 0.0f;
    float S = s, SD = dg * s;
    for (int o = 16; o > 0; o >>= 1) {
      S += __shfl_xor_sync(0xffffffffu, S, o);
      SD += __shfl_xor_sync(0xffffffffu, SD, o);
    }
    const float ds = route_scale * (dg / S - SD / (S * S));
    out = ds * s * (1.0f - s);
  } else {
    const float p = act ? gate[(size_t)t * k + lane] / route_scale : 0.0f;
    float PD = p * dg;
    for (int o = 16; o > 0; o >>= 1) PD += __shfl_xor_sync(0xffffffffu, PD, o);
    out = route_scale * p * (dg - PD);
  }
  if (act) {
    row[e] = out;
    if (rowb) rowb[e] = __float2bfloat16_rn(out);
  }
}

// dx[t] = sum_j dxp[inv_row[t][j]] + dxs[t] + dxr[t], fp32 in slot order,
// rounded once to the storage type. dxs / dxr may be null.
template <typename T>
__global__ void __launch_bounds__(256) unpermute_sum_kernel(
    const float* __restrict__ dxp, const int* __restrict__ inv_row, const float* __restrict__ dxs,
    const float* __restrict__ dxr, T* __restrict__ dx, int d, int k) {
  const int t = blockIdx.x;
  __shared__ int rows[kMaxTopK];
  if (threadIdx.x < k) rows[threadIdx.x] = inv_row[(size_t)t * k + threadIdx.x];
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float v = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int r = rows[j];
      if (r >= 0) v += dxp[(size_t)r * d + c];
    }
    if (dxs) v += dxs[(size_t)t * d + c];
    if (dxr) v += dxr[(size_t)t * d + c];
    dx[(size_t)t * d + c] = from_f32<T>(v);
  }
}

}  // namespace

cudaError_t launch_swiglu_bwd(int dtype, const void* a, const void* b, const float* dhp,
                              const int* inv_row, const float* gate, float* dgate, void* hg, void* dadb,
                              int n_rows, int f, int f_pad, cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  if (dtype == MOE_DTYPE_F32)
    swiglu_bwd_kernel<float><<<n_rows, 256, 0, s>>>((const float*)a, (const float*)b, dhp, inv_row, gate,
                                                    dgate, (float*)hg, (float*)dadb, f, f_pad);
  else
    swiglu_bwd_kernel<__nv_bfloat16><<<n_rows, 256, 0, s>>>(
        (const __nv_bfloat16*)a, (const __nv_bfloat16*)b, dhp, inv_row, gate, dgate, (__nv_bfloat16*)hg,
        (__nv_bfloat16*)dadb, f, f_pad);
  return cudaGetLastError();
}

cudaError_t launch_gate_bwd(const float* logits, const int* idx, const float* gate, const float* dgate,
                            float* dl, void* dl_bf16, int e_pad, int T, int E, int k, int gate_mode,
                            float route_scale, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  gate_bwd_kernel<<<ceil_div(T, 8), 256, 0, s>>>(logits, idx, gate, dgate, dl, dl_bf16, e_pad, T, E, k,
                                                 gate_mode, route_scale);
  return cudaGetLastError();
}

cudaError_t launch_unpermute_sum(int dtype, const float* dxp, const int* inv_row, const float* dxs,
                                 const float* dxr, void* dx, int T, int d, int k, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (dtype == MOE_DTYPE_F32)
    unpermute_sum_kernel<float><<<T, 256, 0, s>>>(dxp, inv_row, dxs, dxr, (float*)dx, d, k);
  else
    unpermute_sum_kernel<__nv_bfloat16><<<T, 256, 0, s>>>(dxp, inv_row, dxs, dxr, (__nv_bfloat16*)dx, d, k);
  return cudaGetLastError();
}

}  // namespace moe
