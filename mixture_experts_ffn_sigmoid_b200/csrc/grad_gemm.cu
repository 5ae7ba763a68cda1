// Strided grouped GEMM on the FMA pipes for the backward pass.
//
//   C_s(i, j) (+)= sum_k A(i, k) * B_s(j, k)
//
// with every operand addressed through explicit strides, so one kernel
// serves the transposed products of the backward pass (gradients with
// respect to the inputs, contracting over a weight's row index, and with
// respect to the weights, contracting over a segment's tokens):
//
//   A(i, k)   = A[i * a_si + k * a_sk]
//   B_s(j, k) = B[s * b_seg + j * b_sj + k * b_sk]
//   C_s(i, j) = C[s * c_seg + i * c_si + j]
//
// Segments (SwiGLU experts of the Sparse MoE FFN note's "Packed forward",
// expert e = packed rows [offsets[e], offsets[e+1])):
//   kSegRows: segment s owns rows i in [off[s], off[s+1]) (C_s ignores c_seg);
//             all K columns; with offsets == null one segment of max_rows rows.
//   kSegK:    segment s owns reduction indices k in [off[s], off[s+1]) and its
//             own output C_s of M x N; with offsets == null there is one
//             segment of K reduction indices.
//
// fp32 accumulation in registers (4 x 4 per thread, 64 x 64 per block, K
// staged through shared memory 16 at a time); C is fp32 or the storage type.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <typename T> __device__ __forceinline__ float ld_f32(const T* p) { return to_f32(*p); }

template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256) grad_gemm_kernel(GradGemmParams p) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  int seg = 0, i0 = 0, i1 = 0, k0 = 0, k1 = 0;
  if (p.seg_mode == kSegRows && !p.offsets) {
    // One dense segment of max_rows rows.
    i0 = blockIdx.x * TM;
    i1 = p.max_rows;
    if (i0 >= i1) return;
    k1 = p.K;
  } else if (p.seg_mode == kSegRows) {
    // blockIdx.x walks the row tiles of all segments in order.
    int bx = blockIdx.x;
    bool found = false;
    for (int s = 0; s < p.n_seg; ++s) {
      const int r0 = p.offsets[s], rows = p.offsets[s + 1] - r0;
      const int tiles = (rows + TM - 1) / TM;
      if (bx < tiles) {
        seg = s;
        i0 = r0 + bx * TM;
        i1 = r0 + rows;
        found = true;
        break;
      }
      bx -= tiles;
    }
    if (!found) return;
    k0 = 0;
    k1 = p.K;
  } else {
    // blockIdx.x = segment * row tiles + row tile.
    const int mt = (p.M + TM - 1) / TM;
    seg = blockIdx.x / mt;
    i0 = (blockIdx.x - seg * mt) * TM;
    i1 = p.M;
    if (p.offsets) {
      k0 = p.offsets[seg];
      k1 = p.offsets[seg + 1];
    } else {
      k0 = 0;
      k1 = p.K;
    }
  }
  const int j0 = blockIdx.y * TN;
  if (j0 >= p.N) return;
  const TA* A = static_cast<const TA*>(p.a);
  const TB* B = static_cast<const TB*>(p.b) + (size_t)seg * p.b_seg;
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  float acc[4][4] = {};
  for (int kb = k0; kb < k1; kb += TK) {
    for (int e = tid; e < TM * TK; e += 256) {
      // Consecutive threads walk i (or j) when that is the unit-stride index.
      int r, c;
      if (p.a_si == 1) { r = e % TM; c = e / TM; } else { r = e / TK; c = e % TK; }
      const int i = i0 + r, k = kb + c;
      As[c][r] = (i < i1 && k < k1) ? ld_f32(A + (size_t)i * p.a_si + (size_t)k * p.a_sk) : 0.0f;
    }
    for (int e = tid; e < TN * TK; e += 256) {
      int r, c;
      if (p.b_sj == 1) { r = e % TN; c = e / TN; } else { r = e / TK; c = e % TK; }
      const int j = j0 + r, k = kb + c;
      Bs[c][r] = (j < p.N && k < k1) ? ld_f32(B + (size_t)j * p.b_sj + (size_t)k * p.b_sk) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = As[kk][ty * 4 + q];
        b[q] = Bs[kk][tx * 4 + q];
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[q][w] = fmaf(a[q], b[w], acc[q][w]);
    }
    __syncthreads();
  }
  TC* C = static_cast<TC*>(p.c) + (p.seg_mode == kSegK ? (size_t)seg * p.c_seg : 0);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = i0 + ty * 4 + q;
    if (i >= i1) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int j = j0 + tx * 4 + w;
      if (j >= p.N) continue;
      TC* dst = C + (size_t)i * p.c_si + j;
      float v = acc[q][w];
      if (p.accumulate) v += to_f32(*dst);
      *dst = from_f32<TC>(v);
    }
  }
}

template <typename TA, typename TB, typename TC>
cudaError_t launch_typed(const GradGemmParams& p, cudaStream_t s) {
  int gx;
  if (p.seg_mode == kSegRows)
    gx = ceil_div(p.max_rows, TM) + (p.offsets ? p.n_seg : 0);
  else
    gx = (p.offsets ? p.n_seg : 1) * ceil_div(p.M, TM);
  if (gx <= 0 || p.N <= 0) return cudaSuccess;
  dim3 grid(gx, ceil_div(p.N, TN));
  grad_gemm_kernel<TA, TB, TC><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grad_gemm(const GradGemmParams& p, cudaStream_t s) {
  const bool bf = p.dtype == MOE_DTYPE_BF16;
  using bf16 = __nv_bfloat16;
  if (!bf) return launch_typed<float, float, float>(p, s);
  if (p.a_f32) {
    return p.c_f32 ? launch_typed<float, bf16, float>(p, s) : launch_typed<float, bf16, bf16>(p, s);
  }
  return p.c_f32 ? launch_typed<bf16, bf16, float>(p, s) : launch_typed<bf16, bf16, bf16>(p, s);
}

}  // namespace moe
