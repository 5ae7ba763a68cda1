// Grouped GEMM on the fp32 FMA pipes, for the fp32 storage type (router
// logits and both expert GEMMs). TF32 tensor cores round operands to 10
// mantissa bits, too coarse for an fp32 path, so this kernel stays on FFMA.
//
//   dual:   out[r][n] = SiLU(sum_c A[r][c] B1[n][c]) * (sum_c A[r][c] B3[n][c])
//   single: out[r][n] = act(sum_c A[r][c] B1[n][c] + bias[n]), act = identity or
//           GELU, bias optional (the generic expert W2 phi(W1 u + b1) + b2 of
//           "Lesson 2 - From the Dense FFN to a Layer of Experts", section 2)
//
// Segment s < n_routed covers packed rows [offsets[s], offsets[s+1]) of A and
// uses expert s's matrices B1[s], B3[s] (N x K each). Segment n_routed, when
// shared_rows > 0, is the dense segment: all rows of A_s against B1_s/B3_s.
// (SwiGLU equation of the Sparse MoE FFN note: FFN(u) = W2 (SiLU(W1 u) * W3 u).)
//
// Tile: 64 rows x 64 columns per block of 256 threads, 4 x 4 outputs per
// thread, K staged through shared memory 16 at a time.
#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

struct Seg {
  const void* a; const void* b1; const void* b3; void* out;
  int row0, rows, N, K;
  const float* bias;   // this segment's bias row [N], or null
  void* pre_a; void* pre_b;   // dual: optional pre-activation outputs
};

template <typename TI, typename TO, bool DUAL>
__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtGemmParams p) {
  __shared__ float As[TK][TM + 4];
  __shared__ float B1s[TK][TN + 4];
  __shared__ float B3s[DUAL ? TK : 1][TN + 4];

  // Find this block's (segment, row tile).
  int bx = blockIdx.x;
  Seg sg;
  bool found = false;
  for (int s = 0; s < p.n_routed; ++s) {
    // Caller offsets clamped into the packed rows (block 0 records a bad one);
    // a decreasing pair is an empty segment.
    uint32_t* err = blockIdx.x == 0 && blockIdx.y == 0 ? p.err : nullptr;
    const int r0 = clamp_offset(p.offsets[s], p.max_rows, err);
    const int rows = max(0, clamp_offset(p.offsets[s + 1], p.max_rows, err) - r0);
    const int tiles = (rows + TM - 1) / TM;
    if (bx < tiles) {
      sg = Seg{p.a, (const char*)p.b1 + (size_t)s * p.N * p.K * sizeof(TI),
               DUAL ? (const char*)p.b3 + (size_t)s * p.N * p.K * sizeof(TI) : nullptr,
               p.out, r0 + bx * TM, min(TM, rows - bx * TM), p.N, p.K,
               p.bias1 ? p.bias1 + (size_t)s * p.N : nullptr, p.pre_a, p.pre_b};
      found = true;
      break;
    }
    bx -= tiles;
  }
  if (!found && p.shared_rows > 0) {
    const int tiles = (p.shared_rows + TM - 1) / TM;
    if (bx < tiles) {
      sg = Seg{p.a_s, p.b1_s, p.b3_s, p.out_s, bx * TM, min(TM, p.shared_rows - bx * TM), p.N_s, p.K_s,
               p.bias1_s, p.pre_a_s, p.pre_b_s};
      found = true;
    }
  }
  if (!found) return;
  const int n0 = blockIdx.y * TN;
  if (n0 >= sg.N) return;

  const TI* A = (const TI*)sg.a;
  const TI* B1 = (const TI*)sg.b1;
  const TI* B3 = (const TI*)sg.b3;
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  float acc1[4][4] = {}, acc3[4][4] = {};

  for (int k0 = 0; k0 < sg.K; k0 += TK) {
    // Stage A (64 x 16) and B (64 x 16), transposed to k-major, zero-padded.
    for (int i = tid; i < TM * TK; i += 256) {
      const int r = i / TK, c = i % TK;
      float va = 0.f, v1 = 0.f, v3 = 0.f;
      if (k0 + c < sg.K) {
        if (r < sg.rows) va = to_f32(A[(size_t)(sg.row0 + r) * sg.K + k0 + c]);
        if (n0 + r < sg.N) {
          v1 = to_f32(B1[(size_t)(n0 + r) * sg.K + k0 + c]);
          if (DUAL) v3 = to_f32(B3[(size_t)(n0 + r) * sg.K + k0 + c]);
        }
      }
      As[c][r] = va;
      B1s[c][r] = v1;
      if (DUAL) B3s[c][r] = v3;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b1[4], b3[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b1[i] = B1s[kk][tx * 4 + i];
        if (DUAL) b3[i] = B3s[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
          if (DUAL) acc3[i][j] = fmaf(a[i], b3[j], acc3[i][j]);
        }
    }
    __syncthreads();
  }

  TO* out = (TO*)sg.out;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= sg.rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= sg.N) continue;
      float v = acc1[i][j];
      if (DUAL) {
        if (sg.pre_a) {
          const size_t o = (size_t)(sg.row0 + r) * sg.N + n;
          static_cast<TO*>(sg.pre_a)[o] = from_f32<TO>(v);
          static_cast<TO*>(sg.pre_b)[o] = from_f32<TO>(acc3[i][j]);
        }
        v = (v / (1.0f + expf(-v))) * acc3[i][j];
      } else {
        if (sg.bias) v += sg.bias[n];
        if (p.act == kActGelu) v = gelu_erf(v);
      }
      out[(size_t)(sg.row0 + r) * sg.N + n] = from_f32<TO>(v);
    }
  }
}

}  // namespace

cudaError_t launch_simt_gemm(int in_dtype, int out_f32, const SimtGemmParams& p, cudaStream_t s) {
  const int row_tiles = ceil_div(p.max_rows, TM) + p.n_routed + ceil_div(p.shared_rows, TM);
  const int nmax = p.N > p.N_s ? p.N : p.N_s;
  if (row_tiles <= 0 || nmax <= 0) return cudaSuccess;
  dim3 grid(row_tiles, ceil_div(nmax, TN));
  if (in_dtype == MOE_DTYPE_F32) {
    if (p.dual) simt_gemm_kernel<float, float, true><<<grid, 256, 0, s>>>(p);
    else simt_gemm_kernel<float, float, false><<<grid, 256, 0, s>>>(p);
  } else if (out_f32) {
    if (p.dual) simt_gemm_kernel<__nv_bfloat16, float, true><<<grid, 256, 0, s>>>(p);
    else simt_gemm_kernel<__nv_bfloat16, float, false><<<grid, 256, 0, s>>>(p);
  } else {
    if (p.dual) simt_gemm_kernel<__nv_bfloat16, __nv_bfloat16, true><<<grid, 256, 0, s>>>(p);
    else simt_gemm_kernel<__nv_bfloat16, __nv_bfloat16, false><<<grid, 256, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace moe
