// Weight gradients of the backward pass on the tensor cores (tcgen05):
//
//   D_s[m][n] = sum_{r in segment s} P[r][m] * Q[r][n]
//
// P and Q are row-major activations over the packed rows r (for dW1 of
// expert e: P = da, Q = x_perm over the expert's rows; for dW2: P = dy
// gathered in packed order, Q = g h). The contraction runs over a
// segment's rows, so both operands are MN-major (m, n contiguous) and the
// reduction length is ragged: expert s owns rows [offsets[s], offsets[s+1])
// (Sparse MoE FFN note, "Packed forward": each expert sees the tokens that
// chose it). Segments no row belongs to get D_s = 0.
//
// Tiles: 128 or 256 m x 256 n per CTA (one M=128, N=256 MMA per 16 rows for
// each 128-row M block; two blocks share the staged Q tile), rows in blocks
// of 64. Both operands arrive as 64 x 64 TMA boxes (128-byte swizzle,
// MN-major: 64-element M/N groups 8 KB apart, 8-row groups 1 KB apart).
// Rows of the last block past the segment's end belong to the next segment:
// the MMAs (16 rows each) stop at the one holding the segment's last row,
// and the MMA warp zeroes that MMA's rows past the end in the P tile in
// shared memory, so they add nothing (Q's rows there are finite data or
// zero fill).
//
// Roles (320 threads, one CTA per SM, persistent over tiles ordered
// segment-major, so CTAs running at once share a segment's rows in L2):
//   warp 0 lane 0 : TMA producer into a 4-stage ring (3 with two M blocks)
//   warp 1        : TMEM allocator; zero-fills partial blocks; lane 0 issues
//                   tcgen05.mma and tcgen05.commit
//   warps 2..9    : epilogue; warp w reads TMEM lane quarter w % 4 of one M
//                   block (or half the columns with one block), 32 columns per
//                   load wait, and writes 32 x 32 boxes with TMA stores
// Every wait is bounded, as in the forward GEMM.
#include "umma_common.cuh"

namespace moe {
namespace {

// All but the newest committed bulk group have read their shared memory.
__device__ __forceinline__ void bulk_wait_read_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// The output map: bf16 [n_seg][M][N], 64-byte swizzle, 32 x 32 x 1 boxes
// (stores clip at each dimension's bound).
bool make_out_tmap(CUtensorMap* tm, void* base, long long n, long long m, long long segs) {
  auto fn = get_encode_fn();
  if (!fn || n <= 0 || m <= 0 || segs <= 0 || (n * 2) % 16) return false;
  cuuint64_t dims[3] = {(cuuint64_t)n, (cuuint64_t)m, (cuuint64_t)segs};
  cuuint64_t strides[2] = {(cuuint64_t)(n * 2), (cuuint64_t)(m * n * 2)};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tile shapes. WG_MB 128-row M blocks per tile: two blocks share each
// staged Q tile, cutting the operands read per output byte by a third, but
// their accumulators (2 x 256 TMEM columns) fill TMEM, so the next tile's
// MMAs wait for the epilogue; one block keeps two accumulator stages. Long
// contractions (hundreds of rows per segment) take two blocks, short ones one.
template <int MB> struct WgShape {
  static constexpr int BM = 128 * MB;
  static constexpr int ACC_STAGES = MB == 1 ? 2 : 1;
  static constexpr int STAGES = MB == 1 ? 4 : 3;
};
constexpr int WG_BN = 256;
constexpr int WG_BK = 64;
constexpr int WG_BOX = 64 * 64 * 2;                      // one 64 x 64 bf16 box
constexpr int WG_B_BYTES = 4 * WG_BOX;                   // 256 n x 64 rows
constexpr int WG_THREADS = 320;
constexpr int WG_EPI_WARPS = 8;
constexpr int WG_STG_BYTES = 2 * 32 * 32 * 2;            // one warp's two 32 x 32 output boxes
constexpr int WG_OBOX = 32 * 32 * 2;                     // one 32 x 32 bf16 output box (64-byte rows)
constexpr int WG_TMEM_COLS = 512;
template <int MB> constexpr int wg_a_bytes() { return 2 * MB * WG_BOX; }
template <int MB> constexpr int wg_stage_bytes() { return wg_a_bytes<MB>() + WG_B_BYTES; }
template <int MB> constexpr int wg_smem() {
  return 1024 + 1024 + WgShape<MB>::STAGES * wg_stage_bytes<MB>() + WG_EPI_WARPS * WG_STG_BYTES;
}

struct WgTile {
  int seg, m0, n0, r0, rows, nk;
};

template <int BM>
__device__ __forceinline__ WgTile wg_tile(const WgradParams& p, int tile, int mt, int nt) {
  WgTile t;
  const int per_seg = mt * nt;
  t.seg = tile / per_seg;
  const int rem = tile - t.seg * per_seg;
  t.m0 = (rem / nt) * BM;
  t.n0 = (rem - (rem / nt) * nt) * WG_BN;
  if (p.offsets) {
    t.r0 = p.offsets[t.seg];
    t.rows = p.offsets[t.seg + 1] - t.r0;
  } else {
    t.r0 = 0;
    t.rows = p.k_total;
  }
  t.nk = t.rows > 0 ? ceil_div(t.rows, WG_BK) : 0;
  return t;
}

__device__ __forceinline__ void st_shared_zero16(uint32_t addr) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
}

template <int WG_MB>
__global__ void __launch_bounds__(WG_THREADS, 1)
    wgrad_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                 const __grid_constant__ CUtensorMap tmD, const WgradParams p) {
  constexpr int WG_BM = WgShape<WG_MB>::BM;
  constexpr int WG_ACC_STAGES = WgShape<WG_MB>::ACC_STAGES;
  constexpr int WG_STAGES = WgShape<WG_MB>::STAGES;
  constexpr int WG_A_BYTES = wg_a_bytes<WG_MB>();
  constexpr int WG_STAGE_BYTES = wg_stage_bytes<WG_MB>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty_bar = full_bar + WG_STAGES;
  uint64_t* accf_bar = empty_bar + WG_STAGES;
  uint64_t* acce_bar = accf_bar + 2;
  uint64_t* drain_bar = acce_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  uint8_t* ring = smem + 1024;
  uint8_t* stage_out = ring + WG_STAGES * WG_STAGE_BYTES;   // epilogue staging, one box per warp

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < WG_STAGES; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&accf_bar[i]), 1);
      mbar_init(smem_u32(&acce_bar[i]), WG_EPI_WARPS);   // one arrival per epilogue warp
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0u;
    fence_mbar_init();
    tmap_prefetch(&tmP);
    tmap_prefetch(&tmQ);
    tmap_prefetch(&tmD);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), WG_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int mt = ceil_div(p.M, WG_BM), nt = ceil_div(p.N, WG_BN);
  const int total = p.n_seg * mt * nt;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const WgTile t = wg_tile<WG_BM>(p, tile, mt, nt);
      for (int kb = 0; kb < t.nk; ++kb) {
        if (!wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.err, p.timeout_ns, true)) {
          ok = false;
          break;
        }
        const uint32_t fb = smem_u32(&full_bar[stage]);
        const uint32_t sa = smem_u32(ring + stage * WG_STAGE_BYTES);
        const uint32_t sbq = sa + WG_A_BYTES;
        const int r = t.r0 + kb * WG_BK;
        // Boxes wholly past M or N are not loaded: the rows (columns) of D
        // they feed are never stored.
        const int na = min(2 * WG_MB, ceil_div(p.M - t.m0, 64)), nb = min(4, ceil_div(p.N - t.n0, 64));
        mbar_expect_tx(fb, (uint32_t)(na + nb) * WG_BOX);
        for (int h = 0; h < na; ++h) tma_load_2d(sa + h * WG_BOX, &tmP, t.m0 + h * 64, r, fb);
        for (int h = 0; h < nb; ++h) tma_load_2d(sbq + h * WG_BOX, &tmQ, t.n0 + h * 64, r, fb);
        if (++stage == WG_STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool issued = false, ok = true;
    const uint32_t idesc = idesc_bf16_f32(128, WG_BN) | (1u << 15) | (1u << 16);
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const WgTile t = wg_tile<WG_BM>(p, tile, mt, nt);
      if (t.nk == 0) continue;                  // the epilogue writes zeros
      // Lane 0 waits; the outcome is broadcast so the warp stays converged.
      int w_ok = lane == 0 ? (int)wait_bounded(smem_u32(&acce_bar[acc]), acc_phase ^ 1u, abort_flag, p.err,
                                               p.timeout_ns, true) : 0;
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + (uint32_t)(acc * WG_BN);   // block b adds b * WG_BN (WG_MB == 2)
      const int na = min(2 * WG_MB, ceil_div(p.M - t.m0, 64));
      for (int kb = 0; kb < t.nk; ++kb) {
        w_ok = lane == 0 ? (int)wait_bounded(smem_u32(&full_bar[stage]), phase, abort_flag, p.err, p.timeout_ns,
                                             true) : 0;
        if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_u32(ring + stage * WG_STAGE_BYTES);
        const int valid = min(WG_BK, t.rows - kb * WG_BK);
        // MMAs of 16 rows each: only those that reach a valid row run, and
        // only the rows past `valid` inside the last of them are zeroed.
        const int n_kk = (valid + 15) / 16;
        const int pad = n_kk * 16 - valid;
        if (pad > 0) {
          // Every lane sees the completed phase itself (it has completed, so
          // the wait returns at once) before overwriting rows TMA wrote.
          wait_bounded(smem_u32(&full_bar[stage]), phase, abort_flag, p.err, p.timeout_ns, false);
          // Rows valid .. valid + pad - 1 of the loaded 64-row P boxes: 128
          // bytes each, 8 x 16 B.
          const int n16 = pad * na * 8;
          for (int i = lane; i < n16; i += 32) {
            const int h = i / (pad * 8);
            const int rem = i - h * pad * 8;
            st_shared_zero16(sa + h * WG_BOX + (valid + rem / 8) * 128 + (rem % 8) * 16);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        tc_fence_after();
        if (lane == 0) {
          const uint64_t b_desc = sw128_mn_desc(sa + WG_A_BYTES);
#pragma unroll
          for (int blk = 0; blk < WG_MB; ++blk) {
            if (blk * 128 >= p.M - t.m0) break;   // block wholly past M: not loaded, not needed
            const uint64_t a_desc = sw128_mn_desc(sa + blk * 2 * WG_BOX);
#pragma unroll
            for (int kk = 0; kk < WG_BK / 16; ++kk) {
              if (kk >= n_kk) break;
              const uint64_t koff = (uint64_t)((kk * 2 * 1024) >> 4);   // two 8-row groups per 16 rows
              umma_bf16(d + blk * WG_BN, a_desc + koff, b_desc + koff, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(smem_u32(&empty_bar[stage]));
        }
        __syncwarp();
        issued = true;
        if (++stage == WG_STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(smem_u32(&accf_bar[acc]));
      __syncwarp();
      if (++acc == WG_ACC_STAGES) { acc = 0; acc_phase ^= 1u; }
    }
    if (issued && lane == 0) {   // every MMA completes before TMEM is freed
      umma_commit(smem_u32(drain_bar));
      wait_bounded(smem_u32(drain_bar), 0u, abort_flag, p.err, p.timeout_ns, false);
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    // Each warp converts its 32 rows x 32 columns at a time to bf16 into one
    // of two staging boxes (row = lane, 16-byte chunk c at c ^ ((row >> 1) & 3),
    // the layout TMA's 64-byte swizzle reads) and lane 0 stores the box with
    // TMA. With two boxes a chunk waits only for the store issued two chunks
    // earlier to have read its box out, so the stores overlap the next
    // chunk's TMEM loads and conversion. The 3-D output map clips rows past M
    // and columns past N.
    const int q = warp & 3;                    // TMEM lane quarter this warp may read
    // Warps 2-5 and 6-9 split the tile: by M block when there are two (each
    // warp then stores all 256 columns of its 32 rows), else by column half.
    const int grp = (warp - 2) >> 2;
    const int blk = WG_MB == 2 ? grp : 0;
    const int ncol = WG_MB == 2 ? WG_BN : WG_BN / 2;
    const int cbeg = WG_MB == 2 ? 0 : grp * (WG_BN / 2);
    const uint32_t box0 = smem_u32(stage_out + (warp - 2) * WG_STG_BYTES);
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t nbox = 0;                         // boxes this warp has stored (selects the buffer)
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const WgTile t = wg_tile<WG_BM>(p, tile, mt, nt);
      const int mrow = t.m0 + blk * 128 + q * 32;   // first row of this warp's boxes
      const int nbeg = t.n0 + cbeg;
      if (t.nk == 0) {
        // No row chose this segment: its gradient is zero. Store a zeroed
        // staging box over the warp's 32 x 32 output boxes.
        if (mrow < p.M && nbeg < p.N) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 4; ++c) st_shared_zero16(box0 + lane * 64 + c * 16);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            for (int c0 = 0; c0 < ncol && nbeg + c0 < p.N; c0 += 32) tma_store_3d(&tmD, box0, nbeg + c0, mrow, t.seg);
            bulk_commit();
          }
          nbox = 1;   // the next box written is the second one
        }
        continue;
      }
      if (!wait_bounded(smem_u32(&accf_bar[acc]), acc_phase, abort_flag, p.err, p.timeout_ns, true)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) +
                             (uint32_t)((WG_MB == 2 ? blk : acc) * WG_BN + cbeg);
      for (int c0 = 0; c0 < ncol; c0 += 32) {
        if (nbeg + c0 >= p.N || mrow >= p.M) break;
        uint32_t ra[16], rb[16];
        tmem_ld16x2_wait(taddr + c0, taddr + c0 + 16, ra, rb);
        const uint32_t box = box0 + (nbox & 1u) * WG_OBOX;
        // The store of two boxes ago (same buffer) must have read it out.
        if (lane == 0) bulk_wait_read_but_one();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = 8 * c + 2 * j;   // columns i, i + 1 of the 32
            const float lo = __uint_as_float(i < 16 ? ra[i] : rb[i - 16]);
            const float hi = __uint_as_float(i + 1 < 16 ? ra[i + 1] : rb[i + 1 - 16]);
            const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
            w[j] = *reinterpret_cast<const uint32_t*>(&h);
          }
          const uint32_t dst = box + lane * 64 + ((c ^ ((lane >> 1) & 3)) * 16);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                       "r"(w[3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmD, box, nbeg + c0, mrow, t.seg);
          bulk_commit();
        }
        ++nbox;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acce_bar[acc]));
      if (++acc == WG_ACC_STAGES) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait_all();   // staging boxes stay live until written out
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, WG_TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_wgrad(const WgradParams& p, int num_sms, cudaStream_t s) {
  if (p.n_seg <= 0 || p.M <= 0 || p.N <= 0) return cudaSuccess;
  CUtensorMap tP, tQ, tD;
  if (!make_tmap_strided(&tP, p.P, p.M, p.p_rows, p.ldP * 2, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_strided(&tQ, p.Q, p.N, p.q_rows, p.ldQ * 2, 64)) return cudaErrorInvalidValue;
  if (!make_out_tmap(&tD, p.out, p.N, p.M, p.n_seg)) return cudaErrorInvalidValue;
  // Two M blocks per tile once segments average more than 256 rows.
  const long long rows_per_seg = (p.offsets ? (long long)p.p_rows : (long long)p.k_total) / p.n_seg;
  const bool two = rows_per_seg > 256;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static int attr_done_mask[2] = {0, 0};
  int& mask = attr_done_mask[two ? 1 : 0];
  if (!(dev < 32 && ((mask >> dev) & 1))) {
    e = two ? cudaFuncSetAttribute(wgrad_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, wg_smem<2>())
            : cudaFuncSetAttribute(wgrad_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, wg_smem<1>());
    if (e != cudaSuccess) return e;
    if (dev < 32) mask |= 1 << dev;
  }
  const int bm = two ? WgShape<2>::BM : WgShape<1>::BM;
  const long long tiles = (long long)p.n_seg * ceil_div(p.M, bm) * ceil_div(p.N, WG_BN);
  const int grid = (int)(tiles < num_sms ? tiles : num_sms);
  if (two) wgrad_kernel<2><<<grid, WG_THREADS, wg_smem<2>(), s>>>(tP, tQ, tD, p);
  else wgrad_kernel<1><<<grid, WG_THREADS, wg_smem<1>(), s>>>(tP, tQ, tD, p);
  return cudaGetLastError();
}

}  // namespace moe
