// C ABI of the MoE FFN forward pass: argument checks, workspace carving and
// kernel enqueue. No entry point allocates, synchronises or copies to the
// host (moe_get_device_error excepted, which exists to do exactly that).
#include <math.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include "moe_internal.cuh"

namespace moe {

int device_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

namespace {

constexpr size_t kAlign = 256;

// A named NVTX range over the host-side enqueue of an entry point or stage,
// for timeline tools (a no-op unless one is attached).
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

struct Layout {
  size_t err, logits, ccount, cbase, thist, tbase, idx, gate, counts, offsets, inv_row, perm_src;
  size_t x_perm, h, h_s, y_perm, y_s, total;
};

// Byte offset, inside the error region (cleared at the start of every call),
// of the fused router's device-wide tile counter.
constexpr size_t kDoneCountOffset = 64;

// The bf16 router of up to 256 experts runs as one fused kernel; otherwise
// a GEMM (split contraction for bf16) feeds the separate top-k and scans.
bool fused_route(const moe_config& c) { return router_fused_supported(c.dtype, c.E); }

// Workspace regions, each 256-byte aligned. Sizes cover the worst case of
// T*k packed rows plus T shared rows.
Layout layout_of(const moe_config& c) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + kAlign - 1) / kAlign * kAlign;
    return o;
  };
  const size_t es = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
  const size_t T = (size_t)c.T, k = (size_t)c.k, E = (size_t)c.E, d = (size_t)c.d, f = (size_t)c.f;
  const size_t fs = (size_t)c.f_shared;
  const size_t nch = (T + kChunk - 1) / kChunk;
  L.err = take(kAlign);
  // Unfused bf16 router logits come as partial sums of a split contraction.
  const size_t n_part =
      (c.dtype == MOE_DTYPE_BF16 && !fused_route(c)) ? (size_t)router_gemm_splits(c.T, c.E, c.d) : 1;
  const size_t ntiles = (T + (size_t)(kChunk * kTileChunks) - 1) / (kChunk * kTileChunks);
  L.logits = take(n_part * T * E * 4);
  L.ccount = take(nch * E * 4);
  L.cbase = take(nch * E * 4);
  L.thist = take(ntiles * E * 4);
  L.tbase = take(ntiles * E * 4);
  L.idx = take(T * k * 4);
  L.gate = take(T * k * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.inv_row = take(T * k * 4);
  L.perm_src = take(T * k * 4);
  L.x_perm = take(T * k * d * es);
  L.h = take(T * k * f * es);
  L.h_s = take(T * fs * es);
  L.y_perm = take(T * k * d * es);
  L.y_s = take(fs > 0 ? T * d * es : 0);
  L.total = off;
  return L;
}

moe_status check_config(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d <= 0 || c->E <= 0 || c->k <= 0 || c->f <= 0 || c->f_shared < 0)
    return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_DTYPE_F32 && c->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->gate_mode != MOE_GATE_SOFTMAX && c->gate_mode != MOE_GATE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (c->k > c->E) return MOE_ERR_INVALID_ARG;
  if (!(c->route_scale > 0.0f) || !isfinite(c->route_scale)) return MOE_ERR_INVALID_ARG;
  if (c->n_groups < 1 || c->topk_groups < 1 || c->topk_groups > c->n_groups) return MOE_ERR_INVALID_ARG;
  if (c->E % c->n_groups != 0) return MOE_ERR_INVALID_ARG;
  if (c->n_groups > 1 && c->E / c->n_groups < 2) return MOE_ERR_INVALID_ARG;
  if ((long long)c->topk_groups * (c->E / c->n_groups) < c->k) return MOE_ERR_INVALID_ARG;
  if (c->E > kMaxExperts || c->k > kMaxTopK || c->n_groups > kMaxGroups) return MOE_ERR_UNSUPPORTED;
  const int v = c->dtype == MOE_DTYPE_F32 ? 4 : 8;
  if (c->d % v || c->f % v || c->f_shared % v) return MOE_ERR_MISALIGNED;
  // Row indices (packed rows, weight rows) travel as 32-bit TMA coordinates.
  const long long lim = 0x7fffffffLL;
  if ((long long)c->T * (c->k + 1) >= lim || (long long)c->E * c->f >= lim ||
      (long long)c->E * c->d >= lim)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A required pointer: NULL -> invalid, not 16-byte aligned -> misaligned.
moe_status need(const void* p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  return aligned16(p) ? MOE_OK : MOE_ERR_MISALIGNED;
}
moe_status need4(const void* p) {   // int32 / fp32 side arrays: 4-byte alignment
  if (!p) return MOE_ERR_INVALID_ARG;
  return (reinterpret_cast<uintptr_t>(p) & 3u) == 0 ? MOE_OK : MOE_ERR_MISALIGNED;
}

#define MOE_TRY(expr)                   \
  do {                                  \
    const moe_status _st = (expr);      \
    if (_st != MOE_OK) return _st;      \
  } while (0)
#define MOE_CUDA(expr)                          \
  do {                                          \
    if ((expr) != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

moe_status check_ws(const moe_config& c, void* ws, size_t ws_bytes) {
  MOE_TRY(need(ws));
  if (ws_bytes < layout_of(c).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

// Whether enqueue_route can also write the permute's row maps: the fused
// router with a single 128-token tile, whose last step knows the offsets and
// every chunk's masks (decode-sized batches).
bool route_writes_maps(const moe_config& c) { return fused_route(c) && c.T <= 128; }

// Router logits -> top-k, gates, chunk histograms -> counts, chunk bases,
// offsets; with inv_row and perm_src (only where route_writes_maps) also the
// row maps the permute would write.
moe_status enqueue_route(const moe_config& c, const void* x, const void* w_router, const float* bias,
                         int* idx, float* gate, int* counts, int* offsets, void* ws, cudaStream_t s,
                         int* inv_row = nullptr, int* perm_src = nullptr) {
  const Layout L = layout_of(c);
  float* logits = at<float>(ws, L.logits);
  const TopkArgs tk = {c.E, c.k, c.gate_mode, c.n_groups, c.topk_groups, c.route_scale, bias};
  if ((inv_row || perm_src) && !route_writes_maps(c)) return MOE_ERR_INVALID_ARG;
  if (fused_route(c)) {
    FusedRouterLaunch a = {x, w_router, c.T, c.E, c.d, tk, logits, idx, gate, at<int>(ws, L.cbase),
                           at<int>(ws, L.thist), at<int>(ws, L.tbase), counts, offsets,
                           at<uint32_t>(ws, L.err), at<uint32_t>(ws, L.err + kDoneCountOffset)};
    a.inv_row = inv_row;
    a.perm_src = perm_src;
    MOE_CUDA(launch_router_fused(a, s));
    return MOE_OK;
  }
  int n_part = 1;
  if (c.dtype == MOE_DTYPE_BF16) {
    n_part = router_gemm_splits(c.T, c.E, c.d);
    MOE_CUDA(launch_router_gemm(x, w_router, c.T, c.E, c.d, logits, n_part, at<uint32_t>(ws, L.err), s));
  } else {
    SimtGemmParams g = {};
    g.dual = 0;
    g.n_routed = 0;
    g.shared_rows = c.T;
    g.a_s = x;
    g.b1_s = w_router;
    g.out_s = logits;
    g.N_s = c.E;
    g.K_s = c.d;
    MOE_CUDA(launch_simt_gemm(c.dtype, 1, g, s));
  }
  RouteParams r = {};
  r.T = c.T; r.E = c.E; r.k = c.k; r.gate_mode = c.gate_mode;
  r.n_groups = c.n_groups; r.topk_groups = c.topk_groups; r.route_scale = c.route_scale;
  r.logits = logits; r.bias = bias; r.topk_idx = idx; r.topk_gate = gate;
  r.n_partials = n_part;
  r.partial_stride = (long long)c.T * c.E;
  r.chunk_counts = at<int>(ws, L.ccount);
  MOE_CUDA(launch_router_topk(r, s));
  const int nch = ceil_div(c.T, kChunk);
  MOE_CUDA(launch_chunk_scan(at<int>(ws, L.ccount), nch, c.E, at<int>(ws, L.cbase), counts, s));
  MOE_CUDA(launch_offsets(counts, c.E, offsets, s));
  return MOE_OK;
}

// Tile bases to add to the chunk bases enqueue_route left in the workspace
// (the fused router's chunk bases count from the start of their tile), or
// null when the chunk bases are already global.
const int* route_tile_base(const moe_config& c, void* ws) {
  return fused_route(c) ? at<int>(ws, layout_of(c).tbase) : nullptr;
}

// Token-tile width of the expert GEMMs. Weight bytes dominate: every token
// tile of an expert streams that expert's weights once more, so tiles are as
// wide as the MMA allows (256) unless experts see only a handful of tokens
// (decode), where a narrow tile leaves shared memory for deeper pipelining.
// Slots in flight per CTA: four, so each SM keeps 4 x 32 KB of weight rows
// (plus the slots' token rows) on the way. A read stream of TMA copies on
// B200 peaks there (about 7.3 TB/s from HBM with 128 KB in flight per SM)
// and loses throughput with more (6.6 TB/s at 192 KB); in the GEMMs four
// measured faster than three, five or eight on the decode, DeepSeek-V3 and
// Mixtral shapes alike.
int inflight_for() { return 4; }

// Whether moe_forward's gate/up GEMM gathers token rows from x (cp.async,
// single-CTA tiles) instead of reading a packed copy: bf16, token tiles
// under 128 (no CTA pairs), 16-byte aligned rows, x under 4 GB. Measured on
// B200: as fast as the packed rows at these shapes, and the permute's copy
// is saved; on CTA pairs the packed copy wins.
int expert_tile_n(const moe_config& c);
bool gather_rows_in_gemm(const moe_config& c, const void* x) {
  return c.dtype == MOE_DTYPE_BF16 && expert_tile_n(c) < 128 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0 &&
         c.d % 8 == 0 && (long long)c.T * c.d * 2 <= 0xffffffffll;
}

int expert_tile_n(const moe_config& c) {
  const double m = (double)c.T * c.k / c.E;
  int bn = (int)ceil(4.0 * m + 16.0);
  bn = (bn + 31) / 32 * 32;
  return bn < 32 ? 32 : (bn > 256 ? 256 : bn);
}

// SwiGLU inner activation of every segment: h = SiLU(x W1^T) * (x W3^T).
moe_status enqueue_gate_up(const moe_config& c, const void* x_perm, const int* offsets, const void* w1,
                           const void* w3, const void* x_sh, const void* ws1, const void* ws3, void* h,
                           void* h_s, uint32_t* err, cudaStream_t s, const int* gather_rows = nullptr,
                           const void* gather_src = nullptr, void* const* pre = nullptr) {
  const bool shared = c.f_shared > 0;
  const int rows = c.T * c.k;
  if (c.dtype == MOE_DTYPE_BF16) {
    UmmaGemmParams g = {};
    g.mode = kUmmaSwiGLU;
    g.n_routed = c.E;
    g.offsets = offsets;
    g.m_rows = c.f;
    g.K = c.d;
    g.shared_rows = shared ? c.T : 0;
    g.m_rows_s = c.f_shared;
    g.K_s = c.d;
    g.bn_max = expert_tile_n(c);
    g.max_inflight = inflight_for();
    g.a = w1; g.a3 = w3; g.b = x_perm;
    g.a_rows_total = (long long)c.E * c.f;
    g.b_rows_total = rows;
    g.a_s = ws1; g.a3_s = ws3; g.b_s = x_sh;
    g.out = h; g.out_ld = c.f;
    g.out_s = h_s; g.out_s_ld = c.f_shared;
    g.err = err;
    g.timeout_ns = kDefaultTimeoutNs;
    g.max_routed_rows = rows;
    if (gather_rows) {          // token rows read straight from x through the packed-row map
      g.b_gather = gather_rows;
      g.b_gather_src = gather_src;
      g.b_gather_rows = c.T;
    }
    if (pre) {
      g.mode = kUmmaSwiGLUSave;
      g.pre_a = pre[0]; g.pre_b = pre[1]; g.pre_a_s = pre[2]; g.pre_b_s = pre[3];
    }
    MOE_CUDA(launch_umma_gemm(g, device_sm_count(), s));
  } else {
    SimtGemmParams g = {};
    g.dual = 1;
    g.n_routed = c.E;
    g.offsets = offsets;
    g.a = x_perm; g.b1 = w1; g.b3 = w3; g.out = h;
    g.N = c.f; g.K = c.d;
    g.shared_rows = shared ? c.T : 0;
    g.a_s = x_sh; g.b1_s = ws1; g.b3_s = ws3; g.out_s = h_s;
    g.N_s = c.f_shared; g.K_s = c.d;
    g.max_rows = rows;
    g.err = err;
    if (pre) { g.pre_a = pre[0]; g.pre_b = pre[1]; g.pre_a_s = pre[2]; g.pre_b_s = pre[3]; }
    MOE_CUDA(launch_simt_gemm(c.dtype, 0, g, s));
  }
  return MOE_OK;
}

// Down projection of every segment: y = h W2^T.
moe_status enqueue_down(const moe_config& c, const void* h, const int* offsets, const void* w2,
                        const void* h_s, const void* ws2, void* y_perm, void* y_sh, uint32_t* err,
                        cudaStream_t s) {
  const bool shared = c.f_shared > 0;
  const int rows = c.T * c.k;
  if (c.dtype == MOE_DTYPE_BF16) {
    UmmaGemmParams q = {};
    q.mode = kUmmaDown;
    q.n_routed = c.E;
    q.offsets = offsets;
    q.m_rows = c.d;
    q.K = c.f;
    q.shared_rows = shared ? c.T : 0;
    q.m_rows_s = c.d;
    q.K_s = c.f_shared;
    q.bn_max = expert_tile_n(c);
    q.max_inflight = inflight_for();
    q.a = w2; q.b = h;
    q.a_rows_total = (long long)c.E * c.d;
    q.b_rows_total = rows;
    q.a_s = ws2; q.b_s = h_s;
    q.out = y_perm; q.out_ld = c.d;
    q.out_s = y_sh; q.out_s_ld = c.d;
    q.err = err;
    q.timeout_ns = kDefaultTimeoutNs;
    q.max_routed_rows = rows;
    MOE_CUDA(launch_umma_gemm(q, device_sm_count(), s));
  } else {
    SimtGemmParams q = {};
    q.dual = 0;
    q.n_routed = c.E;
    q.offsets = offsets;
    q.a = h; q.b1 = w2; q.out = y_perm;
    q.N = c.d; q.K = c.f;
    q.shared_rows = shared ? c.T : 0;
    q.a_s = h_s; q.b1_s = ws2; q.out_s = y_sh;
    q.N_s = c.d; q.K_s = c.f_shared;
    q.max_rows = rows;
    q.err = err;
    MOE_CUDA(launch_simt_gemm(c.dtype, 0, q, s));
  }
  return MOE_OK;
}

moe_status enqueue_experts(const moe_config& c, const void* x_perm, const int* offsets, const void* w1,
                           const void* w3, const void* w2, const void* x_sh, const void* ws1,
                           const void* ws3, const void* ws2, void* y_perm, void* y_sh, void* ws,
                           cudaStream_t s, void* const* pre = nullptr, const int* gather_rows = nullptr,
                           const void* gather_src = nullptr) {
  const Layout L = layout_of(c);
  void* h = at<char>(ws, L.h);
  void* h_s = at<char>(ws, L.h_s);
  uint32_t* err = at<uint32_t>(ws, L.err);
  MOE_TRY(enqueue_gate_up(c, x_perm, offsets, w1, w3, x_sh, ws1, ws3, h, h_s, err, s, gather_rows, gather_src,
                          pre));
  return enqueue_down(c, h, offsets, w2, h_s, ws2, y_perm, y_sh, err, s);
}

// Generic experts: h = GELU(x W1^T + b1), y = h W2^T + b2 (routed segments only).
moe_status enqueue_gelu_experts(const moe_config& c, const void* x_perm, const int* offsets,
                                const void* w1, const float* b1, const void* w2, const float* b2,
                                void* y_perm, void* ws, cudaStream_t s) {
  const Layout L = layout_of(c);
  void* h = at<char>(ws, L.h);
  uint32_t* err = at<uint32_t>(ws, L.err);
  const int rows = c.T * c.k;
  if (c.dtype == MOE_DTYPE_BF16) {
    UmmaGemmParams g = {};
    g.mode = kUmmaBiasAct;
    g.n_routed = c.E;
    g.offsets = offsets;
    g.m_rows = c.f;
    g.K = c.d;
    g.bn_max = expert_tile_n(c);
    g.max_inflight = inflight_for();
    g.a = w1; g.a3 = w1; g.b = x_perm;
    g.a_rows_total = (long long)c.E * c.f;
    g.b_rows_total = rows;
    g.out = h; g.out_ld = c.f;
    g.err = err;
    g.timeout_ns = kDefaultTimeoutNs;
    g.max_routed_rows = rows;
    g.row_bias = b1;
    g.act = kActGelu;
    MOE_CUDA(launch_umma_gemm(g, device_sm_count(), s));
    UmmaGemmParams q = g;
    q.m_rows = c.d;
    q.K = c.f;
    q.a = w2; q.a3 = w2; q.b = h;
    q.a_rows_total = (long long)c.E * c.d;
    q.out = y_perm; q.out_ld = c.d;
    q.row_bias = b2;
    q.act = kActNone;
    MOE_CUDA(launch_umma_gemm(q, device_sm_count(), s));
  } else {
    SimtGemmParams g = {};
    g.dual = 0;
    g.n_routed = c.E;
    g.offsets = offsets;
    g.a = x_perm; g.b1 = w1; g.out = h;
    g.N = c.f; g.K = c.d;
    g.max_rows = rows;
    g.err = err;
    g.bias1 = b1;
    g.act = kActGelu;
    MOE_CUDA(launch_simt_gemm(c.dtype, 0, g, s));
    SimtGemmParams q = g;
    q.a = h; q.b1 = w2; q.out = y_perm;
    q.N = c.d; q.K = c.f;
    q.bias1 = b2;
    q.act = kActNone;
    MOE_CUDA(launch_simt_gemm(c.dtype, 0, q, s));
  }
  return MOE_OK;
}

// ---------------------------------------------------------------- backward
// Regions of the backward workspace that follow the forward layout.
struct BwdLayout {
  size_t a, b, a_s, b_s, dyp, dhp, dhs, hg, hgs, dadb, dadbs, dgate, dl, dlb, dxp, dxs, dxr, total;
  int f_pad, fs_pad, e_pad;
};

BwdLayout bwd_layout_of(const moe_config& c) {
  BwdLayout B;
  size_t off = layout_of(c).total;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + kAlign - 1) / kAlign * kAlign;
    return o;
  };
  const size_t es = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
  const size_t T = (size_t)c.T, k = (size_t)c.k, E = (size_t)c.E, d = (size_t)c.d, f = (size_t)c.f;
  const size_t fs = (size_t)c.f_shared, rows = T * k;
  B.f_pad = (c.f + 63) / 64 * 64;
  B.fs_pad = (c.f_shared + 63) / 64 * 64;
  B.a = take(rows * f * es);
  B.b = take(rows * f * es);
  B.a_s = take(T * fs * es);
  B.b_s = take(T * fs * es);
  B.dyp = take(rows * d * es);
  B.dhp = take(rows * f * 4);
  B.dhs = take(T * fs * 4);
  B.hg = take(rows * f * es);
  B.hgs = take(T * fs * es);
  B.dadb = take(rows * 2 * (size_t)B.f_pad * es);
  B.dadbs = take(T * 2 * (size_t)B.fs_pad * es);
  B.dgate = take(rows * 4);
  B.dl = take(T * E * 4);
  B.e_pad = (c.E + 7) / 8 * 8;
  B.dlb = take(T * (size_t)B.e_pad * 2);
  B.dxp = take(rows * d * 4);
  B.dxs = take(fs > 0 ? T * d * 4 : 0);
  B.dxr = take(T * d * 4);
  B.total = off;
  return B;
}

// C = A B^T through the strided SIMT kernel (see grad_gemm.cu for the
// addressing); a helper to keep the call sites short.
GradGemmParams gg(const moe_config& c, int seg_mode, int n_seg, const int* offsets) {
  GradGemmParams g = {};
  g.dtype = c.dtype;
  g.seg_mode = seg_mode;
  g.n_seg = n_seg;
  g.offsets = offsets;
  return g;
}

// Input-gradient GEMM on the tensor cores: out[r][m] = sum_c W[c][m] g[r][c]
// per routed segment (W stacked [E * c_rows][m_rows]) and, when sh_rows > 0,
// the dense segment (W_s [c_rows_s][m_rows_s]); fp32 output. w2nd / ws2nd
// take over after k_split / k_split_s 64-wide blocks of the contraction.
struct DgradArgs {
  const int* offsets; int n_routed;
  const void* g; int K; const void* w; const void* w2nd; int c_rows; int m_rows; int k_split; float* out;
  int sh_rows; const void* g_s; int K_s; const void* w_s; const void* ws2nd; int c_rows_s; int m_rows_s;
  int k_split_s; float* out_s;
  int bn;
};
moe_status enqueue_dgrad(const DgradArgs& a, int rows, uint32_t* err, cudaStream_t s) {
  UmmaGemmParams g = {};
  g.mode = kUmmaDgrad;
  g.out_f32 = 1;
  g.n_routed = a.n_routed;
  g.offsets = a.offsets;
  g.m_rows = a.m_rows;
  g.K = a.K;
  g.shared_rows = a.sh_rows;
  g.m_rows_s = a.m_rows_s;
  g.K_s = a.K_s;
  g.bn_max = a.bn;
  g.max_inflight = inflight_for();
  g.a = a.w; g.a3 = a.w2nd; g.b = a.g;
  g.a_rows_total = (long long)a.n_routed * a.c_rows;
  g.b_rows_total = rows;
  g.a_s = a.w_s; g.a3_s = a.ws2nd; g.b_s = a.g_s;
  g.a_k_rows = a.c_rows; g.a_k_rows_s = a.c_rows_s;
  g.k_split = a.k_split; g.k_split_s = a.k_split_s;
  g.out = a.out; g.out_ld = a.m_rows;
  g.out_s = a.out_s; g.out_s_ld = a.m_rows_s;
  g.err = err;
  g.timeout_ns = kDefaultTimeoutNs;
  g.max_routed_rows = rows;
  MOE_CUDA(launch_umma_gemm(g, device_sm_count(), s));
  return MOE_OK;
}

int dense_tile_n(int T) {
  const int bn = (T + 15) / 16 * 16;
  return bn > 256 ? 256 : (bn < 16 ? 16 : bn);
}

// Pre-activations a = W1 u and b = W3 u of every routed row and shared row.
moe_status enqueue_preact(const moe_config& c, const void* x_perm, const int* offsets, const void* x,
                          const void* w1, const void* w3, const void* ws1, const void* ws3, void* a,
                          void* b, void* a_s, void* b_s, uint32_t* err, cudaStream_t s) {
  const bool shared = c.f_shared > 0;
  const int rows = c.T * c.k;
  for (int which = 0; which < 2; ++which) {
    const void* w = which ? w3 : w1;
    const void* wsh = which ? ws3 : ws1;
    void* out = which ? b : a;
    void* out_s = which ? b_s : a_s;
    if (c.dtype == MOE_DTYPE_BF16) {
      UmmaGemmParams g = {};
      g.mode = kUmmaBiasAct;
      g.n_routed = c.E;
      g.offsets = offsets;
      g.m_rows = c.f;
      g.K = c.d;
      g.shared_rows = shared ? c.T : 0;
      g.m_rows_s = c.f_shared;
      g.K_s = c.d;
      g.bn_max = expert_tile_n(c);
      g.max_inflight = inflight_for();
      g.a = w; g.a3 = w; g.b = x_perm;
      g.a_rows_total = (long long)c.E * c.f;
      g.b_rows_total = rows;
      g.a_s = wsh; g.a3_s = wsh; g.b_s = x;
      g.out = out; g.out_ld = c.f;
      g.out_s = out_s; g.out_s_ld = c.f_shared;
      g.err = err;
      g.timeout_ns = kDefaultTimeoutNs;
      g.max_routed_rows = rows;
      g.act = kActNone;
      MOE_CUDA(launch_umma_gemm(g, device_sm_count(), s));
    } else {
      GradGemmParams g = gg(c, kSegRows, c.E, offsets);
      g.N = c.f; g.K = c.d; g.max_rows = rows;
      g.a = x_perm; g.a_si = c.d; g.a_sk = 1;
      g.b = w; g.b_seg = (long long)c.f * c.d; g.b_sj = c.d; g.b_sk = 1;
      g.c = out; g.c_si = c.f;
      MOE_CUDA(launch_grad_gemm(g, s));
      if (shared) {
        GradGemmParams q = gg(c, kSegRows, 1, nullptr);
        q.N = c.f_shared; q.K = c.d; q.max_rows = c.T;
        q.a = x; q.a_si = c.d; q.a_sk = 1;
        q.b = wsh; q.b_sj = c.d; q.b_sk = 1;
        q.c = out_s; q.c_si = c.f_shared;
        MOE_CUDA(launch_grad_gemm(q, s));
      }
    }
  }
  return MOE_OK;
}

// recompute: route, pack x and compute the pre-activations here; otherwise
// they are the state a training forward left in this workspace.
moe_status enqueue_backward(const moe_config& c, const void* x, const void* w_router, const float* bias,
                            const void* w1, const void* w3, const void* w2, const void* ws1,
                            const void* ws3, const void* ws2, const void* dy, void* dx, void* dw_router,
                            void* dw1, void* dw3, void* dw2, void* dws1, void* dws3, void* dws2,
                            void* ws, cudaStream_t s, bool recompute = true) {
  const Layout L = layout_of(c);
  const BwdLayout Bw = bwd_layout_of(c);
  const bool shared = c.f_shared > 0;
  const int rows = c.T * c.k;
  const long long d = c.d, f = c.f, fs = c.f_shared, E = c.E;
  const int fp = Bw.f_pad, fsp = Bw.fs_pad;
  uint32_t* err = at<uint32_t>(ws, L.err);
  int* idx = at<int>(ws, L.idx);
  float* gate = at<float>(ws, L.gate);
  int* offsets = at<int>(ws, L.offsets);
  int* inv_row = at<int>(ws, L.inv_row);
  int* perm_src = at<int>(ws, L.perm_src);
  char* x_perm = at<char>(ws, L.x_perm);
  char* dyp = at<char>(ws, Bw.dyp);
  const int nsm = device_sm_count();
  // Forward state: routing, packed x, pre-activations; then packed dy.
  if (recompute) {
    MOE_TRY(enqueue_route(c, x, w_router, bias, idx, gate, at<int>(ws, L.counts), offsets, ws, s));
    MOE_CUDA(launch_permute(c.dtype, x, idx, offsets, at<int>(ws, L.cbase), route_tile_base(c, ws), c.T, c.d,
                            c.E, c.k, x_perm, perm_src, inv_row, nsm, s, true, err));
    MOE_TRY(enqueue_preact(c, x_perm, offsets, x, w1, w3, ws1, ws3, at<char>(ws, Bw.a), at<char>(ws, Bw.b),
                           at<char>(ws, Bw.a_s), at<char>(ws, Bw.b_s), err, s));
  }
  MOE_CUDA(launch_permute(c.dtype, dy, idx, offsets, at<int>(ws, L.cbase), route_tile_base(c, ws), c.T, c.d,
                          c.E, c.k, dyp, perm_src, inv_row, nsm, s, true, err));
  // dh' = W2^T dy per packed row (gate not applied), and the shared expert's.
  const bool tc = c.dtype == MOE_DTYPE_BF16;
  constexpr int kNoSplit = 1 << 30;
  if (tc) {
    DgradArgs a = {};
    a.offsets = offsets; a.n_routed = c.E;
    a.g = dyp; a.K = c.d; a.w = w2; a.w2nd = nullptr; a.c_rows = c.d; a.m_rows = c.f; a.k_split = kNoSplit;
    a.out = at<float>(ws, Bw.dhp);
    if (shared) {
      a.sh_rows = c.T; a.g_s = dy; a.K_s = c.d; a.w_s = ws2; a.ws2nd = nullptr; a.c_rows_s = c.d;
      a.m_rows_s = c.f_shared; a.k_split_s = kNoSplit; a.out_s = at<float>(ws, Bw.dhs);
    }
    a.bn = expert_tile_n(c);
    MOE_TRY(enqueue_dgrad(a, rows, err, s));
  } else {
    GradGemmParams g = gg(c, kSegRows, c.E, offsets);
    g.c_f32 = 1;
    g.N = c.f; g.K = c.d; g.max_rows = rows;
    g.a = dyp; g.a_si = d; g.a_sk = 1;
    g.b = w2; g.b_seg = d * f; g.b_sj = 1; g.b_sk = f;
    g.c = at<char>(ws, Bw.dhp); g.c_si = f;
    MOE_CUDA(launch_grad_gemm(g, s));
    if (shared) {
      GradGemmParams q = gg(c, kSegRows, 1, nullptr);
      q.c_f32 = 1;
      q.N = c.f_shared; q.K = c.d; q.max_rows = c.T;
      q.a = dy; q.a_si = d; q.a_sk = 1;
      q.b = ws2; q.b_sj = 1; q.b_sk = fs;
      q.c = at<char>(ws, Bw.dhs); q.c_si = fs;
      MOE_CUDA(launch_grad_gemm(q, s));
    }
  }
  // SwiGLU backward: dgate, hg = g h, [da | db].
  float* dgate = at<float>(ws, Bw.dgate);
  MOE_CUDA(launch_swiglu_bwd(c.dtype, at<char>(ws, Bw.a), at<char>(ws, Bw.b), at<float>(ws, Bw.dhp), inv_row,
                             gate, dgate, at<char>(ws, Bw.hg), at<char>(ws, Bw.dadb), rows, c.f, fp, s));
  if (shared)
    MOE_CUDA(launch_swiglu_bwd(c.dtype, at<char>(ws, Bw.a_s), at<char>(ws, Bw.b_s), at<float>(ws, Bw.dhs),
                               nullptr, nullptr, nullptr, at<char>(ws, Bw.hgs), at<char>(ws, Bw.dadbs), c.T,
                               c.f_shared, fsp, s));
  // Gates -> router logits.
  float* dl = at<float>(ws, Bw.dl);
  MOE_CUDA(launch_gate_bwd(at<float>(ws, L.logits), idx, gate, dgate, dl, tc ? at<char>(ws, Bw.dlb) : nullptr,
                           Bw.e_pad, c.T, c.E, c.k, c.gate_mode, c.route_scale, s));
  // Input gradients: dx_perm = da W1 + db W3 per packed row; shared; router.
  const size_t es = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
  if (tc) {
    DgradArgs a = {};
    a.offsets = offsets; a.n_routed = c.E;
    a.g = at<char>(ws, Bw.dadb); a.K = 2 * fp; a.w = w1; a.w2nd = w3; a.c_rows = c.f; a.m_rows = c.d;
    a.k_split = fp / 64; a.out = at<float>(ws, Bw.dxp);
    if (shared) {
      a.sh_rows = c.T; a.g_s = at<char>(ws, Bw.dadbs); a.K_s = 2 * fsp; a.w_s = ws1; a.ws2nd = ws3;
      a.c_rows_s = c.f_shared; a.m_rows_s = c.d; a.k_split_s = fsp / 64; a.out_s = at<float>(ws, Bw.dxs);
    }
    a.bn = expert_tile_n(c);
    MOE_TRY(enqueue_dgrad(a, rows, err, s));
    DgradArgs r = {};
    r.n_routed = 0;
    r.sh_rows = c.T; r.g_s = at<char>(ws, Bw.dlb); r.K_s = Bw.e_pad; r.w_s = w_router; r.ws2nd = nullptr;
    r.c_rows_s = c.E; r.m_rows_s = c.d; r.k_split_s = kNoSplit; r.out_s = at<float>(ws, Bw.dxr);
    r.bn = dense_tile_n(c.T);
    MOE_TRY(enqueue_dgrad(r, c.T, err, s));
  }
  for (int which = 0; which < 2 && !tc; ++which) {
    GradGemmParams g = gg(c, kSegRows, c.E, offsets);
    g.c_f32 = 1;
    g.accumulate = which;
    g.N = c.d; g.K = c.f; g.max_rows = rows;
    g.a = at<char>(ws, Bw.dadb) + (size_t)which * fp * es; g.a_si = 2LL * fp; g.a_sk = 1;
    g.b = which ? w3 : w1; g.b_seg = f * d; g.b_sj = 1; g.b_sk = d;
    g.c = at<char>(ws, Bw.dxp); g.c_si = d;
    MOE_CUDA(launch_grad_gemm(g, s));
    if (shared) {
      GradGemmParams q = gg(c, kSegRows, 1, nullptr);
      q.c_f32 = 1;
      q.accumulate = which;
      q.N = c.d; q.K = c.f_shared; q.max_rows = c.T;
      q.a = at<char>(ws, Bw.dadbs) + (size_t)which * fsp * es; q.a_si = 2LL * fsp; q.a_sk = 1;
      q.b = which ? ws3 : ws1; q.b_sj = 1; q.b_sk = d;
      q.c = at<char>(ws, Bw.dxs); q.c_si = d;
      MOE_CUDA(launch_grad_gemm(q, s));
    }
  }
  if (!tc) {
    GradGemmParams q = gg(c, kSegRows, 1, nullptr);
    q.a_f32 = 1; q.c_f32 = 1;
    q.N = c.d; q.K = c.E; q.max_rows = c.T;
    q.a = dl; q.a_si = E; q.a_sk = 1;
    q.b = w_router; q.b_sj = 1; q.b_sk = d;
    q.c = at<char>(ws, Bw.dxr); q.c_si = d;
    MOE_CUDA(launch_grad_gemm(q, s));
  }
  MOE_CUDA(launch_unpermute_sum(c.dtype, at<float>(ws, Bw.dxp), inv_row, shared ? at<float>(ws, Bw.dxs) : nullptr,
                                at<float>(ws, Bw.dxr), dx, c.T, c.d, c.k, s));
  // Weight gradients, each a sum over the segment's tokens.
  if (tc) {
    const int nsm2 = device_sm_count();
    auto wg = [&](int n_seg, const int* offs, int k_total, int M, int N, const void* P, long long ldP,
                  long long p_rows, const void* Q, long long ldQ, long long q_rows, void* out) -> moe_status {
      WgradParams w = {};
      w.n_seg = n_seg; w.offsets = offs; w.k_total = k_total; w.M = M; w.N = N;
      w.P = P; w.ldP = ldP; w.p_rows = p_rows; w.Q = Q; w.ldQ = ldQ; w.q_rows = q_rows; w.out = out;
      w.err = err; w.timeout_ns = kDefaultTimeoutNs;
      MOE_CUDA(launch_wgrad(w, nsm2, s));
      return MOE_OK;
    };
    char* dadb = at<char>(ws, Bw.dadb);
    MOE_TRY(wg(c.E, offsets, 0, c.f, c.d, dadb, 2LL * fp, rows, x_perm, d, rows, dw1));
    MOE_TRY(wg(c.E, offsets, 0, c.f, c.d, dadb + (size_t)fp * es, 2LL * fp, rows, x_perm, d, rows, dw3));
    MOE_TRY(wg(c.E, offsets, 0, c.d, c.f, dyp, d, rows, at<char>(ws, Bw.hg), f, rows, dw2));
    if (shared) {
      char* dadbs = at<char>(ws, Bw.dadbs);
      MOE_TRY(wg(1, nullptr, c.T, c.f_shared, c.d, dadbs, 2LL * fsp, c.T, x, d, c.T, dws1));
      MOE_TRY(wg(1, nullptr, c.T, c.f_shared, c.d, dadbs + (size_t)fsp * es, 2LL * fsp, c.T, x, d, c.T, dws3));
      MOE_TRY(wg(1, nullptr, c.T, c.d, c.f_shared, dy, d, c.T, at<char>(ws, Bw.hgs), fs, c.T, dws2));
    }
    MOE_TRY(wg(1, nullptr, c.T, c.E, c.d, at<char>(ws, Bw.dlb), Bw.e_pad, c.T, x, d, c.T, dw_router));
    return MOE_OK;
  }
  for (int which = 0; which < 2; ++which) {         // dW1, dW3 [E][f][d]
    GradGemmParams g = gg(c, kSegK, c.E, offsets);
    g.M = c.f; g.N = c.d;
    g.a = at<char>(ws, Bw.dadb) + (size_t)which * fp * es; g.a_si = 1; g.a_sk = 2LL * fp;
    g.b = x_perm; g.b_sj = 1; g.b_sk = d;
    g.c = which ? dw3 : dw1; g.c_seg = f * d; g.c_si = d;
    MOE_CUDA(launch_grad_gemm(g, s));
    if (shared) {
      GradGemmParams q = gg(c, kSegK, 1, nullptr);
      q.M = c.f_shared; q.N = c.d; q.K = c.T;
      q.a = at<char>(ws, Bw.dadbs) + (size_t)which * fsp * es; q.a_si = 1; q.a_sk = 2LL * fsp;
      q.b = x; q.b_sj = 1; q.b_sk = d;
      q.c = which ? dws3 : dws1; q.c_si = d;
      MOE_CUDA(launch_grad_gemm(q, s));
    }
  }
  {                                                  // dW2 [E][d][f]
    GradGemmParams g = gg(c, kSegK, c.E, offsets);
    g.M = c.d; g.N = c.f;
    g.a = dyp; g.a_si = 1; g.a_sk = d;
    g.b = at<char>(ws, Bw.hg); g.b_sj = 1; g.b_sk = f;
    g.c = dw2; g.c_seg = d * f; g.c_si = f;
    MOE_CUDA(launch_grad_gemm(g, s));
    if (shared) {
      GradGemmParams q = gg(c, kSegK, 1, nullptr);
      q.M = c.d; q.N = c.f_shared; q.K = c.T;
      q.a = dy; q.a_si = 1; q.a_sk = d;
      q.b = at<char>(ws, Bw.hgs); q.b_sj = 1; q.b_sk = fs;
      q.c = dws2; q.c_si = fs;
      MOE_CUDA(launch_grad_gemm(q, s));
    }
  }
  {                                                  // dW_router [E][d]
    GradGemmParams q = gg(c, kSegK, 1, nullptr);
    q.a_f32 = 1;
    q.M = c.E; q.N = c.d; q.K = c.T;
    q.a = dl; q.a_si = 1; q.a_sk = E;
    q.b = x; q.b_sj = 1; q.b_sk = d;
    q.c = dw_router; q.c_si = d;
    MOE_CUDA(launch_grad_gemm(q, s));
  }
  return MOE_OK;
}

moe_status clear_error_word(void* ws, cudaStream_t s) {
  MOE_CUDA(cudaMemsetAsync(at<char>(ws, 0), 0, kAlign, s));
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_check_config(const moe_config* cfg) { return check_config(cfg); }

size_t moe_workspace_size(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return layout_of(*cfg).total;
}

moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router, const float* bias,
                     int32_t* topk_idx, float* topk_gate, int32_t* expert_counts,
                     int32_t* expert_offsets, void* workspace, size_t ws_bytes, void* stream) {
  TraceRange trace("moe_route");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(need4(expert_counts));
  MOE_TRY(need4(expert_offsets));
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (c.T == 0) {
    MOE_CUDA(cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * c.E, s));
    MOE_CUDA(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (c.E + 1), s));
    return MOE_OK;
  }
  MOE_TRY(need(x));
  MOE_TRY(need(w_router));
  MOE_TRY(need4(topk_idx));
  MOE_TRY(need4(topk_gate));
  if (bias) MOE_TRY(need4(bias));
  MOE_TRY(clear_error_word(workspace, s));
  return enqueue_route(c, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets,
                       workspace, s);
}

moe_status moe_route_maps(const moe_config* cfg, const void* x, const void* w_router, const float* bias,
                          int32_t* topk_idx, float* topk_gate, int32_t* expert_counts,
                          int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_row, void* workspace,
                          size_t ws_bytes, void* stream) {
  TraceRange trace("moe_route_maps");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  if (!route_writes_maps(c)) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(need4(expert_counts));
  MOE_TRY(need4(expert_offsets));
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (c.T == 0) {
    MOE_CUDA(cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * c.E, s));
    MOE_CUDA(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (c.E + 1), s));
    return MOE_OK;
  }
  MOE_TRY(need(x));
  MOE_TRY(need(w_router));
  MOE_TRY(need4(topk_idx));
  MOE_TRY(need4(topk_gate));
  MOE_TRY(need4(perm_src));
  MOE_TRY(need4(inv_row));
  if (bias) MOE_TRY(need4(bias));
  MOE_TRY(clear_error_word(workspace, s));
  return enqueue_route(c, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets,
                       workspace, s, inv_row, perm_src);
}

int moe_route_maps_supported(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return -1;
  return route_writes_maps(*cfg) ? 1 : 0;
}

moe_status moe_permute(const moe_config* cfg, const void* x, const int32_t* topk_idx,
                       const int32_t* expert_offsets, void* x_perm, int32_t* perm_src,
                       int32_t* inv_row, void* workspace, size_t ws_bytes, void* stream) {
  TraceRange trace("moe_permute");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need4(topk_idx));
  MOE_TRY(need4(expert_offsets));
  MOE_TRY(need4(perm_src));
  MOE_TRY(need4(inv_row));
  const bool copy = x_perm != nullptr;     // NULL: write the maps only
  if (copy) {
    MOE_TRY(need(x));
    MOE_TRY(need(x_perm));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_TRY(clear_error_word(workspace, s));
  const Layout L = layout_of(c);
  const int nch = ceil_div(c.T, kChunk);
  MOE_CUDA(launch_chunk_counts(topk_idx, c.T, c.k, c.E, at<int>(workspace, L.ccount), s));
  MOE_CUDA(launch_chunk_scan(at<int>(workspace, L.ccount), nch, c.E, at<int>(workspace, L.cbase),
                             at<int>(workspace, L.counts), s));
  MOE_CUDA(launch_permute(c.dtype, x, topk_idx, expert_offsets, at<int>(workspace, L.cbase), nullptr, c.T,
                          c.d, c.E, c.k, x_perm, perm_src, inv_row, device_sm_count(), s, copy,
                          at<uint32_t>(workspace, L.err)));
  return MOE_OK;
}

moe_status moe_expert_swiglu(const moe_config* cfg, const void* x_perm, const int32_t* expert_offsets,
                             const void* w1, const void* w3, const void* w2, const void* x_shared,
                             const void* ws1, const void* ws3, const void* ws2, void* y_perm,
                             void* y_shared, void* workspace, size_t ws_bytes, void* stream) {
  TraceRange trace("moe_expert_swiglu");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need(x_perm));
  MOE_TRY(need4(expert_offsets));
  MOE_TRY(need(w1));
  MOE_TRY(need(w3));
  MOE_TRY(need(w2));
  MOE_TRY(need(y_perm));
  if (c.f_shared > 0) {
    MOE_TRY(need(x_shared));
    MOE_TRY(need(ws1));
    MOE_TRY(need(ws3));
    MOE_TRY(need(ws2));
    MOE_TRY(need(y_shared));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_TRY(clear_error_word(workspace, s));
  return enqueue_experts(c, x_perm, expert_offsets, w1, w3, w2, x_shared, ws1, ws3, ws2, y_perm,
                         y_shared, workspace, s);
}

moe_status moe_expert_gate_up(const moe_config* cfg, const void* x_perm, const int32_t* expert_offsets,
                              const void* w1, const void* w3, const void* x_shared, const void* ws1,
                              const void* ws3, void* h, void* h_shared, void* workspace,
                              size_t ws_bytes, void* stream) {
  TraceRange trace("moe_expert_gate_up");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need(x_perm));
  MOE_TRY(need4(expert_offsets));
  MOE_TRY(need(w1));
  MOE_TRY(need(w3));
  MOE_TRY(need(h));
  if (c.f_shared > 0) {
    MOE_TRY(need(x_shared));
    MOE_TRY(need(ws1));
    MOE_TRY(need(ws3));
    MOE_TRY(need(h_shared));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_TRY(clear_error_word(workspace, s));
  return enqueue_gate_up(c, x_perm, expert_offsets, w1, w3, x_shared, ws1, ws3, h, h_shared,
                         at<uint32_t>(workspace, 0), s);
}

moe_status moe_expert_gate_up_gather(const moe_config* cfg, const void* x, const int32_t* perm_src,
                                     const int32_t* expert_offsets, const void* w1, const void* w3,
                                     const void* ws1, const void* ws3, void* h, void* h_shared,
                                     void* workspace, size_t ws_bytes, void* stream) {
  TraceRange trace("moe_expert_gate_up_gather");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  if (c.dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  // cp.async reads 16-byte pieces of the rows at 32-bit offsets
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || c.d % 8 || (long long)c.T * c.d * 2 > 0xffffffffll)
    return MOE_ERR_UNSUPPORTED;
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need(x));
  MOE_TRY(need4(perm_src));
  MOE_TRY(need4(expert_offsets));
  MOE_TRY(need(w1));
  MOE_TRY(need(w3));
  MOE_TRY(need(h));
  if (c.f_shared > 0) {
    MOE_TRY(need(ws1));
    MOE_TRY(need(ws3));
    MOE_TRY(need(h_shared));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_TRY(clear_error_word(workspace, s));
  const Layout L = layout_of(c);
  // The routed B tensor map still needs a valid source; the workspace's packed
  // region is never read on this path.
  return enqueue_gate_up(c, at<char>(workspace, L.x_perm), expert_offsets, w1, w3,
                         c.f_shared > 0 ? x : nullptr, ws1, ws3, h, h_shared,
                         at<uint32_t>(workspace, 0), s, perm_src, x);
}

moe_status moe_expert_down(const moe_config* cfg, const void* h, const int32_t* expert_offsets,
                           const void* w2, const void* h_shared, const void* ws2, void* y_perm,
                           void* y_shared, void* workspace, size_t ws_bytes, void* stream) {
  TraceRange trace("moe_expert_down");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need(h));
  MOE_TRY(need4(expert_offsets));
  MOE_TRY(need(w2));
  MOE_TRY(need(y_perm));
  if (c.f_shared > 0) {
    MOE_TRY(need(h_shared));
    MOE_TRY(need(ws2));
    MOE_TRY(need(y_shared));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_TRY(clear_error_word(workspace, s));
  return enqueue_down(c, h, expert_offsets, w2, h_shared, ws2, y_perm, y_shared,
                      at<uint32_t>(workspace, 0), s);
}

moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* inv_row,
                       const float* topk_gate, const void* y_shared, void* y, void* stream) {
  TraceRange trace("moe_combine");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need(y_perm));
  MOE_TRY(need4(inv_row));
  MOE_TRY(need4(topk_gate));
  MOE_TRY(need(y));
  if (y_shared) MOE_TRY(need(y_shared));
  MOE_CUDA(launch_combine(c.dtype, y_perm, inv_row, topk_gate, y_shared, y, c.T, c.d, c.k,
                          device_sm_count(), static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router, const float* bias,
                       const void* w1, const void* w3, const void* w2, const void* ws1,
                       const void* ws3, const void* ws2, void* y, void* workspace, size_t ws_bytes,
                       void* stream) {
  TraceRange trace("moe_forward");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need(x));
  MOE_TRY(need(w_router));
  if (bias) MOE_TRY(need4(bias));
  MOE_TRY(need(w1));
  MOE_TRY(need(w3));
  MOE_TRY(need(w2));
  MOE_TRY(need(y));
  if (c.f_shared > 0) {
    MOE_TRY(need(ws1));
    MOE_TRY(need(ws3));
    MOE_TRY(need(ws2));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Layout L = layout_of(c);
  void* ws = workspace;
  MOE_TRY(clear_error_word(ws, s));
  int* idx = at<int>(ws, L.idx);
  float* gate = at<float>(ws, L.gate);
  int* offsets = at<int>(ws, L.offsets);
  // Token rows for the gate/up GEMM. With single-CTA token tiles (few
  // tokens per expert, e.g. decode) the GEMM gathers each expert's rows from
  // x through perm_src, and only the row maps are needed: the router writes
  // them itself when the batch is one tile, else the permute writes them.
  // With CTA pairs the packed copy plus TMA rows is faster, so the permute
  // copies the rows.
  const bool gather = gather_rows_in_gemm(c, x);
  const bool maps_in_route = gather && route_writes_maps(c);
  {
    TraceRange stage("moe_forward.route");
    MOE_TRY(enqueue_route(c, x, w_router, bias, idx, gate, at<int>(ws, L.counts), offsets, ws, s,
                          maps_in_route ? at<int>(ws, L.inv_row) : nullptr,
                          maps_in_route ? at<int>(ws, L.perm_src) : nullptr));
  }
  if (!maps_in_route) {
    TraceRange stage("moe_forward.permute");
    MOE_CUDA(launch_permute(c.dtype, x, idx, offsets, at<int>(ws, L.cbase), route_tile_base(c, ws), c.T, c.d,
                            c.E, c.k, at<char>(ws, L.x_perm), at<int>(ws, L.perm_src), at<int>(ws, L.inv_row),
                            device_sm_count(), s, !gather, at<uint32_t>(ws, L.err)));
  }
  const bool shared = c.f_shared > 0;
  void* y_s = shared ? at<char>(ws, L.y_s) : nullptr;
  {
    TraceRange stage("moe_forward.experts");
    // On the gather path the routed B tensor map still needs a valid
    // source: the workspace's packed region, never read.
    MOE_TRY(enqueue_experts(c, at<char>(ws, L.x_perm), offsets, w1, w3, w2, shared ? x : nullptr, ws1,
                            ws3, ws2, at<char>(ws, L.y_perm), y_s, ws, s, nullptr,
                            gather ? at<int>(ws, L.perm_src) : nullptr, gather ? x : nullptr));
  }
  TraceRange stage("moe_forward.combine");
  MOE_CUDA(launch_combine(c.dtype, at<char>(ws, L.y_perm), at<int>(ws, L.inv_row), gate, y_s, y, c.T,
                          c.d, c.k, device_sm_count(), s));
  return MOE_OK;
}

int moe_forward_gathers_rows(const moe_config* cfg, const void* x) {
  if (check_config(cfg) != MOE_OK) return -1;
  return gather_rows_in_gemm(*cfg, x) ? 1 : 0;
}

moe_status moe_expert_gelu(const moe_config* cfg, const void* x_perm, const int32_t* expert_offsets,
                           const void* w1, const float* b1, const void* w2, const float* b2,
                           void* y_perm, void* workspace, size_t ws_bytes, void* stream) {
  TraceRange trace("moe_expert_gelu");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  if (c.f_shared > 0) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need(x_perm));
  MOE_TRY(need4(expert_offsets));
  MOE_TRY(need(w1));
  MOE_TRY(need(w2));
  MOE_TRY(need(y_perm));
  if (b1) MOE_TRY(need4(b1));
  if (b2) MOE_TRY(need4(b2));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_TRY(clear_error_word(workspace, s));
  return enqueue_gelu_experts(c, x_perm, expert_offsets, w1, b1, w2, b2, y_perm, workspace, s);
}

moe_status moe_forward_gelu(const moe_config* cfg, const void* x, const void* w_router,
                            const float* bias, const void* w1, const float* b1, const void* w2,
                            const float* b2, void* y, void* workspace, size_t ws_bytes,
                            void* stream) {
  TraceRange trace("moe_forward_gelu");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  if (c.f_shared > 0) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(check_ws(c, workspace, ws_bytes));
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need(x));
  MOE_TRY(need(w_router));
  if (bias) MOE_TRY(need4(bias));
  MOE_TRY(need(w1));
  MOE_TRY(need(w2));
  MOE_TRY(need(y));
  if (b1) MOE_TRY(need4(b1));
  if (b2) MOE_TRY(need4(b2));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Layout L = layout_of(c);
  void* ws = workspace;
  MOE_TRY(clear_error_word(ws, s));
  int* idx = at<int>(ws, L.idx);
  float* gate = at<float>(ws, L.gate);
  int* offsets = at<int>(ws, L.offsets);
  MOE_TRY(enqueue_route(c, x, w_router, bias, idx, gate, at<int>(ws, L.counts), offsets, ws, s));
  MOE_CUDA(launch_permute(c.dtype, x, idx, offsets, at<int>(ws, L.cbase), route_tile_base(c, ws), c.T, c.d,
                          c.E, c.k, at<char>(ws, L.x_perm), at<int>(ws, L.perm_src), at<int>(ws, L.inv_row),
                          device_sm_count(), s, true, at<uint32_t>(ws, L.err)));
  MOE_TRY(enqueue_gelu_experts(c, at<char>(ws, L.x_perm), offsets, w1, b1, w2, b2,
                               at<char>(ws, L.y_perm), ws, s));
  MOE_CUDA(launch_combine(c.dtype, at<char>(ws, L.y_perm), at<int>(ws, L.inv_row), gate, nullptr, y,
                          c.T, c.d, c.k, device_sm_count(), s));
  return MOE_OK;
}

size_t moe_backward_workspace_size(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return bwd_layout_of(*cfg).total;
}

}  // extern "C"

namespace moe {
namespace {
moe_status backward_entry(const moe_config* cfg, const void* x, const void* w_router, const float* bias,
                          const void* w1, const void* w3, const void* w2, const void* ws1, const void* ws3,
                          const void* ws2, const void* dy, void* dx, void* dw_router, void* dw1, void* dw3,
                          void* dw2, void* dws1, void* dws3, void* dws2, void* workspace, size_t ws_bytes,
                          void* stream, bool recompute) {
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(need(workspace));
  if (ws_bytes < bwd_layout_of(c).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (c.T == 0) {
    // No tokens: every weight gradient is zero.
    MOE_TRY(need(dw_router)); MOE_TRY(need(dw1)); MOE_TRY(need(dw3)); MOE_TRY(need(dw2));
    const size_t es = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
    MOE_CUDA(cudaMemsetAsync(dw_router, 0, (size_t)c.E * c.d * es, s));
    MOE_CUDA(cudaMemsetAsync(dw1, 0, (size_t)c.E * c.f * c.d * es, s));
    MOE_CUDA(cudaMemsetAsync(dw3, 0, (size_t)c.E * c.f * c.d * es, s));
    MOE_CUDA(cudaMemsetAsync(dw2, 0, (size_t)c.E * c.d * c.f * es, s));
    if (c.f_shared > 0) {
      MOE_TRY(need(dws1)); MOE_TRY(need(dws3)); MOE_TRY(need(dws2));
      MOE_CUDA(cudaMemsetAsync(dws1, 0, (size_t)c.f_shared * c.d * es, s));
      MOE_CUDA(cudaMemsetAsync(dws3, 0, (size_t)c.f_shared * c.d * es, s));
      MOE_CUDA(cudaMemsetAsync(dws2, 0, (size_t)c.d * c.f_shared * es, s));
    }
    return MOE_OK;
  }
  MOE_TRY(need(x));
  MOE_TRY(need(w_router));
  if (bias) MOE_TRY(need4(bias));
  MOE_TRY(need(w1)); MOE_TRY(need(w3)); MOE_TRY(need(w2));
  MOE_TRY(need(dy)); MOE_TRY(need(dx));
  MOE_TRY(need(dw_router)); MOE_TRY(need(dw1)); MOE_TRY(need(dw3)); MOE_TRY(need(dw2));
  if (c.f_shared > 0) {
    MOE_TRY(need(ws1)); MOE_TRY(need(ws3)); MOE_TRY(need(ws2));
    MOE_TRY(need(dws1)); MOE_TRY(need(dws3)); MOE_TRY(need(dws2));
  }
  MOE_TRY(clear_error_word(workspace, s));
  return enqueue_backward(c, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, dy, dx, dw_router, dw1, dw3, dw2,
                          dws1, dws3, dws2, workspace, s, recompute);
}
}  // namespace
}  // namespace moe

extern "C" {

moe_status moe_backward(const moe_config* cfg, const void* x, const void* w_router, const float* bias,
                        const void* w1, const void* w3, const void* w2, const void* ws1, const void* ws3,
                        const void* ws2, const void* dy, void* dx, void* dw_router, void* dw1, void* dw3,
                        void* dw2, void* dws1, void* dws3, void* dws2, void* workspace, size_t ws_bytes,
                        void* stream) {
  TraceRange trace("moe_backward");
  return backward_entry(cfg, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, dy, dx, dw_router, dw1, dw3, dw2,
                        dws1, dws3, dws2, workspace, ws_bytes, stream, true);
}

moe_status moe_backward_saved(const moe_config* cfg, const void* x, const void* w_router, const void* w1,
                              const void* w3, const void* w2, const void* ws1, const void* ws3,
                              const void* ws2, const void* dy, void* dx, void* dw_router, void* dw1,
                              void* dw3, void* dw2, void* dws1, void* dws3, void* dws2, void* workspace,
                              size_t ws_bytes, void* stream) {
  TraceRange trace("moe_backward_saved");
  return backward_entry(cfg, x, w_router, nullptr, w1, w3, w2, ws1, ws3, ws2, dy, dx, dw_router, dw1, dw3,
                        dw2, dws1, dws3, dws2, workspace, ws_bytes, stream, false);
}

moe_status moe_forward_train(const moe_config* cfg, const void* x, const void* w_router, const float* bias,
                             const void* w1, const void* w3, const void* w2, const void* ws1,
                             const void* ws3, const void* ws2, void* y, void* workspace, size_t ws_bytes,
                             void* stream) {
  TraceRange trace("moe_forward_train");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(need(workspace));
  if (ws_bytes < bwd_layout_of(c).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (c.T == 0) return MOE_OK;
  MOE_TRY(need(x));
  MOE_TRY(need(w_router));
  if (bias) MOE_TRY(need4(bias));
  MOE_TRY(need(w1));
  MOE_TRY(need(w3));
  MOE_TRY(need(w2));
  MOE_TRY(need(y));
  if (c.f_shared > 0) {
    MOE_TRY(need(ws1));
    MOE_TRY(need(ws3));
    MOE_TRY(need(ws2));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Layout L = layout_of(c);
  const BwdLayout Bw = bwd_layout_of(c);
  void* ws = workspace;
  MOE_TRY(clear_error_word(ws, s));
  int* idx = at<int>(ws, L.idx);
  float* gate = at<float>(ws, L.gate);
  int* offsets = at<int>(ws, L.offsets);
  MOE_TRY(enqueue_route(c, x, w_router, bias, idx, gate, at<int>(ws, L.counts), offsets, ws, s));
  MOE_CUDA(launch_permute(c.dtype, x, idx, offsets, at<int>(ws, L.cbase), route_tile_base(c, ws), c.T, c.d,
                          c.E, c.k, at<char>(ws, L.x_perm), at<int>(ws, L.perm_src), at<int>(ws, L.inv_row),
                          device_sm_count(), s, true, at<uint32_t>(ws, L.err)));
  const bool shared = c.f_shared > 0;
  void* y_s = shared ? at<char>(ws, L.y_s) : nullptr;
  void* pre[4] = {at<char>(ws, Bw.a), at<char>(ws, Bw.b), shared ? at<char>(ws, Bw.a_s) : nullptr,
                  shared ? at<char>(ws, Bw.b_s) : nullptr};
  MOE_TRY(enqueue_experts(c, at<char>(ws, L.x_perm), offsets, w1, w3, w2, shared ? x : nullptr, ws1, ws3, ws2,
                          at<char>(ws, L.y_perm), y_s, ws, s, pre));
  MOE_CUDA(launch_combine(c.dtype, at<char>(ws, L.y_perm), at<int>(ws, L.inv_row), gate, y_s, y, c.T, c.d, c.k,
                          device_sm_count(), s));
  return MOE_OK;
}

moe_status moe_balance_update(const moe_config* cfg, const int32_t* expert_counts, float* bias,
                              float gamma, float* entropy, void* stream) {
  TraceRange trace("moe_balance_update");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(need4(expert_counts));
  if (!bias && !entropy) return MOE_ERR_INVALID_ARG;
  if (bias) MOE_TRY(need4(bias));
  if (entropy) MOE_TRY(need4(entropy));
  if (bias && (!(gamma >= 0.0f) || !isfinite(gamma))) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(launch_balance_update(expert_counts, c.E, (long long)c.T * c.k, gamma, bias, entropy,
                                 static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_get_device_error(void* workspace, void* stream) {
  MOE_TRY(need(workspace));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return MOE_ERR_CUDA;
  if (word & kErrTimeoutWait) return MOE_ERR_TIMEOUT;
  if (word & kErrBadIndex) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(void* workspace, size_t ws_bytes, int64_t timeout_ns,
                                     void* stream) {
  MOE_TRY(need(workspace));
  if (ws_bytes < kAlign || timeout_ns <= 0) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_TRY(clear_error_word(workspace, s));
  MOE_CUDA(launch_wait_timeout_selftest(static_cast<uint32_t*>(workspace), timeout_ns, s));
  return MOE_OK;
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_MISALIGNED: return "pointer or row stride not 16-byte aligned";
    case MOE_ERR_UNSUPPORTED: return "configuration beyond this build's limits";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "a bounded device wait timed out";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Router without a caller workspace.
//
// Some callers cannot allocate device memory at the point where they route:
// code running inside another framework's allocator-free region, a plugin
// host that hands out only the tensors it owns, or a call made while the
// process must not grow its device footprint. For them, moe_route_noalloc
// keeps the router's scratch (logits, per-chunk histograms and bases, and the
// error word) in one fixed array that lives in this library's device image.
// The array is created with the library's module on every GPU that loads it
// and stays until the process exits. Its host-side name is only a stand-in
// for the symbol, never a device address: the address is looked up once per
// device with cudaGetSymbolAddress while that device is current.
// ---------------------------------------------------------------------------
#include <atomic>

namespace {
constexpr size_t kRouteScratchBytes = size_t(24) << 20;   // 24 MiB per device
constexpr int kMaxDevices = 64;
std::atomic<void*> g_route_scratch_addr[kMaxDevices];
}  // namespace

static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

namespace {
// Device address of the scratch array on the current device (set-up on the
// first call per device; needs no allocation).
moe_status route_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  void* p = g_route_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_route_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return MOE_OK;
}
}  // namespace

extern "C" moe_status moe_route_noalloc(const moe_config* cfg, const void* x, const void* w_router,
                                        const float* bias, int32_t* topk_idx, float* topk_gate,
                                        int32_t* expert_counts, int32_t* expert_offsets,
                                        void* stream) {
  TraceRange trace("moe_route_noalloc");
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(need4(expert_counts));
  MOE_TRY(need4(expert_offsets));
  // The router uses the leading regions of the workspace layout (error word,
  // logits, chunk histograms, chunk bases); they must fit in the array.
  if (layout_of(c).idx > kRouteScratchBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (c.T == 0) {
    MOE_CUDA(cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * c.E, s));
    MOE_CUDA(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (c.E + 1), s));
    return MOE_OK;
  }
  MOE_TRY(need(x));
  MOE_TRY(need(w_router));
  MOE_TRY(need4(topk_idx));
  MOE_TRY(need4(topk_gate));
  if (bias) MOE_TRY(need4(bias));
  void* scratch = nullptr;
  MOE_TRY(route_scratch(&scratch));
  MOE_TRY(clear_error_word(scratch, s));   // the only region that must start at zero
  return enqueue_route(c, x, w_router, bias, topk_idx, topk_gate, expert_counts, expert_offsets,
                       scratch, s);
}

// The fixed array's error word (its first bytes) on the current device:
// synchronise the stream, read the word, clear it.
extern "C" moe_status moe_route_noalloc_device_error(void* stream) {
  void* scratch = nullptr;
  MOE_TRY(route_scratch(&scratch));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  MOE_CUDA(cudaStreamSynchronize(s));
  MOE_CUDA(cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, s));
  MOE_CUDA(cudaMemsetAsync(scratch, 0, sizeof(word), s));
  MOE_CUDA(cudaStreamSynchronize(s));
  if (word & kErrTimeoutWait) return MOE_ERR_TIMEOUT;
  return (word & kErrBadIndex) ? MOE_ERR_INVALID_ARG : MOE_OK;
}
