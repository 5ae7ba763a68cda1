// Routing of one token by one warp: biased, optionally group-limited top-k
// over the token's router logits, gates from the unbiased affinities.
//
// Sparse MoE FFN (DeepSeek-V3 note), "How it works", Routing paragraph:
//   s = sigmoid(u . e_i); top-K on s + b (after group masking: keep the
//   topk_groups best groups, group score = sum of its two largest s + b);
//   gates = unbiased selected s, renormalised over the winners, times
//   route_scale.
// MoE cheat sheet, "The router in code": the bias moves the selection only;
//   softmax over the chosen raw scores (max-subtracted), which sums to 1.
//
// Lane l holds the logits of experts l, l + 32, l + 64, ... (NPL of them).
// On return, lane j < k holds the j-th winner in `e` (winners taken largest
// b' first, equal b' to the lower id), its position `pos` among the k
// winners in ascending expert id, and its gate.
#pragma once

#include <math.h>

#include "moe_internal.cuh"

namespace moe {

__device__ __forceinline__ float route_sigmoid(float l) { return 1.0f / (1.0f + expf(-l)); }

template <int NPL>
__device__ __forceinline__ void route_token(const float (&lg)[NPL], int lane, const TopkArgs& p, int& my_e,
                                            int& pos, float& gate) {
  constexpr unsigned kFull = 0xffffffffu;
  const int E = p.E, k = p.k;
  float v[NPL];                      // biased selection score b' = s + bias
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    float b = -INFINITY;
    if (e < E) {
      const float s = (p.gate_mode == MOE_GATE_SIGMOID) ? route_sigmoid(lg[i]) : lg[i];
      b = s + (p.bias ? p.bias[e] : 0.0f);
      // A NaN score (NaN or infinite input, NaN bias) ranks below every
      // number, so it can neither win over a real score nor lose every
      // comparison and leave the arg-max without a candidate.
      if (isnan(b)) b = -INFINITY;
    }
    v[i] = b;
  }

  if (p.n_groups > 1) {
    // Group score = sum of the two largest b' of the group; lane G ends up
    // holding group G's score.
    const int gsz = E / p.n_groups;
    float my_gscore = -INFINITY;
    for (int G = 0; G < p.n_groups; ++G) {
      float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E && e / gsz == G) {
          const float x = v[i];
          if (x > m1) { m2 = m1; m1 = x; } else if (x > m2) { m2 = x; }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float o1 = __shfl_xor_sync(kFull, m1, off);
        const float o2 = __shfl_xor_sync(kFull, m2, off);
        const float hi = fmaxf(m1, o1);
        const float lo = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
        m1 = hi;
        m2 = lo;
      }
      if (lane == G) my_gscore = isnan(m1 + m2) ? -INFINITY : m1 + m2;   // +inf + -inf
    }
    // Keep the topk_groups best groups; ties go to the lower group index.
    int rank = 0;
    for (int G = 0; G < p.n_groups; ++G) {
      const float o = __shfl_sync(kFull, my_gscore, G);
      if (o > my_gscore || (o == my_gscore && G < lane)) ++rank;
    }
    const unsigned kept = __ballot_sync(kFull, lane < p.n_groups && rank < p.topk_groups);
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((kept >> (e / gsz)) & 1u)) v[i] = -INFINITY;
    }
  }

  // k rounds of a warp arg-max: largest b' first, equal b' to the lower id.
  // kNone marks "no candidate yet": the first untaken in-range expert a lane
  // sees always becomes its candidate, and a real candidate always beats
  // kNone in the reduction. Round r < k <= E leaves at least one untaken
  // expert, so every winner is an id in [0, E) whatever the scores hold.
  constexpr int kNone = 0x7fffffff;
  unsigned taken = 0u;
  my_e = -1;                         // lane j < k ends with the j-th winner
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int be = kNone;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u)) {
        if (be == kNone || v[i] > bv || (v[i] == bv && e < be)) { bv = v[i]; be = e; }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(kFull, bv, off);
      const int oe = __shfl_xor_sync(kFull, be, off);
      if (oe != kNone && (be == kNone || ov > bv || (ov == bv && oe < be))) { bv = ov; be = oe; }
    }
    if (be == kNone) be = 0;         // unreachable (k <= E); keeps the id in range regardless
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == r) my_e = be;
  }

  // Winners in ascending expert id.
  pos = 0;
  for (int j = 0; j < k; ++j) {
    const int o = __shfl_sync(kFull, my_e, j);
    if (o < my_e) ++pos;
  }
  // The unbiased logit of each winner, from the lane that holds it.
  const bool act = lane < k;
  const int src = act ? (my_e & 31) : lane, slot = act ? (my_e >> 5) : 0;
  float l = 0.0f;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const float o = __shfl_sync(kFull, lg[i], src);
    if (slot == i) l = o;
  }
  // Gates from the UNBIASED value of each winner.
  float num;
  if (p.gate_mode == MOE_GATE_SIGMOID) {
    num = act ? route_sigmoid(l) : 0.0f;
  } else {
    float m = act ? l : -INFINITY;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    num = act ? expf(l - m) : 0.0f;
  }
  float sum = num;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
  gate = p.route_scale * (num / sum);
}

}  // namespace moe
