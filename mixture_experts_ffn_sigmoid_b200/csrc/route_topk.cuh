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
// Each lane holds NPL logits. Up to 256 experts (NPL <= 8) the layout is
// blocked: lane l holds experts l*NPL .. l*NPL + NPL - 1, so lane order is
// expert order (a group of experts is a run of whole lanes, and the lowest
// lane holding a score holds its lowest id). Above 256 it is strided: lane l
// holds experts l, l + 32, l + 64, ... (route_expert gives the mapping).
// On return, lane j < k holds the j-th winner in `e` (winners taken largest
// b' first, equal b' to the lower id), its position `pos` among the k
// winners in ascending expert id, and its gate.
#pragma once

#include <math.h>

#include "moe_internal.cuh"

namespace moe {

__device__ __forceinline__ float route_sigmoid(float l) { return 1.0f / (1.0f + expf(-l)); }
// The same with the fast exponential and divide (a few ulp): used for the
// selection scores of up to 256 experts, where it is far below the fp32
// logits' own error; the gates use route_sigmoid. Large |l| saturate to 0
// and 1 as they should.
__device__ __forceinline__ float select_sigmoid(float l) { return __fdividef(1.0f, 1.0f + __expf(-l)); }

// An fp32 score as an unsigned key with the same order: a > b exactly when
// key(a) > key(b), for every non-NaN pair (-0 is folded into +0 first, since
// the two compare equal). Keys of real scores, -inf included, are > 0, so 0
// can mark "no candidate". A warp can then reduce scores with the hardware
// integer reductions (redux.sync) instead of shuffle trees.
__device__ __forceinline__ uint32_t score_key(float v) {
  const uint32_t u = __float_as_uint(v == 0.0f ? 0.0f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// The expert whose logit lane `lane` holds in slot i.
template <int NPL>
__host__ __device__ constexpr int route_expert(int lane, int i) {
  return NPL <= 8 ? lane * NPL + i : lane + 32 * i;
}

// `lrow` holds the same logits in memory, [E] for this token; the winners'
// logits are read back from it where it is given (a row in shared memory
// is one load instead of NPL shuffles). With more than 256 experts
// (NPL > 8) it must not be null.
template <int NPL>
__device__ __forceinline__ void route_token(const float (&lg)[NPL], int lane, const TopkArgs& p, int& my_e,
                                            int& pos, float& gate, const float* lrow = nullptr) {
  constexpr unsigned kFull = 0xffffffffu;
  const int E = p.E, k = p.k;
  // The lane's biases: one or two vector loads where the blocked layout
  // and the table's alignment allow, else one load per expert.
  float bias[NPL];
  constexpr int BV = NPL >= 4 ? 4 : NPL;
  if (NPL <= 8 && p.bias && (reinterpret_cast<uintptr_t>(p.bias) & (BV * 4 - 1)) == 0 &&
      (lane + 1) * NPL <= E) {
#pragma unroll
    for (int h = 0; h < NPL / BV; ++h) {
      const float* src = p.bias + lane * NPL + h * BV;
      if constexpr (BV == 4) {
        const float4 b4 = *reinterpret_cast<const float4*>(src);
        bias[4 * h] = b4.x; bias[4 * h + 1] = b4.y; bias[4 * h + 2] = b4.z; bias[4 * h + 3] = b4.w;
      } else if constexpr (BV == 2) {
        const float2 b2 = *reinterpret_cast<const float2*>(src);
        bias[2 * h] = b2.x; bias[2 * h + 1] = b2.y;
      } else {
        bias[h] = src[0];
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = route_expert<NPL>(lane, i);
      bias[i] = (p.bias && e < E) ? p.bias[e] : 0.0f;
    }
  }
  float v[NPL];                      // biased selection score b' = s + bias
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = route_expert<NPL>(lane, i);
    float b = -INFINITY;
    if (e < E) {
      const float s = (p.gate_mode == MOE_GATE_SIGMOID) ? (NPL <= 8 ? select_sigmoid(lg[i]) : route_sigmoid(lg[i]))
                                                        : lg[i];
      b = s + bias[i];
      // A NaN score (NaN or infinite input, NaN bias) ranks below every
      // number, so it can neither win over a real score nor lose every
      // comparison and leave the arg-max without a candidate.
      if (isnan(b)) b = -INFINITY;
    }
    v[i] = b;
  }

  if (p.n_groups > 1) {
    const int gsz = E / p.n_groups;
    // Blocked layout with whole lanes per group (L = gsz / NPL lanes, a power
    // of two): each lane's two largest b' of its group, merged over the
    // group's lanes by butterfly (the larger of the maxima; the larger of the
    // smaller maximum and both seconds), then each lane ranks its own group.
    const int L = gsz / NPL;
    if (NPL <= 8 && gsz % NPL == 0 && (L & (L - 1)) == 0) {
      float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const float x = v[i];
        if (x > m1) { m2 = m1; m1 = x; } else if (x > m2) { m2 = x; }
      }
      for (int off = 1; off < L; off <<= 1) {
        const float o1 = __shfl_xor_sync(kFull, m1, off);
        const float o2 = __shfl_xor_sync(kFull, m2, off);
        const float hi = fmaxf(m1, o1);
        m2 = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
        m1 = hi;
      }
      float gs = m1 + m2;
      if (isnan(gs)) gs = -INFINITY;   // +inf + -inf
      // Keep the topk_groups best groups; ties go to the lower group index.
      // Lanes past the last group hold no expert and keep nothing.
      const int my_g = lane / L;
      int rank = 0;
      for (int G = 0; G < p.n_groups; ++G) {
        const float o = __shfl_sync(kFull, gs, G * L);
        if (o > gs || (o == gs && G < my_g)) ++rank;
      }
      if (!(my_g < p.n_groups && rank < p.topk_groups)) {
#pragma unroll
        for (int i = 0; i < NPL; ++i) v[i] = -INFINITY;
      }
    } else {
    // Any other grouping: lane G ends up holding group G's score. Each held
    // expert's group is worked out once.
    // Group of held expert i (-1 past E): kept in registers for up to 256
    // experts, recomputed where more experts would crowd the registers.
    constexpr bool kKeepGid = NPL <= 8;
    constexpr int kGidRegs = kKeepGid ? NPL : 1;
    int gid_reg[kGidRegs];
#pragma unroll
    for (int i = 0; i < kGidRegs; ++i) {
      const int e = route_expert<NPL>(lane, i);
      gid_reg[i] = e < E ? e / gsz : -1;
    }
    auto gid = [&](int i) -> int {
      if (kKeepGid) return gid_reg[i];
      const int e = route_expert<NPL>(lane, i);
      return e < E ? e / gsz : -1;
    };
    float my_gscore = -INFINITY;
    for (int G = 0; G < p.n_groups; ++G) {
      // This lane's two largest b' of group G, then the group's: its largest
      // is the largest lane maximum; its second is that again when two lanes
      // hold it, else the larger of that lane's second and every other
      // lane's maximum.
      float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        if (gid(i) == G) {
          const float x = v[i];
          if (x > m1) { m2 = m1; m1 = x; } else if (x > m2) { m2 = x; }
        }
      }
      const uint32_t k1 = score_key(m1), k2 = score_key(m2);
      const uint32_t g1 = __reduce_max_sync(kFull, k1);
      const unsigned at_max = __ballot_sync(kFull, k1 == g1);
      const uint32_t g2 = __popc(at_max) > 1 ? g1 : __reduce_max_sync(kFull, k1 == g1 ? k2 : k1);
      const float gs = key_score(g1) + key_score(g2);
      if (lane == G) my_gscore = isnan(gs) ? -INFINITY : gs;   // +inf + -inf
    }
    // Keep the topk_groups best groups; ties go to the lower group index.
    int rank = 0;
    for (int G = 0; G < p.n_groups; ++G) {
      const float o = __shfl_sync(kFull, my_gscore, G);
      if (o > my_gscore || (o == my_gscore && G < lane)) ++rank;
    }
    const unsigned kept = __ballot_sync(kFull, lane < p.n_groups && rank < p.topk_groups);
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (gid(i) >= 0 && !((kept >> gid(i)) & 1u)) v[i] = -INFINITY;
    }
  }

  if constexpr (NPL <= 8) {
    // Each lane sorts its (key(b'), slot) pairs once, best first (larger
    // key, then the lower slot; experts past E have key 0 and come last),
    // and each of the k rounds looks at the lanes' heads only: the warp's
    // largest head key, held by the lowest such lane, whose head is then
    // the lowest id with that key (lanes hold ascending experts). The
    // winning lane drops its head. A lane's head is its best untaken expert,
    // so the winners are those of a full rescan.
    uint32_t kv[NPL];
    int sl[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      kv[i] = route_expert<NPL>(lane, i) < E ? score_key(v[i]) : 0u;
      sl[i] = i;
    }
    auto cmp_swap = [&](int a, int b) {   // after it, position a holds the better pair
      const bool b_first = kv[b] > kv[a] || (kv[b] == kv[a] && sl[b] < sl[a]);
      const uint32_t fk = b_first ? kv[b] : kv[a], gk = b_first ? kv[a] : kv[b];
      const int fs = b_first ? sl[b] : sl[a], gsl = b_first ? sl[a] : sl[b];
      kv[a] = fk; kv[b] = gk; sl[a] = fs; sl[b] = gsl;
    };
    if constexpr (NPL == 2) {
      cmp_swap(0, 1);
    } else if constexpr (NPL == 4) {
      cmp_swap(0, 1); cmp_swap(2, 3); cmp_swap(0, 2); cmp_swap(1, 3); cmp_swap(1, 2);
    } else if constexpr (NPL == 8) {   // Batcher's odd-even merge sort of 8
      cmp_swap(0, 1); cmp_swap(2, 3); cmp_swap(4, 5); cmp_swap(6, 7);
      cmp_swap(0, 2); cmp_swap(1, 3); cmp_swap(4, 6); cmp_swap(5, 7);
      cmp_swap(1, 2); cmp_swap(5, 6);
      cmp_swap(0, 4); cmp_swap(1, 5); cmp_swap(2, 6); cmp_swap(3, 7);
      cmp_swap(2, 4); cmp_swap(3, 5);
      cmp_swap(1, 2); cmp_swap(3, 4); cmp_swap(5, 6);
    }
    my_e = -1;
    for (int r = 0; r < k; ++r) {
      const uint32_t best = __reduce_max_sync(kFull, kv[0]);
      const int wl = __ffs(__ballot_sync(kFull, kv[0] == best)) - 1;
      int be = wl * NPL + __shfl_sync(kFull, sl[0], wl);
      if (be >= E) be = 0;             // unreachable (k <= E); keeps the id in range regardless
      if (lane == wl) {                // this lane's head won: drop it
#pragma unroll
        for (int i = 0; i + 1 < NPL; ++i) { kv[i] = kv[i + 1]; sl[i] = sl[i + 1]; }
        kv[NPL - 1] = 0u;
      }
      if (lane == r) my_e = be;
    }
  } else {
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
    // The warp's largest candidate score, then the lowest id holding it.
    const uint32_t key = be == kNone ? 0u : score_key(bv);
    const uint32_t best = __reduce_max_sync(kFull, key);
    be = (int)__reduce_min_sync(kFull, (key == best && be != kNone) ? (uint32_t)be : 0xffffffffu);
    if (be < 0 || be >= E) be = 0;   // unreachable (k <= E); keeps the id in range regardless
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == r) my_e = be;
  }
  }

  // Winners in ascending expert id.
  pos = 0;
  for (int j = 0; j < k; ++j) {
    const int o = __shfl_sync(kFull, my_e, j);
    if (o < my_e) ++pos;
  }
  // The unbiased logit of each winner, from the lane that holds it (or from
  // memory, once every lane's stores are visible to the warp).
  const bool act = lane < k;
  float l = 0.0f;
  if (NPL > 8 || lrow) {     // callers with more than 256 experts pass lrow
    __syncwarp();
    if (act) l = lrow[my_e];
  } else {
    const int src = act ? my_e / NPL : lane, slot = act ? my_e % NPL : 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const float o = __shfl_sync(kFull, lg[i], src);
      if (slot == i) l = o;
    }
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
