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

// `lrow` holds the same logits in memory, [E] for this token; with more than
// 256 experts (NPL > 8) the winners' logits are read back from it rather
// than kept in registers, and it must not be null.
template <int NPL>
__device__ __forceinline__ void route_token(const float (&lg)[NPL], int lane, const TopkArgs& p, int& my_e,
                                            int& pos, float& gate, const float* lrow = nullptr) {
  constexpr unsigned kFull = 0xffffffffu;
  const int E = p.E, k = p.k;
  float v[NPL];                      // biased selection score b' = s + bias
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    float b = -INFINITY;
    if (e < E) {
      const float s = (p.gate_mode == MOE_GATE_SIGMOID) ? (NPL <= 8 ? select_sigmoid(lg[i]) : route_sigmoid(lg[i]))
                                                        : lg[i];
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
    // holding group G's score. Each held expert's group is worked out once.
    const int gsz = E / p.n_groups;
    // Group of held expert i (-1 past E): kept in registers for up to 256
    // experts, recomputed where more experts would crowd the registers.
    constexpr bool kKeepGid = NPL <= 8;
    constexpr int kGidRegs = kKeepGid ? NPL : 1;
    int gid_reg[kGidRegs];
#pragma unroll
    for (int i = 0; i < kGidRegs; ++i) {
      const int e = lane + 32 * i;
      gid_reg[i] = e < E ? e / gsz : -1;
    }
    auto gid = [&](int i) -> int {
      if (kKeepGid) return gid_reg[i];
      const int e = lane + 32 * i;
      return e < E ? e / gsz : -1;
    };
    float my_gscore = -INFINITY;
    if (NPL <= 8 && gsz == 32 && p.n_groups == NPL) {
      // Groups of 32: lane l holds exactly one expert of group G (l + 32 G),
      // so the group's two largest are the two largest lane values.
#pragma unroll
      for (int G = 0; G < NPL; ++G) {
        const uint32_t k1 = score_key(v[G]);
        const uint32_t g1 = __reduce_max_sync(kFull, k1);
        const unsigned at_max = __ballot_sync(kFull, k1 == g1);
        const uint32_t g2 = __popc(at_max) > 1 ? g1 : __reduce_max_sync(kFull, k1 == g1 ? 0u : k1);
        const float gs = key_score(g1) + key_score(g2);
        if (lane == G) my_gscore = isnan(gs) ? -INFINITY : gs;
      }
    } else
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

  if constexpr (NPL <= 8) {
    // Each lane sorts its (b', id) pairs once, best first (larger b', then
    // the lower id; ids past E last), and each of the k rounds looks at the
    // lanes' heads only: the warp's largest head score, then the lowest id
    // holding it, and the winning lane shifts its list by one. A lane's head
    // is its best untaken expert, so the winners are those of a full rescan.
    constexpr int kNoId = 0x7fffffff;
    float sv[NPL];
    int se[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      sv[i] = e < E ? v[i] : -INFINITY;
      se[i] = e < E ? e : kNoId;
    }
    auto cmp_swap = [&](int a, int b) {   // after it, position a holds the better pair
      const bool b_first = se[b] != kNoId && (se[a] == kNoId || sv[b] > sv[a] || (sv[b] == sv[a] && se[b] < se[a]));
      const float fv = b_first ? sv[b] : sv[a], gv = b_first ? sv[a] : sv[b];
      const int fe = b_first ? se[b] : se[a], ge = b_first ? se[a] : se[b];
      sv[a] = fv; sv[b] = gv; se[a] = fe; se[b] = ge;
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
      const bool has = se[0] != kNoId;
      const uint32_t key = has ? score_key(sv[0]) : 0u;
      const uint32_t best = __reduce_max_sync(kFull, key);
      int be = (int)__reduce_min_sync(kFull, (has && key == best) ? (uint32_t)se[0] : 0xffffffffu);
      if (be < 0 || be >= E) be = 0;   // unreachable (k <= E); keeps the id in range regardless
      if (has && se[0] == be) {        // this lane's head won: drop it
#pragma unroll
        for (int i = 0; i + 1 < NPL; ++i) { sv[i] = sv[i + 1]; se[i] = se[i + 1]; }
        sv[NPL - 1] = -INFINITY;
        se[NPL - 1] = kNoId;
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
  if (NPL > 8) {             // callers with more than 256 experts pass lrow
    __syncwarp();
    if (act) l = lrow[my_e];
  } else {
    const int src = act ? (my_e & 31) : lane, slot = act ? (my_e >> 5) : 0;
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
