// Per-token routing shared by the router kernels (inline device code): affinity, merge weights,
// group-limited token-choice top-k with the lowest-index tie-break, importance and entropy
// sums.  The logits come from either router kernel; this part is the same for both.
//
// "Top-k 路由（Top-k Routing）" (compassingai), "門控函式的數學形式" Steps 2-3;
// "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife), section 4;
// "别只比较 Top-k" (ailearn moe-comparison), Score / Select / Merge steps.
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {

constexpr int kMaxEPL = 8;       // experts per lane in the selection phase (E <= 256)

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

struct RouterArgs {
  const void* x; const void* Wg; const float* bias;
  int32_t* ids; float* gates; float* logits; float* probsT; float* partials;
  int T, D, E, k, score, gate, expert_choice;
  const float* lpart;       // when set: logits are the sum of ksplit partials [ksplit][T][E]
  int ksplit;
  int n_group = 1, topk_group = 1;   // group-limited selection (n_group <= 1: none)
};

// Group-limited selection ("Mixture of Experts (MoE)" routing variant (c): groups first, then
// experts inside them; moe-comparison "Group/node limited" row).  The experts form n_group
// contiguous groups of size = E / n_group; a group scores its largest key, the token keeps its
// topk_group best groups (ties to the lower group) and every other expert's key becomes -inf.
// Lane l holds experts l + 32 i in key[i].  size is a power of two <= 32 (a group lies inside
// one register slot: a segmented shuffle max) or a multiple of 32 (a slot lies inside one
// group: a warp max); n_group <= 32, so lane g can hold group g's score.
template <int NS>
__device__ __forceinline__ void group_limit(float (&key)[NS], int E, int n_group, int topk_group,
                                            int lane) {
  if (n_group <= 1 || topk_group >= n_group) return;
  const int size = E / n_group;
  float gs = -INFINITY;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    if (32 * i >= E) break;
    float v = (lane + 32 * i < E) ? key[i] : -INFINITY;
    if (size < 32) {
      for (int o = size >> 1; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      const int src = lane * size - 32 * i;     // first lane of group `lane` in slot i
      const float w = __shfl_sync(0xffffffffu, v, src & 31);
      if (lane < n_group && src >= 0 && src < 32) gs = fmaxf(gs, w);
    } else {
      v = warp_max(v);
      if (lane == (32 * i) / size) gs = fmaxf(gs, v);
    }
  }
  uint32_t kept = 0;
  bool used = lane >= n_group;
  for (int r = 0; r < topk_group; ++r) {
    float bk = used ? -INFINITY : gs;
    int bi = used ? 0x7fffffff : lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ok > bk || (ok == bk && oi < bi)) { bk = ok; bi = oi; }
    }
    kept |= 1u << (bi & 31);
    if (lane == bi) used = true;
  }
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const int e = lane + 32 * i;
    if (e < E && !((kept >> (e / size)) & 1u)) key[i] = -INFINITY;
  }
}

// Tensor-core router fused with this selection (router_tc.cu): bf16, D % 64 == 0, E <= 256.
bool router_tc_ok(const moe_desc_t& d);
cudaError_t launch_router_tc(const moe_desc_t& d, const RouterArgs& a, int* n_partials,
                             cudaStream_t s);

// Order-preserving map of a float key to an unsigned integer (-0 counts as +0, so that equal
// keys compare equal as in float compares), for warp reductions with redux.sync.
__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t b = __float_as_uint(f + 0.0f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord_to_float(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// NT tokens in lockstep (their dependency chains interleave: the selection is latency-bound,
// one warp per token).  Lane l holds s[t][i] = logit of expert l + 32 i of token tok[t] (-inf
// past E); tokens with has[t] false are computed on and discarded.  For each token: writes its
// logits row (when a.logits), adds its probabilities to imp and its -sum p log p to ent (token
// 0 first, then token 1, ...); under expert choice writes its probabilities as
// gates[tok][e] and leaves them in p, under token choice writes its k expert ids and merge
// weights.  Top-k: k rounds of a warp arg-max over (key desc, expert id asc), each two
// redux.sync reductions: the largest key (order-preserving integers), then the smallest expert
// id holding it.
// NS = expert slots per lane (E <= 32 NS): the loops below cover only those.
template <int NS, int NT>
__device__ __forceinline__ void select_tokens(const RouterArgs& a, const int (&tok)[NT],
                                              const bool (&has)[NT], const float (&s)[NT][NS],
                                              float (&imp)[NS], float& ent,
                                              float (&p)[NT][NS], int lane) {
  const int E = a.E;
  float sel_w[NT][NS];   // weight used in the merge (softmax p or sigmoid affinity)
  float key[NT][NS];
  if (a.logits) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (!has[t]) continue;
#pragma unroll
      for (int i = 0; i < NS; ++i) {
        const int e = lane + 32 * i;
        if (e < E) a.logits[(int64_t)tok[t] * E + e] = s[t][i];
      }
    }
  }
  if (a.score == MOE_SCORE_SOFTMAX) {
    float m[NT], z[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      m[t] = -INFINITY;
#pragma unroll
      for (int i = 0; i < NS; ++i) m[t] = fmaxf(m[t], s[t][i]);
      m[t] = ord_to_float(__reduce_max_sync(0xffffffffu, ord_key(m[t])));
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      z[t] = 0.f;
#pragma unroll
      for (int i = 0; i < NS; ++i) {
        const int e = lane + 32 * i;
        p[t][i] = (e < E) ? expf(s[t][i] - m[t]) : 0.f;
        z[t] += p[t][i];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int t = 0; t < NT; ++t) z[t] += __shfl_xor_sync(0xffffffffu, z[t], o);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float inv = 1.0f / z[t];
#pragma unroll
      for (int i = 0; i < NS; ++i) {
        p[t][i] = p[t][i] * inv;
        key[t][i] = s[t][i];         // softmax is monotone in the logit within a row
        sel_w[t][i] = p[t][i];
      }
    }
  } else {
    float asum[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      asum[t] = 0.f;
#pragma unroll
      for (int i = 0; i < NS; ++i) {
        const int e = lane + 32 * i;
        const float af = (e < E) ? 1.0f / (1.0f + expf(-s[t][i])) : 0.f;
        sel_w[t][i] = af;
        key[t][i] = (e < E) ? af + (a.bias ? a.bias[e] : 0.f) : -INFINITY;
        asum[t] += af;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int t = 0; t < NT; ++t) asum[t] += __shfl_xor_sync(0xffffffffu, asum[t], o);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float inv = 1.0f / asum[t];
#pragma unroll
      for (int i = 0; i < NS; ++i) p[t][i] = sel_w[t][i] * inv;
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    if (!has[t]) continue;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      imp[i] += p[t][i];
      if (p[t][i] > 0.f) ent -= p[t][i] * logf(p[t][i]);
    }
  }

  if (a.expert_choice) {
    // merge weights are the softmax probabilities; selection happens per expert later (the
    // caller stages the transposed copy from p)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (!has[t]) continue;
#pragma unroll
      for (int i = 0; i < NS; ++i) {
        const int e = lane + 32 * i;
        if (e < E) a.gates[(int64_t)tok[t] * E + e] = p[t][i];
      }
    }
    return;
  }

#pragma unroll
  for (int t = 0; t < NT; ++t) group_limit<NS>(key[t], E, a.n_group, a.topk_group, lane);

  // top-k rounds; okey = 0 marks a slot that is taken or past E (every real key maps above 0)
  uint32_t okey[NT][NS];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < NS; ++i)   // a NaN key never wins a comparison: never a candidate
      okey[t][i] = (lane + 32 * i < E && key[t][i] == key[t][i]) ? ord_key(key[t][i]) : 0u;
  int my_id[NT];         // lane j < k keeps slot j
  float my_w[NT], wsum[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    my_id[t] = -1;
    my_w[t] = 0.f;
    wsum[t] = 0.f;
  }
  for (int j = 0; j < a.k; ++j) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      // this lane's best untaken slot: largest key, and among equal keys the first slot
      // (the lowest expert id of this lane)
      uint32_t bk = 0u;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < NS; ++i)
        if (okey[t][i] > bk) { bk = okey[t][i]; bi = lane + 32 * i; }
      const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
      const int wi = (int)__reduce_min_sync(0xffffffffu, (unsigned)(bk == wk ? bi : 0x7fffffff));
      // owner lane marks it and broadcasts its merge weight
      const int owner = wi & 31, slot = wi >> 5;
      float w = 0.f;
#pragma unroll
      for (int i = 0; i < NS; ++i)
        if (lane == owner && i == slot) { okey[t][i] = 0u; w = sel_w[t][i]; }
      w = __shfl_sync(0xffffffffu, w, owner);
      wsum[t] += w;
      if (lane == j) { my_id[t] = wi; my_w[t] = w; }
    }
  }
  if (lane < a.k) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (!has[t]) continue;
      const float g = (a.gate == MOE_GATE_RENORM) ? my_w[t] / wsum[t] : my_w[t];
      a.ids[(int64_t)tok[t] * a.k + lane] = my_id[t];
      a.gates[(int64_t)tok[t] * a.k + lane] = g;
    }
  }
}

// One token (select_tokens with NT = 1).
template <int NS>
__device__ __forceinline__ void select_token(const RouterArgs& a, int tok, const float (&s)[NS],
                                             float (&imp)[NS], float& ent, float (&p)[NS],
                                             int lane) {
  const int tk[1] = {tok};
  const bool has[1] = {true};
  float s1[1][NS], p1[1][NS];
#pragma unroll
  for (int i = 0; i < NS; ++i) s1[0][i] = s[i];
  select_tokens<NS, 1>(a, tk, has, s1, imp, ent, p1, lane);
#pragma unroll
  for (int i = 0; i < NS; ++i) p[i] = p1[0][i];
}

}  // namespace moe
