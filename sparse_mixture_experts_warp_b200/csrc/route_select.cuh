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

// One token.  Lane l holds s[i] = logit of expert l + 32 i (-inf past E).  Writes the token's
// logits row (when a.logits), adds its probabilities to imp and its -sum p log p to ent; under
// expert choice writes its probabilities as gates[tok][e] and leaves them in p, under token
// choice writes its k expert ids and merge weights.
// NS = expert slots per lane (E <= 32 NS): the loops below cover only those.
template <int NS>
__device__ __forceinline__ void select_token(const RouterArgs& a, int tok, const float (&s)[NS],
                                             float (&imp)[NS], float& ent, float (&p)[NS],
                                             int lane) {
  const int E = a.E;
  float key[NS];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < NS; ++i) m = fmaxf(m, s[i]);
  if (a.logits) {
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      const int e = lane + 32 * i;
      if (e < E) a.logits[(int64_t)tok * E + e] = s[i];
    }
  }
  float sel_w[NS];   // weight used in the merge (softmax p or sigmoid affinity)
  if (a.score == MOE_SCORE_SOFTMAX) {
    m = warp_max(m);
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      const int e = lane + 32 * i;
      p[i] = (e < E) ? expf(s[i] - m) : 0.f;
      z += p[i];
    }
    z = warp_sum(z);
    const float inv = 1.0f / z;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      p[i] = p[i] * inv;
      key[i] = s[i];             // softmax is monotone in the logit within a row
      sel_w[i] = p[i];
      imp[i] += p[i];
      if (p[i] > 0.f) ent -= p[i] * logf(p[i]);
    }
  } else {
    float asum = 0.f;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      const int e = lane + 32 * i;
      const float af = (e < E) ? 1.0f / (1.0f + expf(-s[i])) : 0.f;
      sel_w[i] = af;
      key[i] = (e < E) ? af + (a.bias ? a.bias[e] : 0.f) : -INFINITY;
      asum += af;
    }
    asum = warp_sum(asum);
    const float inv = 1.0f / asum;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      p[i] = sel_w[i] * inv;
      imp[i] += p[i];
      if (p[i] > 0.f) ent -= p[i] * logf(p[i]);
    }
  }

  if (a.expert_choice) {
    // merge weights are the softmax probabilities; selection happens per expert later (the
    // caller stages the transposed copy from p)
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      const int e = lane + 32 * i;
      if (e < E) a.gates[(int64_t)tok * E + e] = p[i];
    }
    return;
  }

  group_limit<NS>(key, E, a.n_group, a.topk_group, lane);

  // top-k: k rounds of a warp arg-max over (key desc, expert id asc)
  bool taken[NS];
#pragma unroll
  for (int i = 0; i < NS; ++i) taken[i] = false;
  int my_id = -1;        // lane j < k keeps slot j
  float my_w = 0.f;
  float wsum = 0.f;
  for (int j = 0; j < a.k; ++j) {
    float bk = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !taken[i] && (key[i] > bk || (key[i] == bk && e < bi))) { bk = key[i]; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ok > bk || (ok == bk && oi < bi)) { bk = ok; bi = oi; }
    }
    // owner lane marks it and broadcasts its merge weight
    const int owner = bi & 31, slot = bi >> 5;
    float w = 0.f;
#pragma unroll
    for (int i = 0; i < NS; ++i)
      if (lane == owner && i == slot) { taken[i] = true; w = sel_w[i]; }
    w = __shfl_sync(0xffffffffu, w, owner);
    wsum += w;
    if (lane == j) { my_id = bi; my_w = w; }
  }
  if (lane < a.k) {
    const float g = (a.gate == MOE_GATE_RENORM) ? my_w / wsum : my_w;
    a.ids[(int64_t)tok * a.k + lane] = my_id;
    a.gates[(int64_t)tok * a.k + lane] = g;
  }
}

}  // namespace moe
