// Router: logits s = W_g . x, softmax or sigmoid affinity, token-choice top-k with the
// lowest-index tie-break, merge weights, importance partials; expert-choice top-c select.
//
// "Top-k 路由（Top-k Routing）" (compassingai), "門控函式的數學形式" Steps 1-2;
// "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife), section 4;
// "别只比较 Top-k" (ailearn moe-comparison), Score / Select / Merge steps (sigmoid affinity and
// a selection-only bias for DeepSeek-V3);
// "Top-k 路由" Token-Choice vs Expert-Choice table (each expert takes its top-C tokens).
//
// Layout: one warp owns TPW consecutive tokens; its lanes split the hidden dimension in
// 16-byte chunks (coalesced row reads of x), accumulate fp32 dot products against 8 experts
// at a time (W_g rows come through L1), and reduce across lanes with shuffles.  The warp then
// holds the token's E logits in shared memory and does the per-token affinity, a k-round warp
// arg-max for top-k, and the merge weights.  Everything stays on chip except x, W_g and the
// outputs.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kTPW = 4;          // tokens per warp
constexpr int kWarps = 8;        // warps per block
constexpr int kEB = 8;           // experts per accumulation block
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

// 16 bytes of x or W_g as fp32 values.
template <bool BF16> struct Chunk;
template <> struct Chunk<true> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const void* base, int64_t elem, float* out) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <> struct Chunk<false> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const void* base, int64_t elem, float* out) {
    float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem));
    out[0] = f.x; out[1] = f.y; out[2] = f.z; out[3] = f.w;
  }
};

struct RouterArgs {
  const void* x; const void* Wg; const float* bias;
  int32_t* ids; float* gates; float* logits; float* probsT; float* partials;
  int T, D, E, k, score, gate, expert_choice;
};

// logits of the warp's TPW tokens for all experts -> s_log[TPW][E]
template <bool BF16>
__device__ __forceinline__ void warp_logits(const RouterArgs& a, int t0, float* s_log, int lane) {
  using C = Chunk<BF16>;
  const int nvec = a.D / C::N;
  for (int e0 = 0; e0 < a.E; e0 += kEB) {
    float acc[kTPW][kEB];
#pragma unroll
    for (int t = 0; t < kTPW; ++t)
#pragma unroll
      for (int e = 0; e < kEB; ++e) acc[t][e] = 0.f;
    const int ne = min(kEB, a.E - e0);
    for (int v = lane; v < nvec; v += 32) {
      float xv[kTPW][C::N];
#pragma unroll
      for (int t = 0; t < kTPW; ++t) {
        if (t0 + t < a.T) {
          C::load(a.x, (int64_t)(t0 + t) * a.D + (int64_t)v * C::N, xv[t]);
        } else {
#pragma unroll
          for (int i = 0; i < C::N; ++i) xv[t][i] = 0.f;
        }
      }
#pragma unroll
      for (int e = 0; e < kEB; ++e) {
        if (e < ne) {
          float wv[C::N];
          C::load(a.Wg, (int64_t)(e0 + e) * a.D + (int64_t)v * C::N, wv);
#pragma unroll
          for (int t = 0; t < kTPW; ++t)
#pragma unroll
            for (int i = 0; i < C::N; ++i) acc[t][e] = fmaf(xv[t][i], wv[i], acc[t][e]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kTPW; ++t)
#pragma unroll
      for (int e = 0; e < kEB; ++e) {
        float v = warp_sum(acc[t][e]);
        if (lane == 0 && e < ne) s_log[t * a.E + e0 + e] = v;
      }
  }
  __syncwarp();
}

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32)
router_kernel(RouterArgs a) {
  extern __shared__ float s_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kWarps + warp;
  const int t0 = gw * kTPW;
  float* s_log = s_all + warp * kTPW * a.E;

  warp_logits<BF16>(a, t0, s_log, lane);

  const int E = a.E;
  float imp[kMaxEPL];
#pragma unroll
  for (int i = 0; i < kMaxEPL; ++i) imp[i] = 0.f;

  for (int t = 0; t < kTPW; ++t) {
    const int tok = t0 + t;
    if (tok >= a.T) break;
    float s[kMaxEPL], p[kMaxEPL], key[kMaxEPL];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kMaxEPL; ++i) {
      const int e = lane + 32 * i;
      s[i] = (e < E) ? s_log[t * E + e] : -INFINITY;
      m = fmaxf(m, s[i]);
    }
    if (a.logits) {
#pragma unroll
      for (int i = 0; i < kMaxEPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) a.logits[(int64_t)tok * E + e] = s[i];
      }
    }
    float sel_w[kMaxEPL];   // weight used in the merge (softmax p or sigmoid affinity)
    if (a.score == MOE_SCORE_SOFTMAX) {
      m = warp_max(m);
      float z = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxEPL; ++i) {
        const int e = lane + 32 * i;
        p[i] = (e < E) ? expf(s[i] - m) : 0.f;
        z += p[i];
      }
      z = warp_sum(z);
      const float inv = 1.0f / z;
#pragma unroll
      for (int i = 0; i < kMaxEPL; ++i) {
        p[i] = p[i] * inv;
        key[i] = s[i];             // softmax is monotone in the logit within a row
        sel_w[i] = p[i];
        imp[i] += p[i];
      }
    } else {
      float asum = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxEPL; ++i) {
        const int e = lane + 32 * i;
        const float af = (e < E) ? 1.0f / (1.0f + expf(-s[i])) : 0.f;
        sel_w[i] = af;
        key[i] = (e < E) ? af + (a.bias ? a.bias[e] : 0.f) : -INFINITY;
        asum += af;
      }
      asum = warp_sum(asum);
      const float inv = 1.0f / asum;
#pragma unroll
      for (int i = 0; i < kMaxEPL; ++i) { p[i] = sel_w[i] * inv; imp[i] += p[i]; }
    }

    if (a.expert_choice) {
      // merge weights are the softmax probabilities; selection happens per expert later
#pragma unroll
      for (int i = 0; i < kMaxEPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
          a.gates[(int64_t)tok * E + e] = p[i];
          a.probsT[(int64_t)e * a.T + tok] = p[i];
        }
      }
      continue;
    }

    // top-k: k rounds of a warp arg-max over (key desc, expert id asc)
    bool taken[kMaxEPL];
#pragma unroll
    for (int i = 0; i < kMaxEPL; ++i) taken[i] = false;
    int my_id = -1;        // lane j < k keeps slot j
    float my_w = 0.f;
    float wsum = 0.f;
    for (int j = 0; j < a.k; ++j) {
      float bk = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < kMaxEPL; ++i) {
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
      for (int i = 0; i < kMaxEPL; ++i)
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

  if (a.partials) {
#pragma unroll
    for (int i = 0; i < kMaxEPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) a.partials[(int64_t)gw * E + e] = imp[i];
    }
  }
}

// importance[e] = (sum over partial rows, fixed order) / T.  One block per expert.
__global__ void importance_reduce_kernel(const float* partials, int n, int E, int T, float* out) {
  const int e = blockIdx.x;
  float s = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += partials[(int64_t)i * E + e];
  __shared__ float red[32];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) out[e] = v / (float)T;
  }
}

// ---- expert choice: per expert, the c largest probabilities (ties -> lower token id) ----

// Block-wide exclusive scan of one int per thread; returns the total in *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  __syncthreads();
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < nw) ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < nw) s_warp[lane] = w;     // inclusive warp totals
  }
  __syncthreads();
  const int before = (warp > 0) ? s_warp[warp - 1] : 0;
  *total = s_warp[nw - 1];
  return before + inc - v;
}

__global__ void __launch_bounds__(1024)
ec_select_kernel(const float* probsT, int T, int c, int32_t* picked) {
  const int e = blockIdx.x;
  const uint32_t* keys = reinterpret_cast<const uint32_t*>(probsT + (int64_t)e * T);
  __shared__ int hist[256];
  __shared__ int s_digit, s_need;
  __shared__ int s_warp[32];
  uint32_t prefix = 0, mask = 0;
  int need = c;
  // Radix select of the c-th largest key, 8 bits per pass, most significant first.
  // Probabilities are >= 0, so their IEEE bit patterns order like the values.
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      const uint32_t kk = keys[t];
      if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & 0xffu], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int cum = 0, d = 255;
      for (; d > 0; --d) {
        if (cum + hist[d] >= need) break;
        cum += hist[d];
      }
      s_digit = d;
      s_need = need - cum;
    }
    __syncthreads();
    prefix |= (uint32_t)s_digit << shift;
    mask |= 0xffu << shift;
    need = s_need;
    __syncthreads();
  }
  // Ordered compaction: every key above the threshold, plus the first `need` keys equal to
  // it in ascending token order.
  int out_base = 0, eq_seen = 0;
  for (int base = 0; base < T; base += blockDim.x) {
    const int t = base + threadIdx.x;
    const uint32_t kk = (t < T) ? keys[t] : 0u;
    const int gt = (t < T && kk > prefix) ? 1 : 0;
    const int eq = (t < T && kk == prefix) ? 1 : 0;
    int eq_total;
    const int eq_rank = block_exclusive_scan(eq, s_warp, &eq_total);
    const int take = gt | (eq && (eq_seen + eq_rank < need));
    int take_total;
    const int pos = block_exclusive_scan(take, s_warp, &take_total);
    if (take && out_base + pos < c) picked[(int64_t)e * c + out_base + pos] = t;
    out_base += take_total;
    eq_seen += eq_total;
    __syncthreads();
  }
}

}  // namespace

int router_partials(const moe_desc_t& d) {
  const int blocks = (d.T + kWarps * kTPW - 1) / (kWarps * kTPW);
  return blocks * kWarps;
}

static cudaError_t launch_router(const RouterArgs& a, bool bf16, int T, cudaStream_t s) {
  const int blocks = (T + kWarps * kTPW - 1) / (kWarps * kTPW);
  if (blocks == 0) return cudaSuccess;
  const size_t smem = (size_t)kWarps * kTPW * a.E * sizeof(float);
  if (bf16) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(router_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    router_kernel<true><<<blocks, kWarps * 32, smem, s>>>(a);
  } else {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(router_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    router_kernel<false><<<blocks, kWarps * 32, smem, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_router_token_choice(const moe_desc_t& d, const void* x, const void* Wg,
                                       const float* bias, int32_t* ids, float* gates,
                                       float* logits, float* imp_partials, int n_partials,
                                       cudaStream_t s) {
  (void)n_partials;
  RouterArgs a{x, Wg, bias, ids, gates, logits, nullptr, imp_partials,
               d.T, d.D, d.E, d.k, d.score, d.gate, 0};
  return launch_router(a, d.dtype == MOE_BF16, d.T, s);
}

cudaError_t launch_router_expert_choice(const moe_desc_t& d, const void* x, const void* Wg,
                                        float* probs, float* probsT, float* logits,
                                        float* imp_partials, int n_partials, cudaStream_t s) {
  (void)n_partials;
  RouterArgs a{x, Wg, nullptr, nullptr, probs, logits, probsT, imp_partials,
               d.T, d.D, d.E, 0, MOE_SCORE_SOFTMAX, MOE_GATE_RAW, 1};
  return launch_router(a, d.dtype == MOE_BF16, d.T, s);
}

cudaError_t launch_ec_select(const moe_desc_t& d, const float* probsT, int32_t* picked,
                             cudaStream_t s) {
  ec_select_kernel<<<d.E, 1024, 0, s>>>(probsT, d.T, d.c, picked);
  return cudaGetLastError();
}

cudaError_t launch_importance_reduce(const float* partials, int n_partials, int E, int T,
                                     float* importance, cudaStream_t s) {
  importance_reduce_kernel<<<E, 256, 0, s>>>(partials, n_partials, E, T, importance);
  return cudaGetLastError();
}

}  // namespace moe
