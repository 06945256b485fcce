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
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "route_select.cuh"

namespace moe {
namespace {

constexpr int kTPW = 4;          // tokens per warp
constexpr int kWarps = 8;        // warps per block
constexpr int kEB = 8;           // experts per accumulation block

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

// logits of the warp's TPW tokens for all experts -> s_log[TPW][E]
template <bool BF16, int TPW>
__device__ __forceinline__ void warp_logits(const RouterArgs& a, int t0, float* s_log, int lane) {
  using C = Chunk<BF16>;
  const int nvec = a.D / C::N;
  for (int e0 = 0; e0 < a.E; e0 += kEB) {
    float acc[TPW][kEB];
#pragma unroll
    for (int t = 0; t < TPW; ++t)
#pragma unroll
      for (int e = 0; e < kEB; ++e) acc[t][e] = 0.f;
    const int ne = min(kEB, a.E - e0);
    for (int v = lane; v < nvec; v += 32) {
      float xv[TPW][C::N];
#pragma unroll
      for (int t = 0; t < TPW; ++t) {
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
          for (int t = 0; t < TPW; ++t)
#pragma unroll
            for (int i = 0; i < C::N; ++i) acc[t][e] = fmaf(xv[t][i], wv[i], acc[t][e]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TPW; ++t)
#pragma unroll
      for (int e = 0; e < kEB; ++e) {
        float v = warp_sum(acc[t][e]);
        if (lane == 0 && e < ne) s_log[t * a.E + e0 + e] = v;
      }
  }
  __syncwarp();
}

// TPW tokens per warp: 4 when the warp computes the logits itself (W_g loads shared by 4
// tokens), 1 when they come from the tensor-core product (more warps in flight).
template <bool BF16, int TPW>
__global__ void __launch_bounds__(kWarps * 32)
router_kernel(RouterArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float s_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kWarps + warp;
  const int t0 = gw * TPW;
  float* s_log = s_all + warp * TPW * a.E;

  if (a.lpart) {
    // logits from the tensor-core router product: fixed-order sum of the k-split partials
    for (int t = 0; t < TPW; ++t) {
      const int tok = t0 + t;
      if (tok >= a.T) break;
      for (int e = lane; e < a.E; e += 32) {
        float v = 0.f;
        for (int sp = 0; sp < a.ksplit; ++sp)
          v += a.lpart[((int64_t)sp * a.T + tok) * a.E + e];
        s_log[t * a.E + e] = v;
      }
    }
    __syncwarp();
  } else {
    warp_logits<BF16, TPW>(a, t0, s_log, lane);
  }

  const int E = a.E;
  float imp[kMaxEPL];
#pragma unroll
  for (int i = 0; i < kMaxEPL; ++i) imp[i] = 0.f;
  float ent = 0.f;                 // this lane's share of the tokens' -sum p log p

  for (int t = 0; t < TPW; ++t) {
    const int tok = t0 + t;
    if (tok >= a.T) break;
    float s[kMaxEPL], p[kMaxEPL];
#pragma unroll
    for (int i = 0; i < kMaxEPL; ++i) {
      const int e = lane + 32 * i;
      s[i] = (e < E) ? s_log[t * E + e] : -INFINITY;
    }
    select_token<kMaxEPL>(a, tok, s, imp, ent, p, lane);
    if (a.expert_choice) {
      // the transposed copy goes through shared memory ([token][E+1]) so that it leaves as
      // rows of the block's 32 consecutive tokens (below)
      float* s_pT = s_all + kWarps * TPW * E;
#pragma unroll
      for (int i = 0; i < kMaxEPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) s_pT[(warp * TPW + t) * (E + 1) + e] = p[i];
      }
    }
  }

  if (a.expert_choice) {
    // probsT[e][t] for the block's 32 tokens: 128-byte rows per expert (conflict-free reads:
    // the row pitch E + 1 puts the 32 tokens of one expert in 32 different banks)
    const float* s_pT = s_all + kWarps * TPW * E;
    const int tb = blockIdx.x * kWarps * TPW;
    __syncthreads();
    for (int i = threadIdx.x; i < E * kWarps * TPW; i += blockDim.x) {
      const int e = i / (kWarps * TPW), j = i % (kWarps * TPW);
      if (tb + j < a.T) a.probsT[(int64_t)e * a.T + tb + j] = s_pT[j * (E + 1) + e];
    }
  }

  if (a.partials) {
    // one partial row per block: E importance sums, then the entropy sum, over the block's
    // warps in a fixed order (s_all held the logits; every warp is past its last use of it)
    ent = warp_sum(ent);
    __syncthreads();
    float* s_part = s_all + warp * (E + 1);
#pragma unroll
    for (int i = 0; i < kMaxEPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) s_part[e] = imp[i];
    }
    if (lane == 0) s_part[E] = ent;
    __syncthreads();
    for (int c = threadIdx.x; c <= E; c += blockDim.x) {
      float sum = 0.f;
      for (int w = 0; w < kWarps; ++w) sum += s_all[w * (E + 1) + c];
      a.partials[(int64_t)blockIdx.x * (E + 1) + c] = sum;
    }
  }
}

// importance[e] = (sum over partial rows, fixed order) / T, one block per expert; block E
// reduces the entropy column into *entropy (mean over tokens).
__global__ void importance_reduce_kernel(const float* partials, int n, int E, int T,
                                         float* importance, float* entropy) {
  pdl_trigger();
  pdl_wait();
  const int e = blockIdx.x;
  float* out = (e < E) ? importance : entropy;
  if (!out) return;
  float s = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += partials[(int64_t)i * (E + 1) + e];
  __shared__ float red[32];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) out[e < E ? e : 0] = v / (float)T;
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

// One block per expert.  staged: the expert's T keys are first copied to shared memory
// (dynamic, T * 4 bytes) with 16-byte loads, so the radix passes and the compaction read them
// from there.
//
// Radix select of the c-th largest key.  Probabilities are >= 0, so their IEEE bit patterns order
// like the values.  The bits above the highest bit in which the largest and smallest key differ
// are common to all keys and are skipped; the rest is resolved 8 bits per pass, most significant
// first, each pass counting the digit of the keys that still match the prefix into one
// 256-bin histogram per warp (lanes of different warps never contend), the bins then summed in
// a fixed order.  Compaction: thread i owns the keys [i * per, (i+1) * per) in token order; one
// block scan of its (above-threshold, equal-to-threshold) counts gives every thread its output
// position and the number of equal keys before it, so the output holds all keys above the
// threshold and the first `need` equal ones, in ascending token order.  Shared memory: the
// keys (T * 4 bytes, when staged) and 32 KB of per-warp histograms.  The digit of a pass comes
// from a scan of the 256 bin totals by 256 threads.
template <bool STAGED>
__global__ void __launch_bounds__(1024)
ec_select_kernel(const float* probsT, int T, int c, int32_t* picked) {
  pdl_trigger();
  pdl_wait();
  constexpr int NW = 32;                     // warps (blockDim.x == 1024)
  const int e = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t* gkeys = reinterpret_cast<const uint32_t*>(probsT + (int64_t)e * T);
  extern __shared__ uint32_t s_keys[];
  const uint32_t* keys = gkeys;
  if (STAGED) {
    // T * 4 bytes from a row start of probsT: 16-byte aligned when T % 4 == 0 (the launcher
    // stages only then)
    const uint4* src = reinterpret_cast<const uint4*>(gkeys);
    uint4* dst = reinterpret_cast<uint4*>(s_keys);
    for (int i = threadIdx.x; i < T / 4; i += blockDim.x) dst[i] = src[i];
    __syncthreads();
    keys = s_keys;
  }
  __shared__ int hist[NW][256];
  __shared__ uint32_t s_max[NW], s_min[NW];
  __shared__ int s_digit, s_need;
  __shared__ int s_warp[32];
  // common high bits of all keys
  uint32_t kmax = 0u, kmin = 0xffffffffu;
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    const uint32_t kk = keys[t];
    kmax = kk > kmax ? kk : kmax;
    kmin = kk < kmin ? kk : kmin;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t a = __shfl_xor_sync(0xffffffffu, kmax, o);
    const uint32_t b = __shfl_xor_sync(0xffffffffu, kmin, o);
    kmax = a > kmax ? a : kmax;
    kmin = b < kmin ? b : kmin;
  }
  if (lane == 0) {
    s_max[warp] = kmax;
    s_min[warp] = kmin;
  }
  __syncthreads();
  kmax = 0u;
  kmin = 0xffffffffu;
  for (int w = 0; w < NW; ++w) {
    kmax = s_max[w] > kmax ? s_max[w] : kmax;
    kmin = s_min[w] < kmin ? s_min[w] : kmin;
  }
  const uint32_t diff = kmax ^ kmin;
  const int top = diff ? 31 - __clz(diff) : -1;      // highest differing bit
  uint32_t mask = top >= 31 ? 0u : ~((2u << top) - 1u);   // bits above `top`
  if (top < 0) mask = 0xffffffffu;
  uint32_t prefix = kmax & mask;
  int need = c;
  for (int lo = top - 7; top >= 0; lo -= 8) {
    const int shift = lo > 0 ? lo : 0;
    const int width = (lo + 7) - shift + 1;            // bits in this digit (<= 8)
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = lane; i < 256; i += 32) hist[warp][i] = 0;
    __syncwarp();
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      const uint32_t kk = keys[t];
      if ((kk & mask) == prefix) atomicAdd(&hist[warp][(kk >> shift) & dmask], 1);
    }
    __syncthreads();
    // bin totals (fixed order over the warps), thread b < 256 holds bin b
    int tot = 0;
    if (threadIdx.x < 256)
      for (int w = 0; w < NW; ++w) tot += hist[w][threadIdx.x];
    __syncthreads();
    if (threadIdx.x < 256) hist[0][threadIdx.x] = tot;
    __syncthreads();
    // the digit: the largest d whose keys, with those of the digits above it, number at least
    // `need`.  Thread j < 256 takes bin 255 - j, so an inclusive scan over j counts the keys at
    // and above that digit; the first j to reach `need` names it.
    if (threadIdx.x < 256) {
      const int b = 255 - (int)threadIdx.x;
      const int v = b <= (int)dmask ? hist[0][b] : 0;
      int inc = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
      }
      if (lane == 31) s_warp[warp] = inc;
      asm volatile("bar.sync 1, 256;" ::: "memory");      // the 8 warps of threads < 256
      int before = 0;
      for (int w = 0; w < warp; ++w) before += s_warp[w];
      inc += before;
      if (inc >= need && inc - v < need) {
        s_digit = b;
        s_need = need - (inc - v);
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s_digit << shift;
    mask |= dmask << shift;
    need = s_need;
    __syncthreads();
    if (shift == 0) break;
  }
  // prefix is now the c-th largest key; take everything above it and the first `need` equal
  // keys in token order
  const int per = (T + blockDim.x - 1) / blockDim.x;
  const int t0 = threadIdx.x * per, t1 = min(T, t0 + per);
  int gt = 0, eq = 0;
  for (int t = t0; t < t1; ++t) {
    const uint32_t kk = keys[t];
    gt += kk > prefix;
    eq += kk == prefix;
  }
  int total;
  const int gt_before = block_exclusive_scan(gt, s_warp, &total);
  int eq_before = block_exclusive_scan(eq, s_warp, &total);
  int pos = gt_before + min(eq_before, need);
  for (int t = t0; t < t1; ++t) {
    const uint32_t kk = keys[t];
    bool take = kk > prefix;
    if (kk == prefix) {
      take = eq_before < need;
      ++eq_before;
    }
    if (take) {
      if (pos < c) picked[(int64_t)e * c + pos] = t;
      ++pos;
    }
  }
}

// ---- fast path: bf16 token choice, E <= 8, D = 256 * NW with 4 <= NW <= 16 ----
//
// The router product is an HBM-bound contraction with N = E <= 8 experts: exactly the N of
// mma.sync m16n8k16, so the FMAs (and the bf16 -> fp32 conversions a CUDA-core dot product
// needs) go to the tensor cores and the kernel is left with streaming x.  One CTA of NW warps
// owns a contiguous range of tokens; warp w owns the hidden slice [256w, 256w + 256).  The k
// order inside the slice is permuted (the same permutation for x and W_g, which leaves the sum
// unchanged) so that each thread's A fragments over the 16 k-steps are eight 16-byte chunks of
// two token rows and its B fragments the same eight chunks of one W_g row: every global load is
// a 16-byte vector load, and the 4 threads of a row read 64 contiguous bytes together.  Per 16-token batch a warp issues 16 MMAs; partial
// logits of the NW warps are summed in a fixed order through shared memory, the next batch's
// loads are already in flight while warps do the per-token affinity / top-k / gates.
constexpr int kFastE = 8;        // MMA N: experts (zero-padded)
constexpr int kFastTB = 16;      // MMA M: tokens per batch
constexpr int kFastMaxNW = 16;

__device__ __forceinline__ void mma_16816_bf16(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two token rows (g, g + 8 of the batch): this thread's 8 chunks of 8 elements, chunk i at
// element kbase + 32 i (kbase = 256 w + 8 tig), so the 4 threads of a row read 64 contiguous
// bytes per load instruction.
__device__ __forceinline__ void load_rows(uint4 (&r0)[8], uint4 (&r1)[8],
                                          const __nv_bfloat16* x, int D, int t0, int t_end,
                                          int g, int kbase) {
  const int ta = t0 + g, tb = t0 + g + 8;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    r0[i] = (ta < t_end)
                ? __ldcs(reinterpret_cast<const uint4*>(x + (int64_t)ta * D + kbase + 32 * i))
                : make_uint4(0u, 0u, 0u, 0u);
    r1[i] = (tb < t_end)
                ? __ldcs(reinterpret_cast<const uint4*>(x + (int64_t)tb * D + kbase + 32 * i))
                : make_uint4(0u, 0u, 0u, 0u);
  }
}

__device__ __forceinline__ void select_token(const RouterArgs& a, int tok, float sv, bool live,
                                             int lane, float& imp, float& ent) {
  const int E = a.E;
  if (a.logits && live) a.logits[(int64_t)tok * E + lane] = sv;
  float selw, key;
  if (a.score == MOE_SCORE_SOFTMAX) {
    const float m = warp_max(sv);
    const float z = live ? expf(sv - m) : 0.f;
    const float p = z / warp_sum(z);
    selw = p;
    key = sv;                    // softmax is monotone in the logit within a row
    imp += p;
    if (p > 0.f) ent -= p * logf(p);
  } else {
    const float af = live ? 1.0f / (1.0f + expf(-sv)) : 0.f;
    selw = af;
    key = live ? af + (a.bias ? a.bias[lane] : 0.f) : -INFINITY;
    const float q = af / warp_sum(af);
    imp += q;
    if (q > 0.f) ent -= q * logf(q);
  }
  {
    float kk[1] = {key};
    group_limit<1>(kk, E, a.n_group, a.topk_group, lane);
    key = kk[0];
  }
  bool taken = !live;
  int my_id = -1;
  float my_w = 0.f, wsum = 0.f;
  for (int j = 0; j < a.k; ++j) {
    float bk = taken ? -INFINITY : key;
    int bi = taken ? 0x7fffffff : lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ok > bk || (ok == bk && oi < bi)) { bk = ok; bi = oi; }
    }
    const float wv = __shfl_sync(0xffffffffu, selw, bi & 31);
    if (lane == bi) taken = true;
    wsum += wv;
    if (lane == j) { my_id = (bi < E) ? bi : -1; my_w = wv; }
  }
  if (lane < a.k) {
    a.ids[(int64_t)tok * a.k + lane] = my_id;
    a.gates[(int64_t)tok * a.k + lane] = (a.gate == MOE_GATE_RENORM) ? my_w / wsum : my_w;
  }
}

__global__ void __launch_bounds__(kFastMaxNW * 32, 1)
router_fast_kernel(RouterArgs a, int tokens_per_cta) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_red[kFastMaxNW][kFastTB][kFastE];
  __shared__ float s_log[kFastTB][kFastE];
  __shared__ float s_imp[kFastTB][kFastE];
  __shared__ float s_ent[kFastTB];
  const int NW = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int E = a.E;
  const int kbase = warp * 256 + tig * 8;    // this thread's chunks: kbase + 32 i, i < 8
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.x);
  const __nv_bfloat16* Wg = static_cast<const __nv_bfloat16*>(a.Wg);
  uint4 wv[8];                               // W_g[g][kbase + 32 i .. + 8)
#pragma unroll
  for (int i = 0; i < 8; ++i)
    wv[i] = (g < E) ? __ldg(reinterpret_cast<const uint4*>(Wg + (int64_t)g * a.D + kbase + 32 * i))
                    : make_uint4(0u, 0u, 0u, 0u);
  const int t_begin = blockIdx.x * tokens_per_cta;
  const int t_end = min(a.T, t_begin + tokens_per_cta);
  float imp = 0.f, ent = 0.f;
  uint4 r0[8], r1[8];
  load_rows(r0, r1, x, a.D, t_begin, t_end, g, kbase);
  for (int t0 = t_begin; t0 < t_end; t0 += kFastTB) {
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // k-steps 2i (chunk elements 0..3) and 2i+1 (chunk elements 4..7)
      mma_16816_bf16(c, r0[i].x, r1[i].x, r0[i].y, r1[i].y, wv[i].x, wv[i].y);
      mma_16816_bf16(c, r0[i].z, r1[i].z, r0[i].w, r1[i].w, wv[i].z, wv[i].w);
    }
    if (t0 + kFastTB < t_end) load_rows(r0, r1, x, a.D, t0 + kFastTB, t_end, g, kbase);
    s_red[warp][g][2 * tig] = c[0];
    s_red[warp][g][2 * tig + 1] = c[1];
    s_red[warp][g + 8][2 * tig] = c[2];
    s_red[warp][g + 8][2 * tig + 1] = c[3];
    __syncthreads();
    if (threadIdx.x < kFastTB * kFastE) {
      const int j = threadIdx.x / kFastE, e = threadIdx.x % kFastE;
      float sum = 0.f;
      for (int ww = 0; ww < NW; ++ww) sum += s_red[ww][j][e];
      s_log[j][e] = sum;
    }
    __syncthreads();
    for (int jj = warp; jj < kFastTB; jj += NW) {
      if (t0 + jj >= t_end) break;
      const bool live = lane < E;
      select_token(a, t0 + jj, live ? s_log[jj][lane] : -INFINITY, live, lane, imp, ent);
    }
  }
  // CTA importance partial: sum over the selection warps in a fixed order
  const int n_sel = NW < kFastTB ? NW : kFastTB;
  if (warp < n_sel && lane < kFastE) s_imp[warp][lane] = imp;
  ent = warp_sum(ent);
  if (warp < n_sel && lane == 0) s_ent[warp] = ent;
  __syncthreads();
  if (a.partials && threadIdx.x <= E) {      // row: E importance sums, then the entropy sum
    float sum = 0.f;
    for (int j = 0; j < n_sel; ++j) sum += (threadIdx.x < E) ? s_imp[j][threadIdx.x] : s_ent[j];
    a.partials[(int64_t)blockIdx.x * (E + 1) + threadIdx.x] = sum;
  }
}

}  // namespace

// Tokens per warp of the generic kernel: 1 when the logits come from the tensor-core product.
static int router_tpw(bool lpart) { return lpart ? 1 : kTPW; }

// Rows of importance partials the generic kernel writes (one per block).
static int generic_partials(const moe_desc_t& d, bool lpart) {
  const int per_block = kWarps * router_tpw(lpart);
  return (d.T + per_block - 1) / per_block;
}

int router_partials(const moe_desc_t& d) {
  // capacity for either kernel: generic = one row per block of 8 (or 32) tokens; fast = one
  // row per CTA (<= 1024)
  const int generic = generic_partials(d, true);
  return generic > 1024 ? generic : 1024;
}

template <bool BF16, int TPW>
static void launch_router_tpw(const RouterArgs& a, int T, cudaStream_t s) {
  const int blocks = (T + kWarps * TPW - 1) / (kWarps * TPW);
  // the warps' logits [kWarps * TPW][E] (then, under expert choice, the transposed
  // probabilities [kWarps * TPW][E + 1] after them); the partial rows [kWarps][E + 1] reuse the
  // start of the buffer at the end, so it holds at least that many
  size_t words = (size_t)kWarps * TPW * a.E;
  if (a.expert_choice) words += (size_t)kWarps * TPW * (a.E + 1);
  const size_t part_words = (size_t)kWarps * (a.E + 1);
  if (words < part_words) words = part_words;
  const size_t smem = words * sizeof(float);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(router_kernel<BF16, TPW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
  (void)launch_pdl(router_kernel<BF16, TPW>, dim3(blocks), dim3(kWarps * 32), smem, s, a);
}

static cudaError_t launch_router(const RouterArgs& a, bool bf16, int T, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (a.lpart)
    launch_router_tpw<true, 1>(a, T, s);        // the tensor-core product is bf16-only
  else if (bf16)
    launch_router_tpw<true, kTPW>(a, T, s);
  else
    launch_router_tpw<false, kTPW>(a, T, s);
  return cudaGetLastError();
}

// Router path.  Default: for bf16 with at most 8 experts the mma.sync kernel (when D is a
// multiple of 256 between 1024 and 4096: measured faster there), otherwise the tensor-core
// router fused with the selection (router_tc.cu: bf16, D % 64 == 0, E <= 256), otherwise the
// SIMT kernel.  MOE_ROUTER selects one path for comparison measurements (each is tested):
// "tc", "fast" (mma.sync, E <= 8), "gemm" (the grouped-GEMM router product, k-split fp32
// partial logits in the step scratch, then the SIMT selection kernel) or "simt".
enum RouterMode { ROUTER_AUTO = -1, ROUTER_TC = 0, ROUTER_GEMM = 1, ROUTER_FAST = 2, ROUTER_SIMT = 3 };
static int router_env() {
  static int v = [] {
    const char* e = getenv("MOE_ROUTER");
    if (!e) return (int)ROUTER_AUTO;
    if (!strcmp(e, "tc")) return (int)ROUTER_TC;
    if (!strcmp(e, "gemm")) return (int)ROUTER_GEMM;
    if (!strcmp(e, "fast")) return (int)ROUTER_FAST;
    if (!strcmp(e, "simt")) return (int)ROUTER_SIMT;
    return (int)ROUTER_AUTO;
  }();
  return v;
}

// The grouped-GEMM router product (MOE_ROUTER=gemm): bf16, 32 <= E <= 256, E % 32 == 0.
bool router_uses_gemm(const moe_desc_t& d) {
  return router_env() == ROUTER_GEMM && d.dtype == MOE_BF16 && d.E >= 32 && d.E % 32 == 0 &&
         d.E <= 256 && d.D % 64 == 0;
}

size_t router_gemm_scratch_bytes(const moe_desc_t& d) {
  return router_uses_gemm(d) ? (size_t)8 * d.T * d.E * sizeof(float) : 0;
}

static bool fast_router_ok(const moe_desc_t& d) {
  return d.dtype == MOE_BF16 && d.select == MOE_TOKEN_CHOICE && d.E <= kFastE &&
         d.D % 256 == 0 && d.D / 256 >= 4 && d.D / 256 <= kFastMaxNW && d.k <= 32;
}

static bool use_router_fast(const moe_desc_t& d) {
  const int m = router_env();
  return (m == ROUTER_AUTO || m == ROUTER_FAST) && fast_router_ok(d);
}

static bool use_router_tc(const moe_desc_t& d) {
  const int m = router_env();
  return (m == ROUTER_TC || (m == ROUTER_AUTO && !fast_router_ok(d))) && router_tc_ok(d);
}

cudaError_t launch_router_token_choice(const moe_desc_t& d, const void* x, const void* Wg,
                                       const float* bias, int32_t* ids, float* gates,
                                       float* logits, float* imp_partials, int* n_partials,
                                       float* lpart, cudaStream_t s) {
  RouterArgs a{x, Wg, bias, ids, gates, logits, nullptr, imp_partials,
               d.T, d.D, d.E, d.k, d.score, d.gate, 0, nullptr, 1};
  a.n_group = d.n_group;
  a.topk_group = d.topk_group;
  if (use_router_tc(d)) return launch_router_tc(d, a, n_partials, s);
  if (router_uses_gemm(d) && lpart) {
    const int ks = router_gemm_splits(d.T, d.D);
    cudaError_t e = launch_router_gemm_bf16(x, d.T, d.D, Wg, d.E, lpart, ks, s);
    if (e != cudaSuccess) return e;
    a.lpart = lpart;
    a.ksplit = ks;
  }
  if (use_router_fast(d)) {
    const int sms = num_sms() < 1024 ? num_sms() : 1024;
    const int tpc = (d.T + sms - 1) / sms;
    const int grid = tpc > 0 ? (d.T + tpc - 1) / tpc : 0;
    *n_partials = grid;
    if (grid == 0) return cudaSuccess;
    (void)launch_pdl(router_fast_kernel, dim3(grid), dim3((d.D / 256) * 32), 0, s, a, tpc);
    return cudaGetLastError();
  }
  *n_partials = generic_partials(d, a.lpart != nullptr);
  return launch_router(a, d.dtype == MOE_BF16, d.T, s);
}

cudaError_t launch_router_expert_choice(const moe_desc_t& d, const void* x, const void* Wg,
                                        float* probs, float* probsT, float* logits,
                                        float* imp_partials, int* n_partials, float* lpart,
                                        cudaStream_t s) {
  RouterArgs a{x, Wg, nullptr, nullptr, probs, logits, probsT, imp_partials,
               d.T, d.D, d.E, 0, MOE_SCORE_SOFTMAX, MOE_GATE_RAW, 1, nullptr, 1};
  if (use_router_tc(d)) return launch_router_tc(d, a, n_partials, s);
  if (router_uses_gemm(d) && lpart) {
    const int ks = router_gemm_splits(d.T, d.D);
    cudaError_t e = launch_router_gemm_bf16(x, d.T, d.D, Wg, d.E, lpart, ks, s);
    if (e != cudaSuccess) return e;
    a.lpart = lpart;
    a.ksplit = ks;
  }
  *n_partials = generic_partials(d, a.lpart != nullptr);
  return launch_router(a, d.dtype == MOE_BF16, d.T, s);
}

cudaError_t launch_ec_select(const moe_desc_t& d, const float* probsT, int32_t* picked,
                             cudaStream_t s) {
  const size_t smem = (size_t)d.T * sizeof(float);
  if (d.T % 4 == 0 && smem <= 180 * 1024) {      // + 33 KB of static shared memory
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(ec_select_kernel<true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    (void)launch_pdl(ec_select_kernel<true>, dim3(d.E), dim3(1024), smem, s, probsT, d.T, d.c, picked);
  } else {
    (void)launch_pdl(ec_select_kernel<false>, dim3(d.E), dim3(1024), 0, s, probsT, d.T, d.c, picked);
  }
  return cudaGetLastError();
}

cudaError_t launch_importance_reduce(const float* partials, int n_partials, int E, int T,
                                     float* importance, float* entropy, cudaStream_t s) {
  (void)launch_pdl(importance_reduce_kernel, dim3(E + 1), dim3(256), 0, s, partials, n_partials, E, T, importance,
                                                          entropy);
  return cudaGetLastError();
}

}  // namespace moe
