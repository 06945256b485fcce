// Combine (unpermute + weighted sum) and the balance statistics.
//
// Combine: "Top-k 路由（Top-k Routing）" (compassingai), Combine box (output = sum of
// gate_score_i * y_i over the selected experts) and "門控函式的數學形式" Step 3;
// "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife), section 6
// (contributions are accumulated, never assigned).  Each output row is produced by one warp
// that walks the token's assignments in slot order through the inverse permutation, so the
// sum has a fixed order and needs no atomics; a dropped or unpicked assignment (row -1) adds
// nothing.  Shared experts ("别只比较 Top-k" family table, DeepSeek rows) add with weight 1.
//
// Statistics: "Top-k 路由" load-balancing loss L = alpha * N * sum_i f_i P_i; Tiny MoE section 8
// (importance before top-k, load after top-k; E * sum p_e f_e = 1 at balance); "别只比较
// Top-k" section "先数 assignments" (max/mean imbalance, [9,4,2,1] -> 2.25) and its monitoring
// list (per-expert counts, max/mean and P95/P99, router entropy).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxList = 256;      // assignments per token held in shared memory (K <= 256)

template <bool BF16> struct Row;
template <> struct Row<true> {     // 8 bf16 per 16 bytes
  static constexpr int N = 8;
  __device__ __forceinline__ static void acc(const uint4* p, float g, float* a) {
    acc_val(__ldcs(p), g, a);
  }
  __device__ __forceinline__ static void acc_val(const uint4 u, float g, float* a) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[2 * i] = fmaf(g, __uint_as_float(w[i] << 16), a[2 * i]);
      a[2 * i + 1] = fmaf(g, __uint_as_float(w[i] & 0xffff0000u), a[2 * i + 1]);
    }
  }
  __device__ __forceinline__ static void store(uint4* p, const float* a) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(a[2 * i], a[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *p = make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <> struct Row<false> {    // 4 fp32 per 16 bytes
  static constexpr int N = 4;
  __device__ __forceinline__ static void acc(const uint4* p, float g, float* a) {
    acc_val(__ldcs(p), g, a);
  }
  __device__ __forceinline__ static void acc_val(const uint4 u, float g, float* a) {
    const float4 f = make_float4(__uint_as_float(u.x), __uint_as_float(u.y),
                                 __uint_as_float(u.z), __uint_as_float(u.w));
    a[0] = fmaf(g, f.x, a[0]); a[1] = fmaf(g, f.y, a[1]);
    a[2] = fmaf(g, f.z, a[2]); a[3] = fmaf(g, f.w, a[3]);
  }
  __device__ __forceinline__ static void store(uint4* p, const float* a) {
    *reinterpret_cast<float4*>(p) = make_float4(a[0], a[1], a[2], a[3]);
  }
};

// The balance statistics of one layer call, computed by one block of 256 threads (E <= 256):
// f, aux, max/mean, kept/dropped, count percentiles (ranks by counting, ties by expert id) and
// the router's mean entropy; fixed-order tree sums (deterministic).  Every thread of the block
// calls it.
__device__ __noinline__ void balance_stats_block(const StatsArgs& a) {
  __shared__ float s_fp[256];
  __shared__ int s_max[256];
  __shared__ int s_sorted[256];
  __shared__ int s_cnt[256];
  const int tid = threadIdx.x;
  const int E = a.E;
  float fp = 0.f;
  int c = 0;
  if (tid < E) {
    c = a.counts[tid];
    s_cnt[tid] = c;
  }
  __syncthreads();
  if (tid < E) {
    const float fe = (float)c / (float)a.n_routes;
    a.f[tid] = fe;
    fp = fe * a.importance[tid];
    // rank of this count among all (ties by expert id): its slot in ascending order
    int rank = 0;
    for (int e = 0; e < E; ++e) {
      const int ce = s_cnt[e];
      rank += (ce < c) || (ce == c && e < tid);
    }
    s_sorted[rank] = c;
  }
  s_fp[tid] = fp;
  s_max[tid] = c;
  __syncthreads();
  for (int hw = 128; hw > 0; hw >>= 1) {        // fixed-order tree
    if (tid < hw) {
      s_fp[tid] += s_fp[tid + hw];
      s_max[tid] = max(s_max[tid], s_max[tid + hw]);
    }
    __syncthreads();
  }
  if (tid == 0) {
    const int kept = a.offsets[E];
    moe_stats_t r;
    r.aux = a.alpha * (float)E * s_fp[0];
    const float mean = (float)a.n_routes / (float)E;
    r.max_over_mean = mean > 0.f ? (float)s_max[0] / mean : 0.f;
    r.n_routes = a.n_routes;
    r.n_kept = kept;
    r.n_dropped = a.n_routes - kept;
    r.reserved = 0;
    r.entropy = a.entropy ? *a.entropy : __int_as_float(0x7fc00000);
    float q[2];
    const double pct[2] = {0.95, 0.99};
    for (int i = 0; i < 2; ++i) {
      const double pos = pct[i] * (double)(E - 1);
      const int lo = (int)pos;
      const int hi = lo + 1 < E ? lo + 1 : lo;
      const double fr = pos - lo;
      q[i] = (float)(s_sorted[lo] + fr * (double)(s_sorted[hi] - s_sorted[lo]));
    }
    r.count_p95 = q[0];
    r.count_p99 = q[1];
    r.reserved2 = 0.f;
    *a.st = r;
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32)
combine_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ inv,
               const float* __restrict__ gates, const uint4* __restrict__ ys, int S, int T,
               int K, int nvec, uint4* __restrict__ out, const StatsArgs sa) {
  pdl_trigger();
  pdl_wait();
  if (sa.st && blockIdx.x == 0) balance_stats_block(sa);
  using R = Row<BF16>;
  __shared__ int s_row[kWarps][kMaxList];
  __shared__ float s_g[kWarps][kMaxList];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= T) return;
  // Compact the token's live assignments, keeping slot order.
  int n = 0;
  for (int j0 = 0; j0 < K; j0 += 32) {
    const int j = j0 + lane;
    const int r = (j < K) ? inv[(int64_t)t * K + j] : -1;
    const float g = (j < K && r >= 0) ? gates[(int64_t)t * K + j] : 0.f;
    const unsigned live = __ballot_sync(0xffffffffu, r >= 0);
    if (r >= 0) {
      const int pos = n + __popc(live & ((1u << lane) - 1u));
      s_row[warp][pos] = r;
      s_g[warp][pos] = g;
    }
    n += __popc(live);
  }
  __syncwarp();
  // four 16-byte chunks per lane at a time: the loads of one assignment row are all in flight
  // before they are accumulated (the same fixed order of the sum as one chunk at a time)
  int v = lane;
  for (; v + 96 < nvec; v += 128) {
    float a[4][R::N];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int i = 0; i < R::N; ++i) a[c][i] = 0.f;
    for (int q = 0; q < n; ++q) {
      const uint4* src = y + (int64_t)s_row[warp][q] * nvec + v;
      const float gq = s_g[warp][q];
      uint4 u[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) u[c] = __ldcs(src + 32 * c);
#pragma unroll
      for (int c = 0; c < 4; ++c) R::acc_val(u[c], gq, a[c]);
    }
    for (int s = 0; s < S; ++s) {
      const uint4* src = ys + ((int64_t)s * T + t) * nvec + v;
      uint4 u[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) u[c] = __ldcs(src + 32 * c);
#pragma unroll
      for (int c = 0; c < 4; ++c) R::acc_val(u[c], 1.0f, a[c]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) R::store(out + (int64_t)t * nvec + v + 32 * c, a[c]);
  }
  for (; v < nvec; v += 32) {
    float a[R::N];
#pragma unroll
    for (int i = 0; i < R::N; ++i) a[i] = 0.f;
    for (int q = 0; q < n; ++q) R::acc(y + (int64_t)s_row[warp][q] * nvec + v, s_g[warp][q], a);
    for (int s = 0; s < S; ++s) R::acc(ys + ((int64_t)s * T + t) * nvec + v, 1.0f, a);
    R::store(out + (int64_t)t * nvec + v, a);
  }
}


// K <= 2 and no shared experts (Mixtral, Switch): each lane keeps 4 chunks x K rows of loads in
// flight before accumulating, so a warp has up to 4 KB outstanding.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <bool BF16, int K>
__global__ void __launch_bounds__(kWarps * 32)
combine_small_k_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ inv,
                       const float* __restrict__ gates, int T, int nvec,
                       uint4* __restrict__ out, const StatsArgs sa, const SplitRows sr) {
  pdl_trigger();
  pdl_wait();
  if (sa.st && blockIdx.x == 0) balance_stats_block(sa);
  using R = Row<BF16>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= T) return;
  int row[K];
  float g[K];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    row[j] = inv[(int64_t)t * K + j];
    g[j] = row[j] >= 0 ? gates[(int64_t)t * K + j] : 0.f;
  }
  const int S = (BF16 && sr.part) ? __ldg(sr.ks) : 1;
  if (BF16 && S > 1) {
    // y rows from the k-split partials: the S partial values of 8 columns summed in split
    // order, rounded once to bf16, stored to y and weighted into the output
    const int64_t live = min((int64_t)__ldg(sr.n_rows), sr.rows);
    const int64_t ncol = (int64_t)nvec * 8;
    const int64_t stride = live * ncol;
    uint4* yw = static_cast<uint4*>(sr.y);
    for (int v = lane; v < nvec; v += 32) {
      float acc[R::N];
#pragma unroll
      for (int i = 0; i < R::N; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < K; ++j) {
        if (row[j] < 0 || row[j] >= live) continue;
        const float* pr = sr.part + (int64_t)row[j] * ncol + 8 * v;
        float4 a0 = __ldcs(reinterpret_cast<const float4*>(pr));
        float4 a1 = __ldcs(reinterpret_cast<const float4*>(pr + 4));
        for (int sp = 1; sp < S; ++sp) {
          const float4 b0 = __ldcs(reinterpret_cast<const float4*>(pr + sp * stride));
          const float4 b1 = __ldcs(reinterpret_cast<const float4*>(pr + sp * stride + 4));
          a0.x += b0.x; a0.y += b0.y; a0.z += b0.z; a0.w += b0.w;
          a1.x += b1.x; a1.y += b1.y; a1.z += b1.z; a1.w += b1.w;
        }
        const uint4 yb = make_uint4(pack_bf16x2(a0.x, a0.y), pack_bf16x2(a0.z, a0.w),
                                    pack_bf16x2(a1.x, a1.y), pack_bf16x2(a1.z, a1.w));
        yw[(int64_t)row[j] * nvec + v] = yb;
        R::acc_val(yb, g[j], acc);
      }
      R::store(out + (int64_t)t * nvec + v, acc);
    }
    return;
  }
  int v = lane;
  for (; v + 96 < nvec; v += 128) {
    uint4 q[K][4];
#pragma unroll
    for (int j = 0; j < K; ++j)
#pragma unroll
      for (int u = 0; u < 4; ++u)
        q[j][u] = row[j] >= 0 ? __ldcs(y + (int64_t)row[j] * nvec + v + 32 * u)
                              : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float acc[R::N];
#pragma unroll
      for (int i = 0; i < R::N; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < K; ++j)
        if (row[j] >= 0) R::acc_val(q[j][u], g[j], acc);
      R::store(out + (int64_t)t * nvec + v + 32 * u, acc);
    }
  }
  for (; v < nvec; v += 32) {
    float acc[R::N];
#pragma unroll
    for (int i = 0; i < R::N; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j)
      if (row[j] >= 0) R::acc(y + (int64_t)row[j] * nvec + v, g[j], acc);
    R::store(out + (int64_t)t * nvec + v, acc);
  }
}

// The statistics as a kernel of their own (moe_balance_stats): one block of 256 threads.
__global__ void __launch_bounds__(256) stats_kernel(const StatsArgs a) {
  pdl_trigger();
  pdl_wait();
  balance_stats_block(a);
}

}  // namespace

StatsArgs stats_args(const moe_desc_t& d, const int32_t* counts, const int32_t* offsets,
                     const float* importance, const float* entropy, float* f,
                     moe_stats_t* stats) {
  StatsArgs a;
  a.counts = counts;
  a.offsets = offsets;
  a.importance = importance;
  a.entropy = entropy;
  a.E = d.E;
  a.n_routes = (d.select == MOE_EXPERT_CHOICE) ? d.E * d.c : d.T * d.k;
  a.alpha = d.aux_alpha;
  a.f = f;
  a.st = stats;
  return a;
}

cudaError_t launch_combine(const moe_desc_t& d, const void* y, const int32_t* inv,
                           const float* gates, const void* y_shared, void* out,
                           cudaStream_t s, const StatsArgs* with_stats,
                           const SplitRows* split) {
  if (d.T == 0) return cudaSuccess;
  StatsArgs sa{};
  if (with_stats) sa = *with_stats;
  SplitRows sr{};
  const bool small_k = !y_shared && d.select == MOE_TOKEN_CHOICE && d.k <= 2;
  if (split) {
    if (small_k && d.dtype == MOE_BF16 && d.D % 8 == 0) {
      sr = *split;
      sr.y = const_cast<void*>(y);
    } else {
      // the general combine reads y: sum the partials into it first
      cudaError_t e = launch_splitk_sum_adaptive(split->part, split->ks, split->rows, d.D,
                                                 split->n_rows, const_cast<void*>(y), s);
      if (e != cudaSuccess) return e;
    }
  }
  const int K = (d.select == MOE_EXPERT_CHOICE) ? d.E : d.k;
  const int esz = (d.dtype == MOE_BF16) ? 2 : 4;
  const int nvec = d.D * esz / 16;
  const int S = y_shared ? d.n_shared : 0;
  const int blocks = (d.T + kWarps - 1) / kWarps;
  if (small_k) {
    const uint4* yy = static_cast<const uint4*>(y);
    uint4* oo = static_cast<uint4*>(out);
    if (d.dtype == MOE_BF16) {
      if (K == 1) (void)launch_pdl(combine_small_k_kernel<true, 1>, dim3(blocks), dim3(kWarps * 32), 0, s, yy, inv, gates, d.T, nvec, oo, sa, sr);
      else (void)launch_pdl(combine_small_k_kernel<true, 2>, dim3(blocks), dim3(kWarps * 32), 0, s, yy, inv, gates, d.T, nvec, oo, sa, sr);
    } else {
      if (K == 1) (void)launch_pdl(combine_small_k_kernel<false, 1>, dim3(blocks), dim3(kWarps * 32), 0, s, yy, inv, gates, d.T, nvec, oo, sa, sr);
      else (void)launch_pdl(combine_small_k_kernel<false, 2>, dim3(blocks), dim3(kWarps * 32), 0, s, yy, inv, gates, d.T, nvec, oo, sa, sr);
    }
    return cudaGetLastError();
  }
  if (d.dtype == MOE_BF16)
    (void)launch_pdl(combine_kernel<true>, dim3(blocks), dim3(kWarps * 32), 0, s, 
        static_cast<const uint4*>(y), inv, gates, static_cast<const uint4*>(y_shared), S, d.T,
        K, nvec, static_cast<uint4*>(out), sa);
  else
    (void)launch_pdl(combine_kernel<false>, dim3(blocks), dim3(kWarps * 32), 0, s, 
        static_cast<const uint4*>(y), inv, gates, static_cast<const uint4*>(y_shared), S, d.T,
        K, nvec, static_cast<uint4*>(out), sa);
  return cudaGetLastError();
}

cudaError_t launch_balance_stats(const moe_desc_t& d, const int32_t* counts,
                                 const int32_t* offsets, const float* importance,
                                 const float* entropy, float* f, moe_stats_t* stats,
                                 cudaStream_t s) {
  (void)launch_pdl(stats_kernel, dim3(1), dim3(256), 0, s,
                   stats_args(d, counts, offsets, importance, entropy, f, stats));
  return cudaGetLastError();
}

}  // namespace moe
