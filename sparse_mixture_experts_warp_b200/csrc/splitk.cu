// Sums of the k-split partials of the small-batch expert schedule.
//
// "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife), section 3
// (SwiGLU expert: hidden = SiLU(x W_gate) * (x W_up), output = hidden W_down) and the classic
// D -> F -> D expert with ReLU or GELU; "别只比较 Top-k" (ailearn moe-comparison), the
// expert-work account ("专家工作账": a small decode batch leaves each expert's products with very
// few rows, so they stream the weights).  With a handful of
// executed rows the grouped GEMM has fewer tiles than SMs, so the products are split along K
// into fp32 partials [S][rows][N] (grouped_gemm_kernel, EPI_F32 with k-splits) and these
// kernels add the S partials in a fixed order (deterministic), apply the activation and round
// once to bf16:
//   launch_splitk_act:  h[r, f] = act(sum_s Pg[s][r][f], sum_s Pu[s][r][f]) (SwiGLU: SiLU(g) * u;
//                       ReLU / GELU: act(u), Pg unused); the partials' rows are ld apart (gate
//                       and up in one buffer: Pu = Pg + ld / 2);
//   launch_splitk_sum:  y[r, n] = sum_s P[s][r][n].
// Rows at or past *n_rows (the executed-row count, offsets[G] on the device) are left alone:
// nothing reads them.  Both are HBM-bound elementwise passes over S * rows * N fp32 values,
// 16-byte loads and 8-byte stores, a grid-stride loop over four columns per thread.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float4 sum_splits(const float* __restrict__ p, int S, int64_t stride,
                                             int64_t off) {
  float4 a = __ldcs(reinterpret_cast<const float4*>(p + off));
  for (int s = 1; s < S; ++s) {
    const float4 b = __ldcs(reinterpret_cast<const float4*>(p + s * stride + off));
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
  }
  return a;
}

// the same arithmetic as the grouped GEMM's fused epilogues
__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}
__device__ __forceinline__ float gelu(float a) {
  return 0.5f * a * (1.0f + erff(a * 0.70710678118654752f));
}

template <int ACT>
__global__ void __launch_bounds__(kThreads)
splitk_act_kernel(const float* __restrict__ pg, const float* __restrict__ pu, int S,
                  int64_t rows, int F, int64_t ld, const int32_t* __restrict__ n_rows,
                  __nv_bfloat16* __restrict__ h) {
  pdl_trigger();
  pdl_wait();
  const int64_t live = min((int64_t)__ldg(n_rows), rows);
  const int q = F / 4;                       // four columns per item
  const int64_t items = live * q;
  const int64_t stride = rows * ld;
  for (int64_t i = blockIdx.x * (int64_t)kThreads + threadIdx.x; i < items;
       i += (int64_t)gridDim.x * kThreads) {
    const int64_t r = i / q;
    const int64_t cidx = (i - r * q) * 4;
    const int64_t off = r * F + cidx;          // in h
    const int64_t poff = r * ld + cidx;        // in the partials
    const float4 u = sum_splits(pu, S, stride, poff);
    float4 o;
    if (ACT == MOE_ACT_SWIGLU) {
      const float4 g = sum_splits(pg, S, stride, poff);
      o = make_float4(silu_mul(g.x, u.x), silu_mul(g.y, u.y), silu_mul(g.z, u.z),
                      silu_mul(g.w, u.w));
    } else if (ACT == MOE_ACT_GELU) {
      o = make_float4(gelu(u.x), gelu(u.y), gelu(u.z), gelu(u.w));
    } else {
      o = make_float4(fmaxf(u.x, 0.f), fmaxf(u.y, 0.f), fmaxf(u.z, 0.f), fmaxf(u.w, 0.f));
    }
    *reinterpret_cast<uint2*>(h + off) = make_uint2(pack2(o.x, o.y), pack2(o.z, o.w));
  }
}

__global__ void __launch_bounds__(kThreads)
splitk_sum_kernel(const float* __restrict__ p, int S, int64_t rows, int N,
                  const int32_t* __restrict__ n_rows, __nv_bfloat16* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const int64_t live = min((int64_t)__ldg(n_rows), rows);
  const int q = N / 4;
  const int64_t items = live * q;
  const int64_t stride = rows * (int64_t)N;
  for (int64_t i = blockIdx.x * (int64_t)kThreads + threadIdx.x; i < items;
       i += (int64_t)gridDim.x * kThreads) {
    const int64_t r = i / q;
    const int64_t off = r * N + (i - r * q) * 4;
    const float4 a = sum_splits(p, S, stride, off);
    *reinterpret_cast<uint2*>(y + off) = make_uint2(pack2(a.x, a.y), pack2(a.z, a.w));
  }
}

// The adaptive split's sum: the split count and the live rows come from the device.
__global__ void __launch_bounds__(kThreads)
splitk_sum_adaptive_kernel(const float* __restrict__ p, const int* __restrict__ ks, int64_t rows,
                           int N, const int32_t* __restrict__ n_rows,
                           __nv_bfloat16* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const int S = __ldg(ks);
  if (S <= 1) return;                       // the product wrote y
  const int64_t live = min((int64_t)__ldg(n_rows), rows);
  const int q = N / 4;
  const int64_t items = live * q;
  const int64_t stride = live * (int64_t)N;
  for (int64_t i = blockIdx.x * (int64_t)kThreads + threadIdx.x; i < items;
       i += (int64_t)gridDim.x * kThreads) {
    const int64_t r = i / q;
    const int64_t off = r * N + (i - r * q) * 4;
    const float4 a = sum_splits(p, S, stride, off);
    *reinterpret_cast<uint2*>(y + off) = make_uint2(pack2(a.x, a.y), pack2(a.z, a.w));
  }
}

// Stream-K sums: the partial slots of a tile are the segments of the CTAs whose k-block ranges
// meet it (the schedule in common.cuh); every group has at most 64 rows, so group g's tiles are
// tiles nt * (non-empty groups before g) + n for its n-tiles n.
constexpr int kMaxGroups = 1024;

// Sum of the nseg partial slots of 4 columns at offset off (slot order).
__device__ __forceinline__ float4 sum_slots(const float* __restrict__ p, int nseg, int64_t stride,
                                            int64_t off) {
  return sum_splits(p, nseg, stride, off);
}

template <int ACT>   // MOE_ACT_*; -1: no activation
__global__ void __launch_bounds__(kThreads)
splitk_streamk_kernel(const float* __restrict__ part, int slots, int64_t rows, int ld, int N,
                      int nkb, int two, const int32_t* __restrict__ offsets, int G, int grid,
                      __nv_bfloat16* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_off[kMaxGroups + 1];
  __shared__ int s_pre[kMaxGroups + 1];
  for (int i = threadIdx.x; i <= G; i += blockDim.x) s_off[i] = __ldg(offsets + i);
  __syncthreads();
  if (threadIdx.x < 32) {
    // exclusive prefix count of the non-empty groups, 32 at a time
    const int lane = threadIdx.x;
    int carry = 0;
    for (int g0 = 0; g0 < G; g0 += 32) {
      const int g = g0 + lane;
      const int ne = (g < G && s_off[g + 1] > s_off[g]) ? 1 : 0;
      int inc = ne;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
      }
      if (g < G) s_pre[g] = carry + inc - ne;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) s_pre[G] = carry;
  }
  __syncthreads();
  const int half = (N + 255) / 256;
  const int nt = two ? 2 * half : half;
  const int64_t work = (int64_t)nt * s_pre[G] * nkb;
  const int gct = streamk_ctas(work, nkb, slots, grid);
  const int64_t r_end = min((int64_t)s_off[G], rows);
  const int64_t live = r_end > s_off[0] ? r_end - s_off[0] : 0;
  const int q = N / 4;
  const int64_t items = live * q;
  const int64_t stride = rows * (int64_t)ld;
  for (int64_t i = blockIdx.x * (int64_t)kThreads + threadIdx.x; i < items;
       i += (int64_t)gridDim.x * kThreads) {
    const int64_t r = i / q + s_off[0];
    const int c = (int)(i - (i / q) * q) * 4;
    // the group of row r: the last g with s_off[g] <= r
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int64_t tb = (int64_t)nt * s_pre[lo];
    const int64_t t0 = tb + c / 256;
    const int n0 = streamk_owner((t0 + 1) * nkb - 1, work, gct) -
                   streamk_owner(t0 * nkb, work, gct) + 1;
    const float4 u = sum_slots(part, n0, stride, r * ld + c);
    float4 o;
    if (ACT == MOE_ACT_SWIGLU) {
      // u above is the gate (product 0); the up product's tile and columns follow
      const int64_t t1 = tb + half + c / 256;
      const int n1 = streamk_owner((t1 + 1) * nkb - 1, work, gct) -
                     streamk_owner(t1 * nkb, work, gct) + 1;
      const float4 v = sum_slots(part, n1, stride, r * ld + ld / 2 + c);
      o = make_float4(silu_mul(u.x, v.x), silu_mul(u.y, v.y), silu_mul(u.z, v.z),
                      silu_mul(u.w, v.w));
    } else if (ACT == MOE_ACT_GELU) {
      o = make_float4(gelu(u.x), gelu(u.y), gelu(u.z), gelu(u.w));
    } else if (ACT == MOE_ACT_RELU) {
      o = make_float4(fmaxf(u.x, 0.f), fmaxf(u.y, 0.f), fmaxf(u.z, 0.f), fmaxf(u.w, 0.f));
    } else {
      o = u;
    }
    *reinterpret_cast<uint2*>(out + r * N + c) = make_uint2(pack2(o.x, o.y), pack2(o.z, o.w));
  }
}

// enough blocks for every item of the allocated rows, at most 4 per SM (grid-stride beyond)
int grid_for(int64_t rows, int n) {
  const int64_t items = rows * (n / 4);
  int64_t b = (items + kThreads - 1) / kThreads;
  const int64_t cap = 4LL * gemm_sm_count();
  if (b > cap) b = cap;
  return (int)(b > 0 ? b : 1);
}

}  // namespace

cudaError_t launch_splitk_streamk(int act, const float* part, int slots, int64_t rows, int ld,
                                  int N, int K, int two, const int32_t* offsets, int G,
                                  void* out, cudaStream_t s) {
  if (rows <= 0 || N <= 0) return cudaSuccess;
  if (N % 4 || slots < 2 || G < 1 || G > kMaxGroups || (two && act != MOE_ACT_SWIGLU))
    return cudaErrorInvalidValue;
  const int nkb = (K + 63) / 64;
  const int grid = grid_for(rows, N);
  const int gemm_grid = gemm_sm_count();
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  if (act == MOE_ACT_SWIGLU)
    (void)launch_pdl(splitk_streamk_kernel<MOE_ACT_SWIGLU>, dim3(grid), dim3(kThreads), 0, s, part,
                     slots, rows, ld, N, nkb, two, offsets, G, gemm_grid, o);
  else if (act == MOE_ACT_GELU)
    (void)launch_pdl(splitk_streamk_kernel<MOE_ACT_GELU>, dim3(grid), dim3(kThreads), 0, s, part,
                     slots, rows, ld, N, nkb, two, offsets, G, gemm_grid, o);
  else if (act == MOE_ACT_RELU)
    (void)launch_pdl(splitk_streamk_kernel<MOE_ACT_RELU>, dim3(grid), dim3(kThreads), 0, s, part,
                     slots, rows, ld, N, nkb, two, offsets, G, gemm_grid, o);
  else
    (void)launch_pdl(splitk_streamk_kernel<-1>, dim3(grid), dim3(kThreads), 0, s, part, slots,
                     rows, ld, N, nkb, two, offsets, G, gemm_grid, o);
  return cudaGetLastError();
}

cudaError_t launch_splitk_act(int act, const float* pg, const float* pu, int S, int64_t rows,
                              int F, const int32_t* n_rows, void* h, cudaStream_t s, int64_t ld) {
  if (ld <= 0) ld = F;
  if (rows <= 0 || F <= 0) return cudaSuccess;
  if (F % 4 || S < 1) return cudaErrorInvalidValue;
  const int grid = grid_for(rows, F);
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(h);
  if (act == MOE_ACT_SWIGLU)
    (void)launch_pdl(splitk_act_kernel<MOE_ACT_SWIGLU>, dim3(grid), dim3(kThreads), 0, s, pg, pu, S, rows, F,
                                                                        ld, n_rows, o);
  else if (act == MOE_ACT_GELU)
    (void)launch_pdl(splitk_act_kernel<MOE_ACT_GELU>, dim3(grid), dim3(kThreads), 0, s, pg, pu, S, rows, F,
                                                                      ld, n_rows, o);
  else
    (void)launch_pdl(splitk_act_kernel<MOE_ACT_RELU>, dim3(grid), dim3(kThreads), 0, s, pg, pu, S, rows, F,
                                                                      ld, n_rows, o);
  return cudaGetLastError();
}

cudaError_t launch_splitk_sum(const float* p, int S, int64_t rows, int N, const int32_t* n_rows,
                              void* y, cudaStream_t s) {
  if (rows <= 0 || N <= 0) return cudaSuccess;
  if (N % 4 || S < 1) return cudaErrorInvalidValue;
  (void)launch_pdl(splitk_sum_kernel, dim3(grid_for(rows, N)), dim3(kThreads), 0, s, 
      p, S, rows, N, n_rows, static_cast<__nv_bfloat16*>(y));
  return cudaGetLastError();
}

cudaError_t launch_splitk_sum_adaptive(const float* p, const int* ks, int64_t rows, int N,
                                       const int32_t* n_rows, void* y, cudaStream_t s) {
  if (rows <= 0 || N <= 0) return cudaSuccess;
  if (N % 4) return cudaErrorInvalidValue;
  const int grid = grid_for(rows, N);
  (void)launch_pdl(splitk_sum_adaptive_kernel, dim3(grid), dim3(kThreads), 0, s, p, ks, rows, N,
                   n_rows, static_cast<__nv_bfloat16*>(y));
  return cudaGetLastError();
}

}  // namespace moe
