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

// enough blocks for every item of the allocated rows, at most 4 per SM (grid-stride beyond)
int grid_for(int64_t rows, int n) {
  const int64_t items = rows * (n / 4);
  int64_t b = (items + kThreads - 1) / kThreads;
  const int64_t cap = 4LL * gemm_sm_count();
  if (b > cap) b = cap;
  return (int)(b > 0 ? b : 1);
}

}  // namespace

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
