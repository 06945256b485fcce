// fp32 expert FFN on CUDA cores (the fp32 workloads: fp32 accumulation end to end, so the
// layer matches an fp64 evaluation to ~1e-6; TF32 tensor cores would not).
//
// "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife),
// section 3: a SwiGLU expert is down(SiLU(x W_gate) * (x W_up)); the classic FFN uses one
// up matrix and an activation (ReLU, or the page's GELU).  Group g owns rows [offsets[g], offsets[g+1]).
#include "common.cuh"

namespace moe {
namespace {

__device__ __forceinline__ int group_of(const int32_t* offsets, int G, int r) {
  int lo = 0, hi = G - 1;                  // largest g with offsets[g] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(128)
ffn_up_f32_kernel(const float* __restrict__ a, int D, int F, const int32_t* offsets, int G,
                  const float* __restrict__ Wgate, const float* __restrict__ Wup, int act,
                  float* __restrict__ h) {
  extern __shared__ float s_x[];
  const int r = blockIdx.x;
  if (r >= offsets[G]) return;
  const int e = group_of(offsets, G, r);
  for (int d = threadIdx.x; d < D; d += blockDim.x) s_x[d] = a[(int64_t)r * D + d];
  __syncthreads();
  for (int f = threadIdx.x; f < F; f += blockDim.x) {
    const float* wu = Wup + ((int64_t)e * F + f) * D;
    float u = 0.f;
    for (int d = 0; d < D; ++d) u = fmaf(wu[d], s_x[d], u);
    float out;
    if (act == MOE_ACT_SWIGLU) {
      const float* wg = Wgate + ((int64_t)e * F + f) * D;
      float g = 0.f;
      for (int d = 0; d < D; ++d) g = fmaf(wg[d], s_x[d], g);
      out = g / (1.0f + expf(-g)) * u;
    } else if (act == MOE_ACT_GELU) {
      out = 0.5f * u * (1.0f + erff(u * 0.70710678118654752f));
    } else {
      out = fmaxf(u, 0.f);
    }
    h[(int64_t)r * F + f] = out;
  }
}

__global__ void __launch_bounds__(128)
ffn_down_f32_kernel(const float* __restrict__ h, int D, int F, const int32_t* offsets, int G,
                    const float* __restrict__ Wdown, float* __restrict__ y) {
  extern __shared__ float s_h[];
  const int r = blockIdx.x;
  if (r >= offsets[G]) return;
  const int e = group_of(offsets, G, r);
  for (int f = threadIdx.x; f < F; f += blockDim.x) s_h[f] = h[(int64_t)r * F + f];
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const float* wd = Wdown + ((int64_t)e * D + d) * F;
    float acc = 0.f;
    for (int f = 0; f < F; ++f) acc = fmaf(wd[f], s_h[f], acc);
    y[(int64_t)r * D + d] = acc;
  }
}

}  // namespace

cudaError_t launch_ffn_up_f32(int act, const float* a, int64_t a_rows, int D, int F,
                              const int32_t* offsets, int n_groups, const float* Wgate,
                              const float* Wup, float* h, cudaStream_t s) {
  if (a_rows <= 0) return cudaSuccess;
  const size_t smem = (size_t)D * sizeof(float);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(ffn_up_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  ffn_up_f32_kernel<<<counted((unsigned)a_rows), 128, smem, s>>>(a, D, F, offsets, n_groups, Wgate, Wup,
                                                        act, h);
  return cudaGetLastError();
}

cudaError_t launch_ffn_down_f32(const float* h, int64_t a_rows, int D, int F,
                                const int32_t* offsets, int n_groups, const float* Wdown,
                                float* y, cudaStream_t s) {
  if (a_rows <= 0) return cudaSuccess;
  const size_t smem = (size_t)F * sizeof(float);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(ffn_down_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  ffn_down_f32_kernel<<<counted((unsigned)a_rows), 128, smem, s>>>(h, D, F, offsets, n_groups, Wdown, y);
  return cudaGetLastError();
}

}  // namespace moe
