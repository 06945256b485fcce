// Backward pass of an fp32 MoE layer (the tiny MoE's precision), selection held fixed.
//
// "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife), section 9:
// the tiny MoE trains in fp32 with total loss = task loss + weight x router aux loss, the
// selected experts' gate / up / down matrices and the selected route weights getting gradients,
// the expert indices fixed integers; "Top-k 路由" section "門控網路的梯度流" (the selected gate
// scores carry the gradient, unselected experts none).  The arithmetic is that of the bf16
// backward (backward.cu) without the bf16 roundings: every product runs in one strided, grouped
// fp32 GEMM on CUDA cores (32 x 32 output tiles through shared memory, a fixed k order), the
// rest in small element-wise kernels.  This is the correctness path of small fp32 layers, not a
// tensor-core path.
#include "common.cuh"

namespace moe {
namespace {

// C_g(i, j) (+)= sum_k A_g(i, k) B_g(k, j) with strided operands:
//   A_g(i, k) = A[g a_g + i a_i + k a_k], B_g(k, j) = B[g b_g + k b_k + j b_j],
//   C_g(i, j) = C[g c_g + i c_i + j c_j].
// ROWS mode: group g owns the rows i in [off[g], off[g+1]) (M = rows bound), k in [0, K).
// KRED mode: group g owns the reduction range k in [off[g], off[g+1]), i in [0, M).
// off == nullptr: one group [0, M) (ROWS) or [0, K) (KRED).
struct F32Gemm {
  const float* A; int64_t a_g, a_i, a_k;
  const float* B; int64_t b_g, b_k, b_j;
  float* C; int64_t c_g, c_i, c_j;
  int M, N, K;
  const int32_t* off;
  int kred, accumulate;
};

constexpr int kT = 32;

__global__ void __launch_bounds__(256) gemm_f32_kernel(F32Gemm p) {
  __shared__ float As[kT][kT + 1];
  __shared__ float Bs[kT][kT + 1];
  const int g = blockIdx.z;
  int i_lo = 0, i_hi = p.M, k_lo = 0, k_hi = p.K;
  if (p.kred) {
    if (p.off) { k_lo = p.off[g]; k_hi = p.off[g + 1]; }
  } else if (p.off) {
    i_lo = p.off[g]; i_hi = p.off[g + 1];
  }
  const int i0 = i_lo + blockIdx.y * kT, j0 = blockIdx.x * kT;
  if (i0 >= i_hi) return;
  const float* A = p.A + (int64_t)g * p.a_g;
  const float* B = p.B + (int64_t)g * p.b_g;
  float* C = p.C + (int64_t)g * p.c_g;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;     // 2 x 2 outputs per thread
  float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  for (int k0 = k_lo; k0 < k_hi; k0 += kT) {
    for (int idx = threadIdx.x; idx < kT * kT; idx += 256) {
      const int r = idx / kT, c = idx % kT;
      const int ia = i0 + r, ka = k0 + c;
      As[r][c] = (ia < i_hi && ka < k_hi) ? A[(int64_t)ia * p.a_i + (int64_t)ka * p.a_k] : 0.f;
      const int kb = k0 + r, jb = j0 + c;
      Bs[r][c] = (kb < k_hi && jb < p.N) ? B[(int64_t)kb * p.b_k + (int64_t)jb * p.b_j] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kT; ++k) {
      const float a0 = As[ty][k], a1 = As[ty + 16][k];
      const float b0 = Bs[k][tx], b1 = Bs[k][tx + 16];
      acc[0][0] = fmaf(a0, b0, acc[0][0]);
      acc[0][1] = fmaf(a0, b1, acc[0][1]);
      acc[1][0] = fmaf(a1, b0, acc[1][0]);
      acc[1][1] = fmaf(a1, b1, acc[1][1]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int i = i0 + ty + 16 * u, j = j0 + tx + 16 * v;
      if (i < i_hi && j < p.N) {
        float* c = C + (int64_t)i * p.c_i + (int64_t)j * p.c_j;
        *c = p.accumulate ? *c + acc[u][v] : acc[u][v];
      }
    }
}

cudaError_t gemm_f32(const F32Gemm& p, int groups, int64_t m_rows_bound, cudaStream_t s) {
  if (groups <= 0 || p.N <= 0 || m_rows_bound <= 0) return cudaSuccess;
  const dim3 grid((p.N + kT - 1) / kT, (unsigned)((m_rows_bound + kT - 1) / kT), groups);
  gemm_f32_kernel<<<counted(grid), 256, 0, s>>>(p);
  return cudaGetLastError();
}

__device__ __forceinline__ float warp_sum32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp per executed row: dY[r] = g dout[t], dg = <dout[t], y[r]>.
__global__ void gather_dy_f32_kernel(const float* __restrict__ dout, const float* __restrict__ y,
                                     const int32_t* __restrict__ row_src,
                                     const float* __restrict__ gates,
                                     const int32_t* __restrict__ offsets, int E, int K, int D,
                                     int64_t rows_max, float* __restrict__ dY,
                                     float* __restrict__ dgates) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows_max || r >= offsets[E]) return;
  const int src = row_src[r];
  const int t = src / K;
  const float gt = gates[src];
  float dot = 0.f;
  for (int c = lane; c < D; c += 32) {
    const float a = dout[(int64_t)t * D + c];
    dot += a * y[r * D + c];
    dY[r * D + c] = gt * a;
  }
  dot = warp_sum32(dot);
  if (lane == 0) dgates[src] = dot;
}

// Activation backward on rows [0, n_rows): SwiGLU from the pre-activations a, b ([rows, F]
// each) to da, db (and h = SiLU(a) b when h is given); ReLU / GELU from z to dz (in da).
template <int ACT>
__global__ void act_backward_f32_kernel(const float* __restrict__ dH, const float* __restrict__ a,
                                        const float* __restrict__ b, const int32_t* n_rows_dev,
                                        int64_t n_rows_host, int F, float* __restrict__ da,
                                        float* __restrict__ db, float* __restrict__ h) {
  const int64_t rows = n_rows_dev ? (int64_t)*n_rows_dev : n_rows_host;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * F;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float dh = dH[i];
    if (ACT == 0) {
      const float av = a[i], bv = b[i];
      const float sg = 1.0f / (1.0f + expf(-av));
      da[i] = dh * bv * (sg * (1.0f + av * (1.0f - sg)));
      db[i] = dh * av * sg;
      if (h) h[i] = av * sg * bv;
    } else if (ACT == 1) {
      da[i] = a[i] > 0.f ? dh : 0.f;
    } else {
      const float z = a[i];
      da[i] = dh * (0.5f * (1.0f + erff(z * 0.70710678118654752f)) +
                    z * expf(-0.5f * z * z) * 0.39894228040143268f);
    }
  }
}

// dx[t] = sum_j dX[inv[t, j]] (fixed slot order) + sum_e ds[t, e] W_g[e] + sum_i dXs[i][t].
__global__ void dx_f32_kernel(const float* __restrict__ dX, const int32_t* __restrict__ inv,
                              const float* __restrict__ ds, const float* __restrict__ Wg, int T,
                              int D, int E, int K, const float* __restrict__ dXs, int n_add,
                              float* __restrict__ dx) {
  const int t = blockIdx.x;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < K; ++j) {
      const int r = inv[(int64_t)t * K + j];
      if (r >= 0) acc += dX[(int64_t)r * D + c];
    }
    for (int e = 0; e < E; ++e) acc += ds[(int64_t)t * E + e] * Wg[(int64_t)e * D + c];
    for (int i = 0; i < n_add; ++i) acc += dXs[((int64_t)i * T + t) * D + c];
    dx[(int64_t)t * D + c] = acc;
  }
}

int ew_grid(int64_t work) {
  int64_t b = (work + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (b > cap) b = cap;
  return b > 0 ? (int)b : 1;
}

cudaError_t act_backward_f32(int act, const float* dH, const float* a, const float* b,
                             const int32_t* n_rows_dev, int64_t rows, int F, float* da,
                             float* db, float* h, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int grid = ew_grid(rows * F);
  if (act == MOE_ACT_SWIGLU)
    act_backward_f32_kernel<0><<<counted(grid), 256, 0, s>>>(dH, a, b, n_rows_dev, rows, F, da,
                                                             db, h);
  else if (act == MOE_ACT_RELU)
    act_backward_f32_kernel<1><<<counted(grid), 256, 0, s>>>(dH, a, b, n_rows_dev, rows, F, da,
                                                             db, h);
  else
    act_backward_f32_kernel<2><<<counted(grid), 256, 0, s>>>(dH, a, b, n_rows_dev, rows, F, da,
                                                             db, h);
  return cudaGetLastError();
}

// Row-grouped products of one expert set: C[rows of g] (+)= A[rows of g] op(W[g]).
//   w_kmajor: W[g] stored [N, K] (nn.Linear [out, in]: x W^T); else stored [K, N] (dY W).
cudaError_t rows_gemm(const float* A, int K, const float* W, bool w_kmajor, int N,
                      const int32_t* off, int G, int64_t rows, float* C, bool accumulate,
                      cudaStream_t s) {
  F32Gemm p{};
  p.A = A; p.a_g = 0; p.a_i = K; p.a_k = 1;
  p.B = W; p.b_g = (int64_t)N * K;
  p.b_k = w_kmajor ? 1 : N;
  p.b_j = w_kmajor ? K : 1;
  p.C = C; p.c_g = 0; p.c_i = N; p.c_j = 1;
  p.M = (int)rows; p.N = N; p.K = K; p.off = off; p.kred = 0; p.accumulate = accumulate;
  return gemm_f32(p, G, rows, s);
}

// Per-group reductions over the group's rows: dW[g] (M x N) = L[rows of g]^T R[rows of g],
// L [rows, M], R [rows, N].
cudaError_t kred_gemm(const float* L, int M, const float* R, int N, const int32_t* off, int G,
                      int64_t rows, float* dW, cudaStream_t s) {
  F32Gemm p{};
  p.A = L; p.a_g = 0; p.a_i = 1; p.a_k = M;
  p.B = R; p.b_g = 0; p.b_k = N; p.b_j = 1;
  p.C = dW; p.c_g = (int64_t)M * N; p.c_i = N; p.c_j = 1;
  p.M = M; p.N = N; p.K = (int)rows; p.off = off; p.kred = 1; p.accumulate = 0;
  return gemm_f32(p, G, M, s);
}

}  // namespace

size_t backward_f32_workspace(const moe_desc_t& d, int64_t A) {
  const int64_t T = d.T, D = d.D, E = d.E, F = d.F, S = d.n_shared, Fs = d.F_shared;
  const int64_t K = d.select == MOE_EXPERT_CHOICE ? E : d.k;
  auto up = [](int64_t v) { return (size_t)((v * 4 + 255) / 256 * 256); };
  size_t b = up(A * D) * 2 /* dY, dXp */ + up(T * K) + up(T * E) + up(A * F) * 5 /* a b dH da db */;
  if (S) b += up(T * Fs) * 6 /* a b dH da db h */ + up(S * T * D);
  return b;
}

cudaError_t launch_backward_f32(const moe_desc_t& d, const moe_layer_views_t& v,
                                const float* x, const float* Wg, const float* W_gate,
                                const float* W_up, const float* W_down,
                                const moe_bwd_shared_t* sh, const float* dout, float aux_grad,
                                float* dx, float* dWg, float* dW_gate, float* dW_up,
                                float* dW_down, void* ws, cudaStream_t s) {
  const int64_t T = d.T, D = d.D, E = d.E, F = d.F, S = d.n_shared, Fs = d.F_shared;
  const int K = d.select == MOE_EXPERT_CHOICE ? d.E : d.k;
  const int64_t A = v.rows;
  const bool glu = d.act == MOE_ACT_SWIGLU;
  uint8_t* p = static_cast<uint8_t*>(ws);
  auto take = [&](int64_t n) {
    float* r = reinterpret_cast<float*>(p);
    p += (size_t)((n * 4 + 255) / 256 * 256);
    return r;
  };
  float* dY = take(A * D);
  float* dXp = take(A * D);
  float* dgates = take(T * K);
  float* ds = take(T * E);
  float* pa = take(A * F);
  float* pb = take(A * F);
  float* dH = take(A * F);
  float* da = take(A * F);
  float* db = take(A * F);
  const float* xp = static_cast<const float*>(v.x_perm);
  const float* h = static_cast<const float*>(v.h);
  const int32_t* off = v.offsets;
  // dY = g dout, dg = <dout, y>
  cudaError_t e = cudaSuccess;
  if (A > 0) {
    gather_dy_f32_kernel<<<counted((unsigned)((A + 7) / 8)), 256, 0, s>>>(
        dout, static_cast<const float*>(v.y), v.row_src, v.gates, off, (int)E, K, (int)D, A,
        dY, dgates);
    e = cudaGetLastError();
  }
  // pre-activations a = x_perm W_gate^T, b (or z) = x_perm W_up^T
  if (e == cudaSuccess && glu) e = rows_gemm(xp, D, W_gate, true, F, off, E, A, pa, false, s);
  if (e == cudaSuccess) e = rows_gemm(xp, D, W_up, true, F, off, E, A, glu ? pb : pa, false, s);
  // dH = dY W_down (W_down[e] stored [D, F])
  if (e == cudaSuccess) e = rows_gemm(dY, D, W_down, false, F, off, E, A, dH, false, s);
  if (e == cudaSuccess)
    e = act_backward_f32(d.act, dH, pa, pb, off + E, A, F, da, db, nullptr, s);
  // dX = da W_gate + db W_up (or dz W_up); W_gate[e], W_up[e] stored [F, D]
  if (e == cudaSuccess)
    e = rows_gemm(da, F, glu ? W_gate : W_up, false, D, off, E, A, dXp, false, s);
  if (e == cudaSuccess && glu) e = rows_gemm(db, F, W_up, false, D, off, E, A, dXp, true, s);
  // router: ds, then dW_g = ds^T x (one group over all tokens)
  if (e == cudaSuccess)
    e = launch_router_backward(d, v.logits, v.expert_ids, v.gates, dgates, v.inv, v.f, aux_grad,
                               ds, s);
  if (e == cudaSuccess) e = kred_gemm(ds, E, x, D, nullptr, 1, T, dWg, s);
  // weight gradients per expert over its rows
  if (e == cudaSuccess) e = kred_gemm(dY, D, h, F, off, E, A, dW_down, s);
  if (e == cudaSuccess && glu) e = kred_gemm(da, F, xp, D, off, E, A, dW_gate, s);
  if (e == cudaSuccess) e = kred_gemm(glu ? db : da, F, xp, D, off, E, A, dW_up, s);
  // shared experts: one group of all T tokens each, dY = dout
  float* dXs = nullptr;
  if (e == cudaSuccess && S > 0) {
    float* sa = take(T * Fs);
    float* sb = take(T * Fs);
    float* sdH = take(T * Fs);
    float* sda = take(T * Fs);
    float* sdb = take(T * Fs);
    float* shh = take(T * Fs);
    dXs = take(S * T * D);
    const int64_t wst = Fs * D;
    for (int64_t i = 0; i < S && e == cudaSuccess; ++i) {
      const float* wg = static_cast<const float*>(sh->Ws_gate) + i * wst;
      const float* wu = static_cast<const float*>(sh->Ws_up) + i * wst;
      const float* wd = static_cast<const float*>(sh->Ws_down) + i * wst;
      e = rows_gemm(x, D, wg, true, Fs, nullptr, 1, T, sa, false, s);
      if (e == cudaSuccess) e = rows_gemm(x, D, wu, true, Fs, nullptr, 1, T, sb, false, s);
      if (e == cudaSuccess) e = rows_gemm(dout, D, wd, false, Fs, nullptr, 1, T, sdH, false, s);
      if (e == cudaSuccess)
        e = act_backward_f32(MOE_ACT_SWIGLU, sdH, sa, sb, nullptr, T, Fs, sda, sdb, shh, s);
      float* dxs = dXs + i * T * D;
      if (e == cudaSuccess) e = rows_gemm(sda, Fs, wg, false, D, nullptr, 1, T, dxs, false, s);
      if (e == cudaSuccess) e = rows_gemm(sdb, Fs, wu, false, D, nullptr, 1, T, dxs, true, s);
      if (e == cudaSuccess) e = kred_gemm(dout, D, shh, Fs, nullptr, 1, T, sh->dWs_down + i * wst, s);
      if (e == cudaSuccess) e = kred_gemm(sda, Fs, x, D, nullptr, 1, T, sh->dWs_gate + i * wst, s);
      if (e == cudaSuccess) e = kred_gemm(sdb, Fs, x, D, nullptr, 1, T, sh->dWs_up + i * wst, s);
    }
  }
  if (e == cudaSuccess && T > 0) {
    dx_f32_kernel<<<counted((unsigned)T), 128, 0, s>>>(dXp, v.inv, ds, Wg, (int)T, (int)D, (int)E,
                                                       K, dXs, (int)S, dx);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace moe
