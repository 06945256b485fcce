// Backward pass of the MoE layer with the selection held fixed (bf16 operands, fp32 math):
// token choice or expert choice, with or without shared experts.
//
// "Top-k 路由（Top-k Routing）" (compassingai), "門控網路的梯度流": the discrete top-k is not
// differentiated; the selected experts' gate scores carry the gradient (softmax normalised over
// the selected logits), unselected experts get none from the gates.
// "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife),
// section 9: total loss = task loss + weight x router aux loss; the selected experts' gate /
// up / down matrices and the selected route weights get task-loss gradients, the soft
// importance gets the balance-loss gradient, the expert indices are fixed integers.
//
// With L = <dout, out> + aux_grad * aux, per kept assignment (t, j) -> row r:
//   dY[r] = g[t,j] dout[t],  dg[t,j] = <dout[t], y[r]>;
// experts (rows of expert e):  dH = dY W_down,  (SwiGLU) da = dH b SiLU'(a), db = dH SiLU(a),
//   dX = da W_gate + db W_up,  dW_down = dY^T h,  dW_gate = da^T x,  dW_up = db^T x;
// router: ds from dg through the merge weights, plus the balance-loss term through P;
//   dW_g = ds^T x,  dx[t] = sum_j dX[r(t, j)] + ds[t] W_g.
// The big products run on the tcgen05 grouped GEMM: dgrad reads the weights as stored, an
// MN-major B operand (or K-major transposed copies when MOE_BWD_WEIGHT_TRANSPOSE=1), wgrad runs
// with groups along K over per-expert row blocks transposed and zero-padded to 64.
// This file holds the memory-bound pieces.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kPad = 64;    // k-block of the weight-gradient GEMM: expert row blocks pad to it

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}

// pad_off[e] = sum over e' < e of the expert row counts rounded up to kPad.
__global__ void pad_offsets_kernel(const int32_t* offsets, int E, int32_t* pad_off) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    int acc = 0;
    pad_off[0] = 0;
    for (int e = 0; e < E; ++e) {
      const int c = offsets[e + 1] - offsets[e];
      acc += (c + kPad - 1) / kPad * kPad;
      pad_off[e + 1] = acc;
    }
  }
}

// One warp per executed row r: dY[r] = g dout[t] (bf16) and dg = <dout[t], y[r]> (fp32).
__global__ void gather_dy_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ y,
                                 const int32_t* __restrict__ row_src,
                                 const float* __restrict__ gates,
                                 const int32_t* __restrict__ offsets, int E, int K, int D,
                                 int64_t rows_max, uint4* __restrict__ dY,
                                 float* __restrict__ dgates) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows_max || r >= offsets[E]) return;
  const int src = row_src[r];
  const int t = src / K;
  const float g = gates[src];
  const int nv = D / 8;
  float dot = 0.f;
  for (int v = lane; v < nv; v += 32) {
    float a[8], b[8], o[8];
    unpack8(dout[(int64_t)t * nv + v], a);
    unpack8(y[r * nv + v], b);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dot += a[i] * b[i];
      o[i] = g * a[i];
    }
    dY[r * nv + v] = pack8(o);
  }
  dot = warp_sum_f(dot);
  if (lane == 0) dgates[src] = dot;
}

// Activation backward on the executed rows, 8 features per thread.
//   SwiGLU (ACT 0): gu row = blocks of [128 gate | 128 up] per 128 features (pitch ldg);
//                   dAB row = [da (F) | db (F)]; with h_out also h = SiLU(a) b (bf16 [rows, F]).
//   ReLU (1), GELU (2): gu = z [rows, F]; dAB = dz [rows, F].
template <int ACT>
__global__ void act_backward_kernel(const uint4* __restrict__ dH, const __nv_bfloat16* __restrict__ gu,
                                    const int32_t* __restrict__ offsets, int E, int F,
                                    int64_t ldg, int64_t rows_max, __nv_bfloat16* __restrict__ dAB,
                                    __nv_bfloat16* __restrict__ h_out) {
  const int nv = F / 8;
  const int64_t rows = min((int64_t)offsets[E], rows_max);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * nv;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / nv;
    const int f = (int)(i - r * nv) * 8;
    float dh[8];
    unpack8(dH[i], dh);
    if (ACT == 0) {
      const int64_t gcol = (int64_t)(f / 128) * 256 + (f % 128);
      float a[8], b[8], da[8], db[8], hv[8];
      unpack8(*reinterpret_cast<const uint4*>(gu + r * ldg + gcol), a);
      unpack8(*reinterpret_cast<const uint4*>(gu + r * ldg + gcol + 128), b);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float s = 1.0f / (1.0f + expf(-a[k]));
        da[k] = dh[k] * b[k] * (s * (1.0f + a[k] * (1.0f - s)));
        db[k] = dh[k] * a[k] * s;
        hv[k] = a[k] * s * b[k];
      }
      *reinterpret_cast<uint4*>(dAB + r * 2 * F + f) = pack8(da);
      *reinterpret_cast<uint4*>(dAB + r * 2 * F + F + f) = pack8(db);
      if (h_out) *reinterpret_cast<uint4*>(h_out + r * F + f) = pack8(hv);
    } else {
      float z[8], dz[8];
      unpack8(*reinterpret_cast<const uint4*>(gu + r * ldg + f), z);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float d;
        if (ACT == 1) {
          d = z[k] > 0.f ? 1.f : 0.f;
        } else {
          d = 0.5f * (1.0f + erff(z[k] * 0.70710678118654752f)) +
              z[k] * expf(-0.5f * z[k] * z[k]) * 0.39894228040143268f;
        }
        dz[k] = dh[k] * d;
      }
      *reinterpret_cast<uint4*>(dAB + r * F + f) = pack8(dz);
    }
  }
}

// 64 x 64 bf16 tile transpose, 256 threads: 16-byte global loads along the source rows and
// 16-byte global stores along the destination rows, scalar accesses to a shared tile of pitch
// 65 elements (spreads a column read over the banks).
//   plain (PAD = false): dst[b][c][dcol0 + r] = src[b][r][c], r < R, c < C;
//   padded (PAD = true): dst[c][j] for the 64-column block j0.. inside expert e's padded block:
//     src row offsets[e] + (j - pad_off[e]) when that is below offsets[e + 1], else 0.
template <bool PAD>
__global__ void __launch_bounds__(256)
transpose64_kernel(const __nv_bfloat16* __restrict__ src, int64_t src_bstride, int R, int C,
                   int64_t lds, __nv_bfloat16* __restrict__ dst, int64_t dst_bstride,
                   int64_t ldd, int dcol0, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ pad_off, int E) {
  __shared__ __nv_bfloat16 tile[64][65];
  const int c0 = blockIdx.y * 64;
  int r0 = blockIdx.x * 64, j0 = r0, rlim = R;
  const __nv_bfloat16* s = src + (int64_t)blockIdx.z * src_bstride;
  __nv_bfloat16* d = dst + (int64_t)blockIdx.z * dst_bstride;
  if (PAD) {
    if (j0 >= pad_off[E]) return;
    int lo = 0, hi = E;                      // expert e with pad_off[e] <= j0 < pad_off[e + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pad_off[mid] <= j0) lo = mid; else hi = mid;
    }
    r0 = offsets[lo] + (j0 - pad_off[lo]);   // first source row of the tile
    rlim = offsets[lo + 1];                  // rows from rlim on are padding
  }
  const int tid = threadIdx.x;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int idx = tid + 256 * k;
    const int row = idx >> 3, cv = (idx & 7) * 8;
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (r0 + row < rlim && c0 + cv < C)
      u = *reinterpret_cast<const uint4*>(s + (int64_t)(r0 + row) * lds + c0 + cv);
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
    for (int i = 0; i < 8; ++i) tile[row][cv + i] = h[i];
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int idx = tid + 256 * k;
    const int col = idx >> 3, rv = (idx & 7) * 8;
    if (c0 + col >= C) continue;
    if (!PAD && r0 + rv >= R) continue;
    uint4 u;
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(&u);
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = tile[rv + i][col];
    if (PAD) {
      *reinterpret_cast<uint4*>(d + (int64_t)(c0 + col) * ldd + j0 + rv) = u;
    } else if (r0 + rv + 8 <= R) {
      *reinterpret_cast<uint4*>(d + (int64_t)(c0 + col) * ldd + dcol0 + r0 + rv) = u;
    } else {
      for (int i = 0; r0 + rv + i < R; ++i) d[(int64_t)(c0 + col) * ldd + dcol0 + r0 + rv + i] = h[i];
    }
  }
}

// One warp per token: ds[t, :] = dL/ds from the merge-weight gradients (selection fixed) plus
// the balance-loss term.  Lane l holds experts l + 32 i.  Under expert choice (ec) the merge
// weight of a picked (token, expert) pair is the softmax probability itself: the raw-gate form
// with K = E slots, slot j being expert j ("Top-k 路由" Token-Choice vs Expert-Choice table).
constexpr int kMaxEL = 8;   // E <= 256
__global__ void router_backward_kernel(const float* __restrict__ logits,
                                       const int32_t* __restrict__ ids,
                                       const float* __restrict__ gates,
                                       const float* __restrict__ dgates,
                                       const int32_t* __restrict__ inv,
                                       const float* __restrict__ f, int T, int E, int K,
                                       int sigmoid_score, int renorm, int ec, float aux_coef,
                                       float* __restrict__ ds) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  float s[kMaxEL], w[kMaxEL], d[kMaxEL];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxEL; ++i) {
    const int e = lane + 32 * i;
    s[i] = e < E ? logits[(int64_t)t * E + e] : -INFINITY;
    m = fmaxf(m, s[i]);
    d[i] = 0.f;
  }
  // w: softmax probabilities or sigmoid affinities
  float wsum = 0.f;
  if (!sigmoid_score) {
    float mm = m;                            // warp max of the logits
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
#pragma unroll
    for (int i = 0; i < kMaxEL; ++i) {
      w[i] = (lane + 32 * i < E) ? expf(s[i] - mm) : 0.f;
      wsum += w[i];
    }
    wsum = warp_sum_f(wsum);
#pragma unroll
    for (int i = 0; i < kMaxEL; ++i) w[i] /= wsum;
  } else {
#pragma unroll
    for (int i = 0; i < kMaxEL; ++i) {
      w[i] = (lane + 32 * i < E) ? 1.0f / (1.0f + expf(-s[i])) : 0.f;
      wsum += w[i];
    }
    wsum = warp_sum_f(wsum);
  }
  // merge-weight gradients of the kept assignments; dot = sum_j g_j dg_j, sel = sum_sel w
  float dot = 0.f, selw = 0.f;
  for (int j = 0; j < K; ++j) {
    const int64_t a = (int64_t)t * K + j;
    const float dg = inv[a] >= 0 ? dgates[a] : 0.f;
    dot += gates[a] * dg;
    const int e = ec ? j : ids[a];           // expert choice: slot j of a token is expert j
#pragma unroll
    for (int i = 0; i < kMaxEL; ++i)
      if (lane + 32 * i == e) selw += w[i];
  }
  selw = warp_sum_f(selw);
  for (int j = 0; j < K; ++j) {
    const int64_t a = (int64_t)t * K + j;
    const float dg = inv[a] >= 0 ? dgates[a] : 0.f;
    const int e = ec ? j : ids[a];
#pragma unroll
    for (int i = 0; i < kMaxEL; ++i) {
      if (lane + 32 * i != e) continue;
      if (!sigmoid_score) {
        // renorm: g = softmax over the selected logits -> ds_e = g_e (dg_e - dot)
        // raw: g = p_e -> dp_e = dg_e (the softmax Jacobian is applied below)
        d[i] += renorm ? gates[a] * (dg - dot) : dg;
      } else {
        // renorm: da_e = (dg_e - dot) / sum_sel a; raw: da_e = dg_e
        d[i] += renorm ? (dg - dot) / selw : dg;
      }
    }
  }
  // d holds: softmax+renorm -> ds (final gate part); softmax+raw -> dp; sigmoid -> da
  float out[kMaxEL];
  if (!sigmoid_score) {
    // balance loss: dp_e += aux_coef f_e, then ds = p (dp - <p, dp>) for the dp parts
    float pd = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxEL; ++i) {
      const int e = lane + 32 * i;
      const float dp = (renorm ? 0.f : d[i]) + (e < E ? aux_coef * f[e] : 0.f);
      out[i] = dp;
      pd += w[i] * dp;
    }
    pd = warp_sum_f(pd);
#pragma unroll
    for (int i = 0; i < kMaxEL; ++i)
      out[i] = w[i] * (out[i] - pd) + (renorm ? d[i] : 0.f);
  } else {
    // balance loss through q = a / sum a: da_e += (dq_e - <q, dq>) / sum a, dq_e = aux_coef f_e
    float qd = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxEL; ++i) {
      const int e = lane + 32 * i;
      qd += (w[i] / wsum) * (e < E ? aux_coef * f[e] : 0.f);
    }
    qd = warp_sum_f(qd);
#pragma unroll
    for (int i = 0; i < kMaxEL; ++i) {
      const int e = lane + 32 * i;
      const float da = d[i] + ((e < E ? aux_coef * f[e] : 0.f) - qd) / wsum;
      out[i] = da * w[i] * (1.0f - w[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxEL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) ds[(int64_t)t * E + e] = out[i];
  }
}

// dx[t] = sum_j dX[inv[t, j]] (fixed slot order) + sum_e ds[t, e] W_g[e] + sum_i dXs[i][t] (the
// shared experts' input gradients, when given); one block per token, 8 columns per thread.
__global__ void dx_kernel(const uint4* __restrict__ dX, const int32_t* __restrict__ inv,
                          const float* __restrict__ ds, const uint4* __restrict__ Wg, int T,
                          int D, int E, int K, const uint4* __restrict__ dXs, int n_add,
                          uint4* __restrict__ dx) {
  extern __shared__ float s_ds[];
  const int t = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_ds[e] = ds[(int64_t)t * E + e];
  __syncthreads();
  const int nv = D / 8;
  for (int v = threadIdx.x; v < nv; v += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < K; ++j) {
      const int r = inv[(int64_t)t * K + j];
      if (r < 0) continue;
      float a[8];
      unpack8(dX[(int64_t)r * nv + v], a);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += a[i];
    }
    for (int e = 0; e < E; ++e) {
      float wv[8];
      unpack8(Wg[(int64_t)e * nv + v], wv);
      const float c = s_ds[e];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += c * wv[i];
    }
    for (int j = 0; j < n_add; ++j) {        // shared experts' input gradients
      float a[8];
      unpack8(dXs[((int64_t)j * T + t) * nv + v], a);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += a[i];
    }
    dx[(int64_t)t * nv + v] = pack8(acc);
  }
}

// dW_g partials: part[chunk][e][d] = sum over the chunk's tokens (in order) of ds[t, e] x[t, d];
// thread per column d, experts 8 at a time.
constexpr int kDwgChunk = 128;
__global__ void dwg_partial_kernel(const float* __restrict__ ds,
                                   const __nv_bfloat16* __restrict__ x, int T, int D, int E,
                                   float* __restrict__ part) {
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  const int chunk = blockIdx.y;
  const int t0 = chunk * kDwgChunk, t1 = min(T, t0 + kDwgChunk);
  if (d >= D) return;
  for (int e0 = 0; e0 < E; e0 += 8) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int t = t0; t < t1; ++t) {
      const float xv = __bfloat162float(x[(int64_t)t * D + d]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (e0 + i < E) acc[i] += ds[(int64_t)t * E + e0 + i] * xv;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (e0 + i < E) part[((int64_t)chunk * E + e0 + i) * D + d] = acc[i];
  }
}

__global__ void dwg_reduce_kernel(const float* __restrict__ part, int n_chunks, int64_t n,
                                  float* __restrict__ dWg) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < n_chunks; ++c) acc += part[(int64_t)c * n + i];
    dWg[i] = acc;
  }
}

int grid_of(int64_t work, int per_block) {
  int64_t b = (work + per_block - 1) / per_block;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (b > cap) b = cap;
  return b > 0 ? (int)b : 1;
}

}  // namespace

int backward_dwg_chunks(int T) { return (T + kDwgChunk - 1) / kDwgChunk; }

cudaError_t launch_pad_offsets(const int32_t* offsets, int E, int32_t* pad_off, cudaStream_t s) {
  pad_offsets_kernel<<<counted(1), 32, 0, s>>>(offsets, E, pad_off);
  return cudaGetLastError();
}

cudaError_t launch_gather_dy(const void* dout, const void* y, const int32_t* row_src,
                             const float* gates, const int32_t* offsets, int E, int K, int D,
                             int64_t rows_max, void* dY, float* dgates, cudaStream_t s) {
  if (rows_max <= 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (rows_max + warps - 1) / warps;
  gather_dy_kernel<<<counted((unsigned)blocks), warps * 32, 0, s>>>(
      static_cast<const uint4*>(dout), static_cast<const uint4*>(y), row_src, gates, offsets, E,
      K, D, rows_max, static_cast<uint4*>(dY), dgates);
  return cudaGetLastError();
}

cudaError_t launch_act_backward(int act, const void* dH, const void* gu, int64_t ldg,
                                const int32_t* offsets, int E, int F, int64_t rows_max,
                                void* dAB, cudaStream_t s, void* h_out) {
  if (rows_max <= 0) return cudaSuccess;
  const int grid = grid_of(rows_max * (F / 8), 256);
  const uint4* h = static_cast<const uint4*>(dH);
  const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(gu);
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(dAB);
  __nv_bfloat16* ho = static_cast<__nv_bfloat16*>(h_out);
  if (act == MOE_ACT_SWIGLU)
    act_backward_kernel<0><<<counted(grid), 256, 0, s>>>(h, g, offsets, E, F, ldg, rows_max, o,
                                                         ho);
  else if (act == MOE_ACT_RELU)
    act_backward_kernel<1><<<counted(grid), 256, 0, s>>>(h, g, offsets, E, F, ldg, rows_max, o,
                                                         nullptr);
  else
    act_backward_kernel<2><<<counted(grid), 256, 0, s>>>(h, g, offsets, E, F, ldg, rows_max, o,
                                                         nullptr);
  return cudaGetLastError();
}

cudaError_t launch_transpose(const void* src, int64_t src_bstride, int R, int C, int64_t lds,
                             void* dst, int64_t dst_bstride, int64_t ldd, int dcol0, int batch,
                             cudaStream_t s) {
  if (R <= 0 || C <= 0 || batch <= 0) return cudaSuccess;
  const dim3 grid((R + 63) / 64, (C + 63) / 64, batch);
  transpose64_kernel<false><<<counted(grid), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(src), src_bstride, R, C, lds,
      static_cast<__nv_bfloat16*>(dst), dst_bstride, ldd, dcol0, nullptr, nullptr, 0);
  return cudaGetLastError();
}

cudaError_t launch_transpose_pad(const void* src, int64_t lds, int C, const int32_t* offsets,
                                 const int32_t* pad_off, int E, int64_t pad_cols, void* dst,
                                 int64_t ldd, cudaStream_t s) {
  if (C <= 0 || pad_cols <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((pad_cols + 63) / 64), (C + 63) / 64, 1);
  transpose64_kernel<true><<<counted(grid), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(src), 0, 0, C, lds, static_cast<__nv_bfloat16*>(dst), 0,
      ldd, 0, offsets, pad_off, E);
  return cudaGetLastError();
}

cudaError_t launch_router_backward(const moe_desc_t& d, const float* logits, const int32_t* ids,
                                   const float* gates, const float* dgates, const int32_t* inv,
                                   const float* f, float aux_grad, float* ds, cudaStream_t s) {
  if (d.T <= 0) return cudaSuccess;
  const int warps = 8;
  const float coef = aux_grad * d.aux_alpha * (float)d.E / (float)d.T;
  const bool ec = d.select == MOE_EXPERT_CHOICE;
  router_backward_kernel<<<counted((d.T + warps - 1) / warps), warps * 32, 0, s>>>(
      logits, ids, gates, dgates, inv, f, d.T, d.E, ec ? d.E : d.k,
      d.score == MOE_SCORE_SIGMOID ? 1 : 0, (!ec && d.gate == MOE_GATE_RENORM) ? 1 : 0,
      ec ? 1 : 0, coef, ds);
  return cudaGetLastError();
}

cudaError_t launch_dx(const void* dX, const int32_t* inv, const float* ds, const void* Wg, int T,
                      int D, int E, int K, void* dx, cudaStream_t s, const void* dXs,
                      int n_add) {
  if (T <= 0) return cudaSuccess;
  dx_kernel<<<counted(T), 256, E * sizeof(float), s>>>(
      static_cast<const uint4*>(dX), inv, ds, static_cast<const uint4*>(Wg), T, D, E, K,
      static_cast<const uint4*>(dXs), dXs ? n_add : 0, static_cast<uint4*>(dx));
  return cudaGetLastError();
}

cudaError_t launch_dwg(const float* ds, const void* x, int T, int D, int E, float* part,
                       float* dWg, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int chunks = backward_dwg_chunks(T);
  dwg_partial_kernel<<<counted(dim3((D + 255) / 256, chunks)), 256, 0, s>>>(
      ds, static_cast<const __nv_bfloat16*>(x), T, D, E, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = (int64_t)E * D;
  dwg_reduce_kernel<<<counted(grid_of(n, 256)), 256, 0, s>>>(part, chunks, n, dWg);
  return cudaGetLastError();
}

}  // namespace moe
