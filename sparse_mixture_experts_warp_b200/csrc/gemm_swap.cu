// Grouped GEMM with the weights as the MMA's M side and the tokens as its N side (sm_100a): an
// alternative schedule to the row tiles of grouped_gemm_kernel, selected by MOE_GEMM_SWAP=1.
//
// The products are those of grouped_gemm_kernel (gemm_sm100.cu): "从 Dense FFN 到 MoE：用一个
// Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife), section 3 (SwiGLU expert:
// hidden = SiLU(x W_gate) * (x W_up), output = hidden W_down; ReLU / GELU experts) and section 12
// (token permutation + grouped GEMM); "别只比较 Top-k" (ailearn moe-comparison), the Execute step
// and the expert-work account (with many experts each one receives a few rows, so its weights
// are read for little arithmetic).
//
// out[r, n] = epi( sum_k A[r, k] * B[g*N + n, k] ) for the rows r of group g, as there.  With
// hundreds of experts and top-k routing a group holds a few dozen to a few hundred rows, unevenly
// (DeepSeek-V3 shape: 32768 rows over 256 experts).  Row tiles of 128 (or 64) rows then run
// partly empty MMAs for every started block of rows, and every row tile reads the weight tile
// again.  This kernel puts the weights on the MMA's M side and the tokens on its N side:
//   D[f, t] = sum_k B[g*N + f, k] * A[row0 + t, k]   (TMEM lane = feature, column = token)
// A tile is 256 weight rows (two M=128 MMAs that share the token operand) by up to 256 tokens of
// one group, and the MMAs' N is the tile's token count rounded up to 16.  Per 64-element k-block
// a stage holds 32 KB of weights and 128 B per token row.
//   EPI_SWIGLU: the two MMAs take the same 128 features of W_gate (TMEM columns [0, 256)) and of
//               W_up (columns [256, 512)), so gate and up of a feature sit in one TMEM lane;
//               out = SiLU(gate) * up;
//   EPI_RELU, EPI_GELU, EPI_NONE: 256 consecutive output features, two halves of 128.
// Roles (one persistent CTA per SM, tiles taken round-robin; tiles are enumerated group by
// group, feature tile by feature tile, token tiles innermost, so the CTAs that run together
// share weight tiles through L2):
//   warp 0      TMA producer: two 128 x 64 weight boxes and the token rows (32-row boxes, or
//               4-row gathers by index straight from the token tensor) into a 3-stage ring of
//               64 KB, mbarrier complete_tx; no multicast;
//   warp 1      MMA issuer (tcgen05.mma.cta_group::1.kind::f16, fp32 accumulators in 512 TMEM
//               columns) and owner of the TMEM allocation;
//   warps 2..9  epilogue: tcgen05.ld 32x32b (warp w reads TMEM lanes 32 (w % 4) .. +31, one
//               output feature per thread), activation, one bf16 store per token: a warp
//               writes 64 contiguous bytes of an output row.
// Rows past the group end inside a token box belong to the next group (or are zero-filled past
// the tensor): they only feed accumulator columns that the epilogue discards.  Every mbarrier
// wait is bounded (globaltimer); a wait that gives up records an error code in the device
// error word and the CTA drains what it has in flight and exits.
// Measured against the row tiles (B200, bf16): slower at the DeepSeek-V3 shape (up projection
// 2.94 against 2.51 ms) and at the Mixtral shape (1.81 against 1.60 ms), faster only for the
// expert-choice down projection (160 against 175 us: full 256-token tiles, a short K, and
// 64-byte store segments).  Each M=128 MMA reads its 128 x 16 weight slice (4 KB) from shared
// memory whatever its N: at N tokens it needs 8192 / N + 64 bytes per clock, more than the
// SM's 128 below N = 128, while the row tiles always run N = 256 (96 bytes per clock).
#include <cuda.h>

#include "common.cuh"
#include "mbar.cuh"
#include "tc_ops.cuh"

namespace moe {
namespace {

constexpr int SW_KB = 64;                           // k elements per stage
constexpr int SW_MMA_K = 16;
constexpr int SW_WROWS = 128;                       // weight rows per MMA (M)
constexpr int SW_TOK = 256;                         // tokens per tile (largest N)
constexpr int SW_WH_BYTES = SW_WROWS * SW_KB * 2;   // one 128-row weight box
constexpr int SW_W_BYTES = 2 * SW_WH_BYTES;
constexpr int SW_X_BYTES = SW_TOK * SW_KB * 2;
constexpr int SW_STAGE = SW_W_BYTES + SW_X_BYTES;   // 64 KB
constexpr int SW_STAGES = 3;
constexpr int SW_XBOX = 32;                         // token rows per tiled box
constexpr int SW_XBOX_BYTES = SW_XBOX * SW_KB * 2;
constexpr int SW_ROW_BYTES = SW_KB * 2;
constexpr int SW_EPI_WARPS = 8;
constexpr int SW_THREADS = 64 + 32 * SW_EPI_WARPS;
constexpr int SW_TMEM_COLS = 512;
constexpr int SW_HALF_COLS = 256;
constexpr uint64_t SW_TIMEOUT_NS = 2000000000ull;   // 2 s per wait
constexpr uint64_t SW_DRAIN_NS = 200000000ull;      // 0.2 s to drain after an abort

struct SwapParams {
  const int32_t* offsets;   // [G+1] device
  __nv_bfloat16* out;       // [rows, N]
  int* err;                 // device error word
  int64_t rows;             // rows allocated in A and out
  int G, N, K;
  int feat_tile;            // output features per tile: 128 (SwiGLU) or 256
  int nt;                   // feature tiles per group
  int fault;                // test hook: 1 = CTA 0 arms its first stage without loading it
  const int32_t* gather_src;   // gather: row r of the grouped operand is token gather_src[r] / div
  int gather_div;
};

struct SwTile {
  int g, f_idx, ntok;
  int row0;                 // first grouped row of the tile
};

// Work item t (group, then feature tile, token tile innermost); g caches the group search.
__device__ __forceinline__ SwTile sw_locate(int t, const int* grp_off, const int* tile_pre,
                                            int& g) {
  if (t < tile_pre[g]) g = 0;
  while (t >= tile_pre[g + 1]) ++g;
  const int m = grp_off[g + 1] - grp_off[g];
  const int mt = (m + SW_TOK - 1) / SW_TOK;
  const int local = t - tile_pre[g];
  SwTile r;
  r.g = g;
  r.f_idx = local / mt;
  const int j = local - r.f_idx * mt;
  r.ntok = min(SW_TOK, m - j * SW_TOK);
  r.row0 = grp_off[g] + j * SW_TOK;
  return r;
}

__device__ __forceinline__ int round16(int n) { return (n + 15) & ~15; }

template <int EPI>
__device__ __forceinline__ float sw_act(float a) {
  if (EPI == EPI_RELU) return fmaxf(a, 0.f);
  if (EPI == EPI_GELU) return 0.5f * a * (1.0f + erff(a * 0.70710678118654752f));
  return a;
}

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(SW_THREADS, 1)
grouped_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmX,
                         const __grid_constant__ CUtensorMap tmW0,
                         const __grid_constant__ CUtensorMap tmW1, const SwapParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);   // stage s: weights, then tokens, at sbase + s * SW_STAGE
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SW_STAGES * SW_STAGE);
  uint64_t* full = bars;
  uint64_t* empty = bars + SW_STAGES;
  uint64_t* tfull = bars + 2 * SW_STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* grp_off = reinterpret_cast<int*>(tmem_holder + 2);   // [G+1]
  int* tile_pre = grp_off + (p.G + 1);                      // [G+1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SW_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, SW_EPI_WARPS * 32);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW0)) : "memory");
    if (EPI == EPI_SWIGLU)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW1)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(SW_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // the set-up above touches this CTA's own memories only; the group table and the operands
  // were written by earlier kernels
  pdl_trigger();
  pdl_wait();
  if (warp == 2) {
    // group row starts and the tile prefix (tiles of group g = ceil(rows_g / 256) * nt)
    int carry = 0;
    if (lane == 0) {
      grp_off[0] = p.offsets[0];
      tile_pre[0] = 0;
    }
    for (int g0 = 0; g0 < p.G; g0 += 32) {
      const int g = g0 + lane;
      int tiles = 0;
      if (g < p.G) {
        const int lo = p.offsets[g], hi = p.offsets[g + 1];
        const int m = hi > lo ? hi - lo : 0;
        tiles = ((m + SW_TOK - 1) / SW_TOK) * p.nt;
        grp_off[g + 1] = hi;
      }
      int inc = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
      }
      if (g < p.G) tile_pre[g + 1] = carry + inc;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = tile_pre[p.G];
  const int nkb = (p.K + SW_KB - 1) / SW_KB;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // Tiled: lane 0 loads everything.  Gathered: lane 0 waits for a free stage, arms it and
    // loads the weights; lane l loads token rows 8 l .. 8 l + 7 (below the tile's N) with two
    // 4-row gathers, rows past the group end reading token row 0.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, issued_par = 0;     // per stage: has a load, parity of the last one
    bool ok = true;
    int g = 0;
    for (int t = blockIdx.x; t < total && ok && (GATHER || lane == 0); t += gridDim.x) {
      const SwTile tl = sw_locate(t, grp_off, tile_pre, g);
      const int wrow = tl.g * p.N + tl.f_idx * p.feat_tile;
      const int n16 = round16(tl.ntok);
      const int nbox = (tl.ntok + SW_XBOX - 1) / SW_XBOX;
      const uint32_t tx = SW_W_BYTES + (GATHER ? n16 * SW_ROW_BYTES : nbox * SW_XBOX_BYTES);
      int src[8];
      const bool mine = GATHER && 8 * lane < n16;
      if (GATHER) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 8 * lane + i;
          src[i] = (mine && r < tl.ntok) ? __ldg(p.gather_src + tl.row0 + r) / p.gather_div : 0;
        }
      }
      for (int kb = 0; kb < nkb; ++kb) {
        const int kx = kb * SW_KB;
        int go = 1;
        if (lane == 0) {
          go = mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, DEVERR_TIMEOUT_TMA,
                         SW_TIMEOUT_NS);
          if (go) mbar_expect_tx(&full[stage], tx);
        }
        if (GATHER) go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) {
          ok = false;
          break;
        }
        // test hook: the stage is armed but never loaded, so the MMA issuer's bounded wait on
        // it runs out; nothing is in flight for this stage
        const bool withhold =
            p.fault == 1 && blockIdx.x == 0 && t == (int)blockIdx.x && kb == 0;
        const uint32_t w_dst = sbase + stage * SW_STAGE, x_dst = w_dst + SW_W_BYTES;
        if (!withhold) {
          if (lane == 0) {
            if (EPI == EPI_SWIGLU) {
              tma_load_2d(w_dst, &tmW0, &full[stage], kx, wrow);
              tma_load_2d(w_dst + SW_WH_BYTES, &tmW1, &full[stage], kx, wrow);
            } else {
              tma_load_2d(w_dst, &tmW0, &full[stage], kx, wrow);
              tma_load_2d(w_dst + SW_WH_BYTES, &tmW0, &full[stage], kx, wrow + SW_WROWS);
            }
            if (!GATHER)
              for (int b = 0; b < nbox; ++b)
                tma_load_2d(x_dst + b * SW_XBOX_BYTES, &tmX, &full[stage], kx,
                            tl.row0 + b * SW_XBOX);
          }
          if (mine) {
            tma_gather4(x_dst + (8 * lane) * SW_ROW_BYTES, &tmX, &full[stage], kx, src[0],
                        src[1], src[2], src[3]);
            tma_gather4(x_dst + (8 * lane + 4) * SW_ROW_BYTES, &tmX, &full[stage], kx, src[4],
                        src[5], src[6], src[7]);
          }
        }
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == SW_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      // let the copies already in flight land before the CTA exits
      for (int s = 0; s < SW_STAGES; ++s)
        if (issued & (1u << s))
          mbar_wait(&full[s], (issued_par >> s) & 1u, abort_flag, p.err, DEVERR_TIMEOUT_TMA,
                    SW_DRAIN_NS, /*honor_abort=*/false);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0, g = 0;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const SwTile tl = sw_locate(t, grp_off, tile_pre, g);
        const uint32_t idesc = idesc_bf16(SW_WROWS, round16(tl.ntok));
        if (!mbar_wait(tempty, (uint32_t)(it & 1) ^ 1u, abort_flag, p.err, DEVERR_TIMEOUT_MMA,
                       SW_TIMEOUT_NS)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, DEVERR_TIMEOUT_MMA,
                         SW_TIMEOUT_NS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w0 = sbase + stage * SW_STAGE, x0 = w0 + SW_W_BYTES;
#pragma unroll
          for (int k = 0; k < SW_KB / SW_MMA_K; ++k) {
            const uint64_t bdesc = sdesc<SW_KB>(x0 + k * SW_MMA_K * 2);
            const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
            umma_bf16(tmem_base, sdesc<SW_KB>(w0 + k * SW_MMA_K * 2), bdesc, accum, idesc);
            umma_bf16(tmem_base + SW_HALF_COLS,
                      sdesc<SW_KB>(w0 + SW_WH_BYTES + k * SW_MMA_K * 2), bdesc, accum, idesc);
          }
          umma_commit(&empty[stage]);       // frees the stage once these MMAs have read it
          if (++stage == SW_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(tfull);         // accumulators ready for the epilogue
      }
      // all MMAs issued by this thread complete before the CTA releases TMEM
      umma_commit(drain);
      mbar_wait(drain, 0u, abort_flag, p.err, DEVERR_TIMEOUT_MMA, ok ? SW_TIMEOUT_NS : SW_DRAIN_NS,
                /*honor_abort=*/false);
    }
  } else {
    // ---------------- epilogue (warps 2 .. 9) ----------------
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int grp = (warp - 2) >> 2;         // SwiGLU: token chunks grp, grp + 2, ...; else: half
    const uint32_t trow = tmem_base + ((uint32_t)(32 * q) << 16);
    int g = 0, it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const SwTile tl = sw_locate(t, grp_off, tile_pre, g);
      int okw = 1;
      if (lane == 0)
        okw = mbar_wait(tfull, (uint32_t)(it & 1), abort_flag, p.err, DEVERR_TIMEOUT_EPI,
                        SW_TIMEOUT_NS);
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      tc_fence_after();
      bool rows_ok = (int64_t)tl.row0 + tl.ntok <= p.rows;
      if (!rows_ok && lane == 0) atomicCAS(p.err, 0, DEVERR_BOUNDS);
      if (EPI == EPI_SWIGLU) {
        const int feat = tl.f_idx * SW_WROWS + 32 * q + lane;
        const bool st = rows_ok && feat < p.N;
        __nv_bfloat16* o = p.out + (int64_t)tl.row0 * p.N + feat;
#pragma unroll 1
        for (int c = grp; 32 * c < tl.ntok; c += 2) {
          uint32_t gv[32], uv[32];
          tmem_ld32(trow + 32 * c, gv);
          tmem_ld32(trow + SW_HALF_COLS + 32 * c, uv);
          tmem_wait_ld();
          const int nv = tl.ntok - 32 * c;
          if (st) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (i < nv) {
                const float gg = __uint_as_float(gv[i]), uu = __uint_as_float(uv[i]);
                o[(int64_t)(32 * c + i) * p.N] =
                    __float2bfloat16_rn(__fdividef(gg, 1.0f + __expf(-gg)) * uu);
              }
            }
          }
        }
      } else {
        const int feat = tl.f_idx * 2 * SW_WROWS + grp * SW_WROWS + 32 * q + lane;
        const bool st = rows_ok && feat < p.N;
        const uint32_t taddr = trow + (uint32_t)(grp * SW_HALF_COLS);
        __nv_bfloat16* o = p.out + (int64_t)tl.row0 * p.N + feat;
#pragma unroll 1
        for (int c = 0; 32 * c < tl.ntok; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + 32 * c, v);
          tmem_wait_ld();
          const int nv = tl.ntok - 32 * c;
          if (st) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < nv)
                o[(int64_t)(32 * c + i) * p.N] =
                    __float2bfloat16_rn(sw_act<EPI>(__uint_as_float(v[i])));
          }
        }
      }
      // every TMEM read of this tile has completed (tcgen05.wait::ld): release the accumulators
      tc_fence_before();
      mbar_arrive(tempty);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(SW_TMEM_COLS)
                 : "memory");
  }
}

size_t swap_smem(int n_groups) {
  return 1024 + (size_t)SW_STAGES * SW_STAGE + (2 * SW_STAGES + 3) * 8 + 8 +
         (size_t)2 * (n_groups + 1) * sizeof(int);
}

template <int EPI, bool GATHER>
cudaError_t launch_swap_epi(const CUtensorMap& x, const CUtensorMap& w0, const CUtensorMap& w1,
                            const SwapParams& p, int grid, size_t smem, cudaStream_t s) {
  auto kern = grouped_gemm_swap_kernel<EPI, GATHER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(SW_THREADS), smem, s, x, w0, w1, p);
}

template <bool GATHER>
cudaError_t launch_swap_gather(int epi, const CUtensorMap& x, const CUtensorMap& w0,
                               const CUtensorMap& w1, const SwapParams& p, int grid, size_t smem,
                               cudaStream_t s) {
  switch (epi) {
    case EPI_SWIGLU: return launch_swap_epi<EPI_SWIGLU, GATHER>(x, w0, w1, p, grid, smem, s);
    case EPI_RELU: return launch_swap_epi<EPI_RELU, GATHER>(x, w0, w1, p, grid, smem, s);
    case EPI_GELU: return launch_swap_epi<EPI_GELU, GATHER>(x, w0, w1, p, grid, smem, s);
    default: return launch_swap_epi<EPI_NONE, GATHER>(x, w0, w1, p, grid, smem, s);
  }
}

}  // namespace

bool swap_epilogue_ok(int epi) {
  return epi == EPI_SWIGLU || epi == EPI_RELU || epi == EPI_GELU || epi == EPI_NONE;
}

cudaError_t launch_grouped_gemm_swap(int epi, const void* A, int64_t a_rows, int K,
                                     const void* B0, const void* B1, int n_groups, int N,
                                     const int32_t* offsets, void* out, cudaStream_t s,
                                     const int32_t* gather_src, int gather_div, int64_t src_rows,
                                     int fault) {
  if (a_rows <= 0 || n_groups <= 0) return cudaSuccess;
  if (!offsets || !swap_epilogue_ok(epi) || (epi == EPI_SWIGLU && !B1) || N <= 0 || K <= 0)
    return cudaErrorInvalidValue;
  if (gather_src && (gather_div < 1 || src_rows <= 0)) return cudaErrorInvalidValue;
  // tensor-map coordinates are 32-bit
  if (a_rows > INT32_MAX || (int64_t)n_groups * N > INT32_MAX) return cudaErrorInvalidValue;
  alignas(64) CUtensorMap tx, tw0, tw1;
  const uint64_t wrows = (uint64_t)n_groups * (uint64_t)N;
  if (gather_src) {
    if (!make_map(&tx, A, (uint64_t)src_rows, (uint64_t)K, 1, SW_KB)) return cudaErrorInvalidValue;
  } else if (!make_map(&tx, A, (uint64_t)a_rows, (uint64_t)K, SW_XBOX, SW_KB)) {
    return cudaErrorInvalidValue;
  }
  if (!make_map(&tw0, B0, wrows, (uint64_t)K, SW_WROWS, SW_KB)) return cudaErrorInvalidValue;
  if (epi == EPI_SWIGLU) {
    if (!make_map(&tw1, B1, wrows, (uint64_t)K, SW_WROWS, SW_KB)) return cudaErrorInvalidValue;
  } else {
    tw1 = tw0;
  }
  SwapParams p{};
  p.offsets = offsets;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.err = device_error_word();
  p.rows = a_rows;
  p.G = n_groups;
  p.N = N;
  p.K = K;
  p.feat_tile = epi == EPI_SWIGLU ? SW_WROWS : 2 * SW_WROWS;
  p.nt = (N + p.feat_tile - 1) / p.feat_tile;
  p.fault = fault;
  p.gather_src = gather_src;
  p.gather_div = gather_div;
  const int64_t max_tiles = ((a_rows + SW_TOK - 1) / SW_TOK + n_groups) * (int64_t)p.nt;
  const int sms = gemm_sm_count();
  const int grid = (int)(max_tiles < sms ? max_tiles : sms);
  const size_t smem = swap_smem(n_groups);
  return gather_src ? launch_swap_gather<true>(epi, tx, tw0, tw1, p, grid, smem, s)
                    : launch_swap_gather<false>(epi, tx, tw0, tw1, p, grid, smem, s);
}

}  // namespace moe
