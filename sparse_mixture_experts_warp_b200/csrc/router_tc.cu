// Router on the fifth-generation tensor cores, fused with the selection.
//
// "Top-k 路由（Top-k Routing）" (compassingai), "門控函式的數學形式" Steps 1-3 (s = W_g x, the
// affinity, top-k); "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡"
// (f3dlife), section 4; "别只比较 Top-k" (ailearn moe-comparison), Score / Select / Merge steps;
// "Top-k 路由" Token-Choice vs Expert-Choice table (the expert-choice probabilities).
//
// One cluster of ks CTAs (ks = 1..4 k-ranges of the hidden dimension) per tile of 128 tokens.
// CTA r of the cluster computes the fp32 partial logits of the tile's tokens over its k-range:
// warp 0 streams x and W_g boxes (64 columns, 128-byte swizzle) into a ring with TMA, warp 1
// issues tcgen05.mma (M = 128 tokens, N = E rounded up to 16, K = 16) into a TMEM accumulator,
// warps 2-5 read it back (one token row per thread) and write it to shared memory as rows
// [token][E] (odd pitch: conflict-free whether a warp reads a row, a column or one element of
// 32 rows).  After a cluster barrier, CTA r takes 128 / ks of the tile's tokens and sums their
// ks partial rows in rank order (the peers' rows through distributed shared memory), and its
// 16 warps route them, one warp per token, with the per-token selection the SIMT router also
// uses.  Column sums of the probability rows give the importance partial of the CTA.  Only x,
// W_g and the routing outputs touch global memory: no partial logits leave the chip.
#include <cuda.h>

#include "common.cuh"
#include "mbar.cuh"
#include "route_select.cuh"
#include "tc_ops.cuh"

namespace moe {
namespace {

constexpr int kRtRows = 128;          // tokens per tile (MMA M)
constexpr int kRtKB = 64;             // k-block: 64 bf16, one 128-byte swizzled row
constexpr int kRtWarps = 16;          // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 TMEM readers;
                                      // all of them route once the logits are in shared memory
constexpr int kRtMaxSplit = 4;        // CTAs per cluster
constexpr int kRtMaxStages = 8;
constexpr uint32_t kRtABytes = kRtRows * kRtKB * 2;       // x box per stage
constexpr uint32_t kRtRingBudget = 192 * 1024;
constexpr uint64_t kRtTimeoutNs = 2000000000ull;          // 2 s per wait
constexpr uint64_t kRtDrainNs = 200000000ull;

struct RtParams {
  RouterArgs a;
  int npad;        // MMA N: E rounded up to a multiple of 16
  int pitch;       // floats per logit row in shared memory (E rounded up to 32, + 1)
  int ks;          // k-ranges = CTAs per cluster
  int kchunk;      // k-blocks per range
  int nkb;         // k-blocks of D
  int stages;      // ring depth
  int tmem_cols;   // TMEM columns allocated (power of two >= 32, >= npad)
  int* err;        // device error word
};

// Shared memory, from the 1024-byte aligned base: the ring (x box + W_g box per stage), reused
// after the main loop for the logit rows [128][pitch]; per-warp entropy sums; the barriers.
struct RtLayout {
  uint32_t aux, bars, total;
};
__host__ __device__ inline RtLayout rt_layout(int E, int npad, int pitch, int stages) {
  RtLayout L;
  const uint32_t ring = (uint32_t)stages * (kRtABytes + (uint32_t)npad * kRtKB * 2);
  const uint32_t rows = (uint32_t)kRtRows * (uint32_t)pitch * 4u;
  uint32_t off = ring > rows ? ring : rows;
  L.aux = off;
  off += (uint32_t)kRtWarps * 4u;
  off = (off + 7u) & ~7u;
  L.bars = off;
  off += (uint32_t)(2 * stages + 2) * 8u + 8u;     // full, empty, tfull, drain; TMEM address, abort flag
  L.total = off;
  return L;
}

// NS: expert slots per lane in the selection (E <= 32 NS).
template <int NS>
__global__ void __launch_bounds__(kRtWarps * 32, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const __grid_constant__ RtParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const RouterArgs& a = p.a;
  const int E = a.E, S = p.stages;
  const RtLayout L = rt_layout(E, p.npad, p.pitch, S);
  const uint32_t b_bytes = (uint32_t)p.npad * kRtKB * 2;
  const uint32_t sA = smem_u32(smem), sB = sA + (uint32_t)S * kRtABytes;
  float* s_log = reinterpret_cast<float*>(smem);          // [128][pitch], after the main loop
  float* s_ent = reinterpret_cast<float*>(smem + L.aux);  // [kRtWarps] entropy sums
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* drain = tfull + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const int m0 = (int)cluster_id_x() * kRtRows;
  const int kb0 = (int)rank * p.kchunk;
  const int kb1 = min(p.nkb, kb0 + p.kchunk);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(p.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // set-up of this CTA's own shared and tensor memory above; x and W_g may come from earlier
  // kernels, and the outputs may still be read by them
  pdl_trigger();
  pdl_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, DEVERR_TIMEOUT_TMA,
                       kRtTimeoutNs)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&full[stage], kRtABytes + b_bytes);
        tma_load_2d(sA + (uint32_t)stage * kRtABytes, &tmX, &full[stage], kb * kRtKB, m0);
        tma_load_2d(sB + (uint32_t)stage * b_bytes, &tmW, &full[stage], kb * kRtKB, 0);
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        // let the copies already in flight land before the ring is reused
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s))
            mbar_wait(&full[s], (issued_par >> s) & 1u, abort_flag, p.err, DEVERR_TIMEOUT_TMA,
                      kRtDrainNs, /*honor_abort=*/false);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = idesc_bf16(kRtRows, p.npad);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.err, DEVERR_TIMEOUT_MMA,
                       kRtTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = sA + (uint32_t)stage * kRtABytes, b0 = sB + (uint32_t)stage * b_bytes;
#pragma unroll
        for (int k = 0; k < kRtKB / 16; ++k)
          umma_bf16(tmem_base, sdesc<kRtKB>(a0 + k * 32), sdesc<kRtKB>(b0 + k * 32),
                    (kb > kb0 || k > 0) ? 1u : 0u, idesc);
        umma_commit(&empty[stage]);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) umma_commit(tfull);
      umma_commit(drain);
      mbar_wait(drain, 0u, abort_flag, p.err, DEVERR_TIMEOUT_MMA, ok ? kRtTimeoutNs : kRtDrainNs,
                /*honor_abort=*/false);
    }
  } else if (warp < 6) {
    // ---------------- TMEM -> logit rows in shared memory ----------------
    const int q = warp & 3;                 // the TMEM lane quarter this warp may read
    const int row = 32 * q + lane;
    int okw = 1;
    if (lane == 0)
      okw = mbar_wait(tfull, 0u, abort_flag, p.err, DEVERR_TIMEOUT_EPI, kRtTimeoutNs);
    okw = __shfl_sync(0xffffffffu, okw, 0);
    if (okw) {
      tc_fence_after();
      for (int c0 = 0; c0 < p.npad; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
        tmem_wait_ld();
        float* dst = s_log + row * p.pitch + c0;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[j] = __uint_as_float(v[j]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(p.tmem_cols)
                 : "memory");
  }

  // ---------------- partial sums over the cluster ----------------
  const int tpc = (kRtRows + p.ks - 1) / p.ks;           // tokens per CTA of the cluster
  const int i0 = min(kRtRows, (int)rank * tpc);
  const int i1 = min(min(kRtRows, i0 + tpc), a.T - m0);
  const int n_rows = i1 > i0 ? i1 - i0 : 0;
  if (p.ks > 1) {
    cluster_sync_all();                     // every CTA's partial rows are in its shared memory
    const uint32_t base = smem_u32(s_log);
    uint32_t peer[kRtMaxSplit];
#pragma unroll
    for (int r = 0; r < kRtMaxSplit; ++r) peer[r] = cluster_map(base, (uint32_t)(r < p.ks ? r : 0));
    // per lane 4 experts of a row at a time, all ranks' values loaded before they are summed
    for (int j = warp; j < n_rows; j += kRtWarps) {
      const int i = i0 + j;
      for (int e0 = lane; e0 < E; e0 += 128) {
        float v[4][kRtMaxSplit];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int r = 0; r < kRtMaxSplit; ++r)
            if (r < p.ks && e0 + 32 * u < E)
              v[u][r] = ld_cluster_f32(peer[r] + (uint32_t)(i * p.pitch + e0 + 32 * u) * 4u);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (e0 + 32 * u >= E) break;
          float acc = v[u][0];
#pragma unroll
          for (int r = 1; r < kRtMaxSplit; ++r)       // rank order
            if (r < p.ks) acc += v[u][r];
          s_log[i * p.pitch + e0 + 32 * u] = acc;     // rows [i0, i1): read by this CTA only
        }
      }
    }
    cluster_sync_all();                     // no CTA reads a peer's shared memory past here
  }

  // ---------------- routing: a warp per token ----------------
  // logits out, affinity, group limit, top-k, merge weights, -sum p log p (the selection
  // shared with the SIMT router); the probabilities replace the logits in the row, for the
  // importance column sums and, under expert choice, the transposed copy
  float imp[NS];
#pragma unroll
  for (int u = 0; u < NS; ++u) imp[u] = 0.f;
  float ent = 0.f;
  // warp w takes tokens w, w + 16, w + 32, ... two at a time in lockstep
  for (int j = warp; j < n_rows; j += 2 * kRtWarps) {
    const int jt[2] = {j, j + kRtWarps};
    const bool has[2] = {true, j + kRtWarps < n_rows};
    int tk[2];
    float sv[2][NS], pr[2][NS];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      tk[t] = m0 + i0 + jt[t];
      const float* row = s_log + (i0 + (has[t] ? jt[t] : j)) * p.pitch;
#pragma unroll
      for (int u = 0; u < NS; ++u) {
        const int e = lane + 32 * u;
        sv[t][u] = e < E ? row[e] : -INFINITY;
      }
    }
    select_tokens<NS, 2>(a, tk, has, sv, imp, ent, pr, lane);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (!has[t]) continue;
      float* row = s_log + (i0 + jt[t]) * p.pitch;
#pragma unroll
      for (int u = 0; u < NS; ++u) {
        const int e = lane + 32 * u;
        if (e < E) row[e] = pr[t][u];
      }
    }
  }
  ent = warp_sum(ent);
  if (lane == 0) s_ent[warp] = ent;
  __syncthreads();
  if (a.expert_choice) {
    // probsT[e][t]: per expert a row segment of this CTA's consecutive tokens
    for (int e = warp; e < E; e += kRtWarps)
      for (int j = lane; j < n_rows; j += 32)
        a.probsT[(int64_t)e * a.T + m0 + i0 + j] = s_log[(i0 + j) * p.pitch + e];
  }
  if (a.partials) {
    // one row per CTA: the E importance sums (columns of the probability rows, in row order),
    // then the entropy sum (warps in order)
    for (int c = threadIdx.x; c <= E; c += blockDim.x) {
      float sum = 0.f;
      if (c < E)
        for (int j = 0; j < n_rows; ++j) sum += s_log[(i0 + j) * p.pitch + c];
      else
        for (int w = 0; w < kRtWarps; ++w) sum += s_ent[w];
      a.partials[(int64_t)blockIdx.x * (E + 1) + c] = sum;
    }
  }
}

struct RtConfig {
  int ks, kchunk, nkb, npad, pitch, stages, tmem_cols, grid;
  size_t smem;
};

RtConfig rt_config(const moe_desc_t& d) {
  RtConfig c{};
  const int mt = (d.T + kRtRows - 1) / kRtRows;
  c.nkb = d.D / kRtKB;
  int ks = mt > 0 ? num_sms() / mt : 1;
  if (ks > kRtMaxSplit) ks = kRtMaxSplit;
  if (ks > c.nkb) ks = c.nkb;
  if (ks < 1) ks = 1;
  c.kchunk = (c.nkb + ks - 1) / ks;
  c.ks = (c.nkb + c.kchunk - 1) / c.kchunk;   // every k-range non-empty
  c.npad = (d.E + 15) / 16 * 16;
  c.pitch = (d.E + 31) / 32 * 32 + 1;     // odd: conflict-free by row, column and thread-per-row
  c.tmem_cols = 32;
  while (c.tmem_cols < c.npad) c.tmem_cols <<= 1;
  const uint32_t stage_bytes = kRtABytes + (uint32_t)c.npad * kRtKB * 2;
  c.stages = (int)(kRtRingBudget / stage_bytes);
  if (c.stages > kRtMaxStages) c.stages = kRtMaxStages;
  c.grid = mt * c.ks;
  c.smem = 1024 + rt_layout(d.E, c.npad, c.pitch, c.stages).total;
  return c;
}

}  // namespace

bool router_tc_ok(const moe_desc_t& d) {
  return d.dtype == MOE_BF16 && d.D % kRtKB == 0 && d.D > 0 && d.E >= 1 && d.E <= 256 &&
         (d.select == MOE_EXPERT_CHOICE || d.k <= 32);
}

cudaError_t launch_router_tc(const moe_desc_t& d, const RouterArgs& a, int* n_partials,
                             cudaStream_t s) {
  const RtConfig c = rt_config(d);
  *n_partials = c.grid;
  if (c.grid == 0) return cudaSuccess;
  if (c.smem > 227 * 1024) return cudaErrorInvalidValue;
  alignas(64) CUtensorMap tx, tw;
  if (!make_map(&tx, a.x, (uint64_t)d.T, (uint64_t)d.D, kRtRows, kRtKB)) return cudaErrorInvalidValue;
  if (!make_map(&tw, a.Wg, (uint64_t)d.E, (uint64_t)d.D, (uint32_t)c.npad, kRtKB))
    return cudaErrorInvalidValue;
  RtParams p{};
  p.a = a;
  p.npad = c.npad;
  p.pitch = c.pitch;
  p.ks = c.ks;
  p.kchunk = c.kchunk;
  p.nkb = c.nkb;
  p.stages = c.stages;
  p.tmem_cols = c.tmem_cols;
  p.err = device_error_word();
  void (*kern)(CUtensorMap, CUtensorMap, RtParams) =
      d.E <= 32 ? router_tc_kernel<1> : d.E <= 64 ? router_tc_kernel<2>
                                      : d.E <= 128 ? router_tc_kernel<4> : router_tc_kernel<8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)c.smem);
  if (e != cudaSuccess) return e;
  note_launch();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c.grid);
  cfg.blockDim = dim3(kRtWarps * 32);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)c.ks;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, tx, tw, p);
}

}  // namespace moe
