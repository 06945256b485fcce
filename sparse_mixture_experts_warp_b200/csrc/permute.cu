// Dispatch: a counting-sort permutation of (token, slot) assignments into expert-contiguous
// rows, with an optional capacity clamp, and the gather of token rows into that order.
//
// "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife),
// section 5 (torch.where lists, per expert, its (token, route slot) pairs in row-major order);
// "Top-k 路由（Top-k Routing）" (compassingai), capacity factor (expert buffer = CF * T/N * k);
// "别只比较 Top-k" (ailearn moe-comparison), capacity + overflow row of the balance table
// (an overflowing token skips the expert).
//
// Token choice, A = T*k assignments a = t*k + j, processed in blocks of kBlockItems:
//   1. hist:   per block, per expert assignment counts                    -> block_hist[blk][E]
//   2. scan:   per expert, exclusive scan over blocks (block bases) and total counts; kept =
//              min(count, C); offsets = exclusive scan of kept over experts
//   3. rank:   per block, the stable rank of each assignment within its expert, from
//              __match_any_sync peer groups inside a warp, per-warp counts in shared memory and
//              the block base -- no atomics decide any order; row = offsets[e] + rank, kept
//              when rank < C
//   4. gather: one warp per token reads x[t] once (16-byte loads) and writes it to each of its
//              kept rows.
// Expert choice: row e*c + i is the i-th picked token of expert e (already in token order).
#include <stdlib.h>

#include "common.cuh"
#include "tc_ops.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;                // 8 warps
constexpr int kChunksPerWarp = 4;            // 32 assignments per chunk
constexpr int kBlockItems = kThreads * kChunksPerWarp;   // 1024 assignments per block
constexpr int kWarpsPerBlock = kThreads / 32;

__global__ void __launch_bounds__(kThreads)
perm_hist_kernel(const int32_t* ids, int A, int E, int32_t* block_hist) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int s_hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kBlockItems;
  for (int i = threadIdx.x; i < kBlockItems; i += blockDim.x) {
    const int a = base + i;
    if (a < A) {
      const int e = ids[a];
      if (e >= 0 && e < E) atomicAdd(&s_hist[e], 1);   // counting only: order-free
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) block_hist[(int64_t)blockIdx.x * E + e] = s_hist[e];
}

// One block; thread e walks the blocks of expert e; then an exclusive scan over experts.
__global__ void __launch_bounds__(1024)
perm_scan_kernel(int32_t* block_hist, int nblk, int E, int cap, int32_t* counts,
                 int32_t* offsets) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_warp[32];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
    for (int b = 0; b < nblk; ++b) {
      const int v = block_hist[(int64_t)b * E + e];
      block_hist[(int64_t)b * E + e] = total;    // becomes the block base of expert e
      total += v;
    }
    counts[e] = total;
  }
  const int kept = (e < E) ? ((cap > 0 && total > cap) ? cap : total) : 0;
  // exclusive scan of kept over experts
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int inc = kept;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < nw) ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < nw) s_warp[lane] = w;
  }
  __syncthreads();
  const int before = (warp > 0) ? s_warp[warp - 1] : 0;
  if (e < E) offsets[e] = before + inc - kept;
  if (e == E - 1) offsets[E] = before + inc;
}

__global__ void __launch_bounds__(kThreads)
perm_rank_kernel(const int32_t* ids, int A, int E, int cap, const int32_t* block_base,
                 const int32_t* offsets, int32_t* row_src, int32_t* inv) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int s_mem[];
  int* s_cnt = s_mem;                             // [warps][E] per-warp counts, then bases
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarpsPerBlock * E; i += blockDim.x) s_cnt[i] = 0;
  __syncthreads();
  const int wbase = blockIdx.x * kBlockItems + warp * (32 * kChunksPerWarp);
  int* my = s_cnt + warp * E;
  const unsigned lt = (1u << lane) - 1u;
  // pass 1: per-warp counts per expert
  for (int ch = 0; ch < kChunksPerWarp; ++ch) {
    const int a = wbase + ch * 32 + lane;
    const int e = (a < A) ? ids[a] : -1;
    const bool ok = (e >= 0 && e < E);
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
    if (ok && (peers & lt) == 0) my[e] += __popc(peers);   // leader of the peer group
    __syncwarp();
  }
  __syncthreads();
  // per expert: exclusive scan over warps, plus the block base
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = block_base[(int64_t)blockIdx.x * E + e];
    for (int w = 0; w < kWarpsPerBlock; ++w) {
      const int v = s_cnt[w * E + e];
      s_cnt[w * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  // pass 2: ranks
  for (int ch = 0; ch < kChunksPerWarp; ++ch) {
    const int a = wbase + ch * 32 + lane;
    const int e = (a < A) ? ids[a] : -1;
    const bool ok = (e >= 0 && e < E);
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
    int rank = 0;
    if (ok) rank = my[e] + __popc(peers & lt);
    __syncwarp();
    if (ok && (peers & lt) == 0) my[e] += __popc(peers);
    __syncwarp();
    if (a < A) {
      int row = -1;
      if (ok && (cap <= 0 || rank < cap)) {
        row = offsets[e] + rank;
        row_src[row] = a;
      }
      inv[a] = row;
    }
  }
}


// Small problems (A <= kFusedMaxItems): histogram, scans and stable ranks in ONE block of 32
// warps.  The expert ids are first staged in shared memory with all loads in flight at once;
// warp w owns the contiguous assignments [w*S, (w+1)*S); pass 1 counts them per expert (peer
// groups from __match_any_sync, leader adds), the per-expert exclusive scan over warps gives
// each warp its base, a block scan over experts gives the offsets, and pass 2 assigns ranks in
// the same order.  One launch instead of three.
constexpr int kFusedMaxItems = 1 << 13;

__global__ void __launch_bounds__(1024)
perm_index_fused_kernel(const int32_t* ids, int A, int E, int cap, int32_t* counts,
                        int32_t* offsets, int32_t* row_src, int32_t* inv) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int s_mem[];
  int* s_cnt = s_mem;                    // [32][E]
  int* s_off = s_mem + 32 * E;           // [E]
  int* s_ids = s_mem + 33 * E;           // [A]
  __shared__ int s_warp[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) s_cnt[i] = 0;
  for (int i = threadIdx.x; i < A; i += blockDim.x) s_ids[i] = ids[i];
  __syncthreads();
  const int per = ((A + 32 * 32 - 1) / (32 * 32)) * 32;       // multiple of 32
  const int lo = warp * per, hi = min(A, lo + per);
  int* my = s_cnt + warp * E;
  const unsigned lt = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int a = base + lane;
    const int e = (a < hi) ? s_ids[a] : -1;
    const bool ok = (e >= 0 && e < E);
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
    if (ok && (peers & lt) == 0) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  int kept = 0;
  const int e = threadIdx.x;
  if (e < E) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int v = s_cnt[w * E + e];
      s_cnt[w * E + e] = run;
      run += v;
    }
    counts[e] = run;
    kept = (cap > 0 && run > cap) ? cap : run;
  }
  // exclusive scan of kept over experts (E <= 1024)
  int inc = kept;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int wv = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wv, o);
      if (lane >= o) wv += n;
    }
    s_warp[lane] = wv;
  }
  __syncthreads();
  const int excl = (warp > 0 ? s_warp[warp - 1] : 0) + inc - kept;
  if (e < E) {
    offsets[e] = excl;
    s_off[e] = excl;
  }
  if (e == E - 1) offsets[E] = excl + kept;
  __syncthreads();
  for (int base = lo; base < hi; base += 32) {
    const int a = base + lane;
    const int ee = (a < hi) ? s_ids[a] : -1;
    const bool ok = (ee >= 0 && ee < E);
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? ee : -1);
    int rank = 0;
    if (ok) rank = my[ee] + __popc(peers & lt);
    __syncwarp();
    if (ok && (peers & lt) == 0) my[ee] += __popc(peers);
    __syncwarp();
    if (a < hi) {
      int row = -1;
      if (ok && (cap <= 0 || rank < cap)) {
        row = s_off[ee] + rank;
        row_src[row] = a;
      }
      inv[a] = row;
    }
  }
}


// Mid-sized problems (kClusterMinItems < A <= kClusterMaxItems, E <= 1024): the index kernel
// above spread over one cluster of up to 8 CTAs.  CTA r stages and ranks the contiguous
// assignments [r*C, (r+1)*C) (C a multiple of 1024: 32 warps x whole 32-assignment batches).
// After its per-warp counts, every CTA reads the per-expert totals of all CTAs of the cluster
// through distributed shared memory: the lower ranks' totals are its base, their sum the
// expert's count.  The capacity clamp and the exclusive scan over experts then give every CTA
// the same offsets (CTA 0 writes counts and offsets).  Ranks are global (base + the warp
// prefix + the rank inside the batch), so rows follow the (token, slot) order across CTAs
// exactly as in the one-CTA kernel.
constexpr int kClusterMaxCTAs = 8;
constexpr int kClusterMinItems = 1 << 11;
constexpr int kClusterMaxItems = kClusterMaxCTAs * (1 << 13);

__global__ void __launch_bounds__(1024)
perm_index_cluster_kernel(const int32_t* ids, int A, int E, int cap, int chunk, int32_t* counts,
                          int32_t* offsets, int32_t* row_src, int32_t* inv) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int s_mem[];
  int* s_cnt = s_mem;                    // [32][E]
  int* s_tot = s_mem + 32 * E;           // [E] this CTA's totals, read by the whole cluster
  int* s_off = s_tot + E;                // [E]
  int* s_base = s_off + E;               // [E]
  int* s_ids = s_base + E;               // [chunk]
  __shared__ int s_warp[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster_cta_rank(), ncta = (int)gridDim.x;   // one cluster
  const int a0 = rank * chunk;
  const int n = max(0, min(A, a0 + chunk) - a0);
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) s_cnt[i] = 0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s_ids[i] = ids[a0 + i];
  __syncthreads();
  const int per = chunk / 32;            // multiple of 32
  const int lo = warp * per, hi = min(n, lo + per);
  int* my = s_cnt + warp * E;
  const unsigned lt = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int a = base + lane;
    const int e = (a < hi) ? s_ids[a] : -1;
    const bool ok = (e >= 0 && e < E);
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
    if (ok && (peers & lt) == 0) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  const int e = threadIdx.x;
  if (e < E) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int v = s_cnt[w * E + e];
      s_cnt[w * E + e] = run;
      run += v;
    }
    s_tot[e] = run;
  }
  cluster_sync_all();                    // every CTA's totals are in its shared memory
  int kept = 0;
  if (e < E) {
    const uint32_t at = smem_u32(s_tot + e);
    int base = 0, total = 0;
    for (int r = 0; r < ncta; ++r) {
      const int v = ld_cluster_s32(cluster_map(at, (uint32_t)r));
      if (r < rank) base += v;
      total += v;
    }
    s_base[e] = base;
    if (rank == 0) counts[e] = total;
    kept = (cap > 0 && total > cap) ? cap : total;
  }
  // exclusive scan of kept over experts (E <= 1024)
  int inc = kept;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int wv = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wv, o);
      if (lane >= o) wv += v;
    }
    s_warp[lane] = wv;
  }
  __syncthreads();
  const int excl = (warp > 0 ? s_warp[warp - 1] : 0) + inc - kept;
  if (e < E) {
    s_off[e] = excl;
    if (rank == 0) offsets[e] = excl;
  }
  if (rank == 0 && e == E - 1) offsets[E] = excl + kept;
  cluster_sync_all();                    // no CTA reads a peer's totals past here
  for (int base = lo; base < hi; base += 32) {
    const int a = base + lane;
    const int ee = (a < hi) ? s_ids[a] : -1;
    const bool ok = (ee >= 0 && ee < E);
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? ee : -1);
    int rk = 0;
    if (ok) rk = s_base[ee] + my[ee] + __popc(peers & lt);
    __syncwarp();
    if (ok && (peers & lt) == 0) my[ee] += __popc(peers);
    __syncwarp();
    if (a < hi) {
      int row = -1;
      if (ok && (cap <= 0 || rk < cap)) {
        row = s_off[ee] + rk;
        row_src[row] = a0 + a;
      }
      inv[a0 + a] = row;
    }
  }
}

// One-pass token-choice permute for small problems (E <= 8, k <= 8, A <= kOnePassMaxItems):
// every CTA owns 32 consecutive tokens.  It first counts ALL assignments per expert (totals)
// and those before its own tokens (its per-expert base) -- the ids are L2-resident and shared
// by all CTAs, so this replaces a grid-wide scan.  Counting uses per-thread packed counters
// (eight 8-bit counts in two registers) and a fixed-order block reduction.  Then it ranks its
// own assignments stably (peer groups of __match_any_sync, per-warp prefix), writes inv /
// row_src (CTA 0 also counts and offsets), and copies its tokens' rows into their expert rows
// with four tokens' loads in flight per warp.  Counting is order-free and every rank is a
// deterministic prefix: the result equals the multi-kernel path bit for bit.
constexpr int kOnePassTokens = 32;
constexpr int kOnePassMaxE = 8;
constexpr int kOnePassMaxK = 8;
constexpr int kOnePassMaxItems = 1 << 14;       // <= 64 ids per thread: 8-bit counts suffice

__device__ __forceinline__ void count_packed(int e, uint32_t& lo, uint32_t& hi) {
  const uint32_t inc = 1u << (8 * (e & 3));
  if (e >= 0 && e < 4) lo += inc;
  else if (e >= 4 && e < 8) hi += inc;
}

__global__ void __launch_bounds__(256)
permute_onepass_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int cap,
                       const uint4* __restrict__ x, int nvec, uint4* __restrict__ xp,
                       int32_t* counts, int32_t* offsets, int32_t* row_src, int32_t* inv) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_all[8][kOnePassMaxE];       // per warp: all assignments
  __shared__ int s_pre[8][kOnePassMaxE];       // per warp: assignments before this CTA's
  __shared__ int s_own[8][kOnePassMaxE];       // per warp: this CTA's, then exclusive bases
  __shared__ int s_off[kOnePassMaxE];
  __shared__ int s_row[kOnePassTokens * kOnePassMaxK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const int A = T * k;
  const int a0 = blockIdx.x * kOnePassTokens * k;
  const int a1 = min(A, a0 + kOnePassTokens * k);
  // 1. packed per-thread counts of all ids and of the ids before a0
  uint32_t all_lo = 0, all_hi = 0, pre_lo = 0, pre_hi = 0;
  for (int base0 = threadIdx.x; base0 < A; base0 += 256 * 8) {
    int ev[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int a = base0 + 256 * u;
      ev[u] = (a < A) ? __ldg(ids + a) : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int a = base0 + 256 * u;
      count_packed(ev[u], all_lo, all_hi);
      if (a < a0) count_packed(ev[u], pre_lo, pre_hi);
    }
  }
  // unpack and reduce over the warp (fixed butterfly), then over warps through shared memory
  int call[kOnePassMaxE], cpre[kOnePassMaxE];
#pragma unroll
  for (int e = 0; e < kOnePassMaxE; ++e) {
    const uint32_t wa = e < 4 ? all_lo : all_hi, wp = e < 4 ? pre_lo : pre_hi;
    call[e] = (int)((wa >> (8 * (e & 3))) & 0xffu);
    cpre[e] = (int)((wp >> (8 * (e & 3))) & 0xffu);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      call[e] += __shfl_xor_sync(0xffffffffu, call[e], o);
      cpre[e] += __shfl_xor_sync(0xffffffffu, cpre[e], o);
    }
  }
  if (lane < kOnePassMaxE) {
    int va = 0, vp = 0;
#pragma unroll
    for (int e = 0; e < kOnePassMaxE; ++e)
      if (lane == e) { va = call[e]; vp = cpre[e]; }
    s_all[warp][lane] = va;
    s_pre[warp][lane] = vp;
    s_own[warp][lane] = 0;
  }
  __syncthreads();
  // own assignments: chunk `warp` of the CTA's range (<= 8 chunks of 32)
  const int oa = a0 + warp * 32 + lane;
  const int oe = (oa < a1) ? ids[oa] : -1;
  const bool ook = oe >= 0 && oe < E;
  const unsigned opeers = __match_any_sync(0xffffffffu, ook ? oe : -1);
  if (ook && (opeers & lt) == 0) s_own[warp][oe] = __popc(opeers);
  __syncthreads();
  // 2. per expert: totals, kept, bases; offsets = exclusive scan of kept (one warp)
  if (warp == 0) {
    int total = 0, pre = 0;
    if (lane < E) {
      for (int w = 0; w < 8; ++w) {
        total += s_all[w][lane];
        pre += s_pre[w][lane];
      }
      int run = pre;                               // exclusive bases of this CTA's warps
      for (int w = 0; w < 8; ++w) {
        const int v = s_own[w][lane];
        s_own[w][lane] = run;
        run += v;
      }
    }
    const int kept = (lane < E) ? ((cap > 0 && total > cap) ? cap : total) : 0;
    int inc = kept;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += n;
    }
    if (lane < E) {
      s_off[lane] = inc - kept;
      if (blockIdx.x == 0) {
        counts[lane] = total;
        offsets[lane] = inc - kept;
      }
    }
    if (blockIdx.x == 0 && lane == E - 1) offsets[E] = inc;
  }
  __syncthreads();
  // 3. stable ranks of this CTA's assignments
  if (oa < a1) {
    int row = -1;
    if (ook) {
      const int rank = s_own[warp][oe] + __popc(opeers & lt);
      if (cap <= 0 || rank < cap) {
        row = s_off[oe] + rank;
        row_src[row] = oa;
      }
    }
    inv[oa] = row;
    s_row[oa - a0] = row;
  }
  __syncthreads();
  if (xp == nullptr) return;      // indices only: the up projection gathers the rows itself
  // 4. copy: warp w copies tokens 4w .. 4w+3 of the CTA's 32; each lane keeps 4 tokens x 4
  //    chunks (256 bytes) of loads in flight before it stores them to the expert rows
  const int tw = blockIdx.x * kOnePassTokens + warp * 4;
  int rows[4][kOnePassMaxK];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int jj = 0; jj < kOnePassMaxK; ++jj)
      rows[u][jj] = (tw + u < T && jj < k) ? s_row[(warp * 4 + u) * k + jj] : -1;
  int v = lane;
  for (; v + 96 < nvec; v += 128) {
    uint4 q[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int c = 0; c < 4; ++c)
        q[u][c] = (tw + u < T) ? __ldcs(x + (int64_t)(tw + u) * nvec + v + 32 * c)
                               : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int jj = 0; jj < kOnePassMaxK; ++jj) {
        const int r = rows[u][jj];
        if (r < 0) continue;
        uint4* dst = xp + (int64_t)r * nvec + v;
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[32 * c] = q[u][c];
      }
  }
  for (; v < nvec; v += 32) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (tw + u >= T) break;
      const uint4 q0 = __ldcs(x + (int64_t)(tw + u) * nvec + v);
#pragma unroll
      for (int jj = 0; jj < kOnePassMaxK; ++jj)
        if (rows[u][jj] >= 0) xp[(int64_t)rows[u][jj] * nvec + v] = q0;
    }
  }
}

// One warp per token: copy x[t] (D elements of `esz` bytes) to each kept row.
__global__ void __launch_bounds__(256)
gather_tc_kernel(const uint4* __restrict__ x, int T, int nvec, int k, const int32_t* inv,
                 uint4* __restrict__ xp) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= T) return;
  int rows[8];
  int nr = 0;
  for (int j = 0; j < k && j < 8; ++j) {
    const int r = inv[(int64_t)warp * k + j];
    rows[j] = r;
    nr = j + 1;
  }
  const uint4* src = x + (int64_t)warp * nvec;
  int v = lane;
  for (; v + 96 < nvec; v += 128) {
    const uint4 a0 = __ldcs(src + v), a1 = __ldcs(src + v + 32), a2 = __ldcs(src + v + 64),
                a3 = __ldcs(src + v + 96);
    for (int j = 0; j < nr; ++j) {
      if (rows[j] < 0) continue;
      uint4* dst = xp + (int64_t)rows[j] * nvec;
      dst[v] = a0; dst[v + 32] = a1; dst[v + 64] = a2; dst[v + 96] = a3;
    }
  }
  for (; v < nvec; v += 32) {
    const uint4 a0 = __ldcs(src + v);
    for (int j = 0; j < nr; ++j) {
      if (rows[j] < 0) continue;
      xp[(int64_t)rows[j] * nvec + v] = a0;
    }
  }
  // k > 8: remaining slots (not used by the shipped workloads, kept correct)
  for (int j = 8; j < k; ++j) {
    const int r = inv[(int64_t)warp * k + j];
    if (r < 0) continue;
    for (int u = lane; u < nvec; u += 32) xp[(int64_t)r * nvec + u] = src[u];
  }
}

// Expert choice: row r = e*c + i takes token picked[r]; inv[t*E + e] = r.
__global__ void ec_fill_kernel(int32_t* inv, int64_t n) {
  pdl_trigger();
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) inv[i] = -1;
}

__global__ void ec_index_kernel(const int32_t* picked, int E, int c, int T, int32_t* counts,
                                int32_t* offsets, int32_t* row_src, int32_t* inv) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r <= E) {
    offsets[r] = r * c;
    if (r < E) counts[r] = c;
  }
  if (r < E * c) {
    const int e = r / c;
    const int t = picked[r];
    if (t >= 0 && t < T) {
      row_src[r] = t * E + e;
      inv[(int64_t)t * E + e] = r;
    } else {
      row_src[r] = -1;
    }
  }
}

__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4* __restrict__ x, int T, int nvec, const int32_t* picked, int rows,
                   uint4* __restrict__ xp) {
  pdl_trigger();
  pdl_wait();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int t = picked[r];
  if (t < 0 || t >= T) return;
  const uint4* src = x + (int64_t)t * nvec;
  uint4* dst = xp + (int64_t)r * nvec;
  for (int v = lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
}

}  // namespace

int permute_blocks(const moe_desc_t& d) {
  const int64_t A = (int64_t)d.T * d.k;
  return (int)((A + kBlockItems - 1) / kBlockItems);
}

// MOE_PERMUTE_CLUSTER=0 keeps the one-CTA index kernel (A <= 8192) and the three-kernel
// histogram path instead of the cluster kernel (comparison measurements; both are tested).
static bool permute_cluster_enabled() {
  static const bool v = [] {
    const char* e = getenv("MOE_PERMUTE_CLUSTER");
    return !(e && e[0] == '0');
  }();
  return v;
}

cudaError_t launch_permute_token_choice(const moe_desc_t& d, const int32_t* ids, const void* x,
                                        void* x_perm, int32_t* counts, int32_t* offsets,
                                        int32_t* row_src, int32_t* inv, int32_t* block_hist,
                                        int32_t cap, cudaStream_t s) {
  const int A = d.T * d.k;
  const int nblk = permute_blocks(d);
  const int E = d.E;
  const int esz = (d.dtype == MOE_BF16) ? 2 : 4;
  const int nvec = d.D * esz / 16;
  if (A > 0 && A <= kOnePassMaxItems && E <= kOnePassMaxE && d.k <= kOnePassMaxK) {
    const int grid = (d.T + kOnePassTokens - 1) / kOnePassTokens;
    (void)launch_pdl(permute_onepass_kernel, dim3(grid), dim3(256), 0, s, ids, d.T, d.k, E, cap,
                                                static_cast<const uint4*>(x), nvec,
                                                static_cast<uint4*>(x_perm), counts, offsets,
                                                row_src, inv);
    return cudaGetLastError();
  }
  if (A > kClusterMinItems && A <= kClusterMaxItems && E <= 1024 && permute_cluster_enabled()) {
    int ncta = (A + 1023) / 1024;
    if (ncta > kClusterMaxCTAs) ncta = kClusterMaxCTAs;
    const int chunk = ((A + ncta - 1) / ncta + 1023) / 1024 * 1024;
    ncta = (A + chunk - 1) / chunk;
    const size_t smem = ((size_t)35 * E + chunk) * sizeof(int);
    cudaError_t e = cudaFuncSetAttribute(perm_index_cluster_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    note_launch();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ncta);
    cfg.blockDim = dim3(1024);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)ncta;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, perm_index_cluster_kernel, ids, A, E, cap, chunk, counts,
                           offsets, row_src, inv);
    if (e != cudaSuccess) return e;
  } else if (A <= kFusedMaxItems) {
    const size_t smem = ((size_t)33 * E + A) * sizeof(int);
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(perm_index_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
    (void)launch_pdl(perm_index_fused_kernel, dim3(1), dim3(1024), smem, s, ids, A, E, cap, counts, offsets, row_src, inv);
  } else {
    (void)launch_pdl(perm_hist_kernel, dim3(nblk), dim3(kThreads), E * sizeof(int), s, ids, A, E, block_hist);
    (void)launch_pdl(perm_scan_kernel, dim3(1), dim3(1024), 0, s, block_hist, nblk, E, cap, counts, offsets);
    (void)launch_pdl(perm_rank_kernel, dim3(nblk), dim3(kThreads), kWarpsPerBlock * E * sizeof(int), s, 
        ids, A, E, cap, block_hist, offsets, row_src, inv);
  }
  if (nblk > 0 && x_perm) {
    const int blocks = (d.T * 32 + 255) / 256;
    (void)launch_pdl(gather_tc_kernel, dim3(blocks), dim3(256), 0, s, static_cast<const uint4*>(x), d.T, nvec, d.k, inv,
                                            static_cast<uint4*>(x_perm));
  }
  return cudaGetLastError();
}

cudaError_t launch_gather_permuted_rows(const moe_desc_t& d, const int32_t* ids,
                                        const int32_t* inv, const void* x, void* x_perm,
                                        cudaStream_t s) {
  const int esz = (d.dtype == MOE_BF16) ? 2 : 4;
  const int nvec = d.D * esz / 16;
  if (d.select == MOE_TOKEN_CHOICE) {
    if (d.T > 0)
      (void)launch_pdl(gather_tc_kernel, dim3((d.T * 32 + 255) / 256), dim3(256), 0, s, 
          static_cast<const uint4*>(x), d.T, nvec, d.k, inv, static_cast<uint4*>(x_perm));
  } else {
    const int rows = d.E * d.c;
    if (rows > 0)
      (void)launch_pdl(gather_rows_kernel, dim3((rows * 32 + 255) / 256), dim3(256), 0, s, 
          static_cast<const uint4*>(x), d.T, nvec, ids, rows, static_cast<uint4*>(x_perm));
  }
  return cudaGetLastError();
}

cudaError_t launch_permute_expert_choice(const moe_desc_t& d, const int32_t* picked,
                                         const void* x, void* x_perm, int32_t* counts,
                                         int32_t* offsets, int32_t* row_src, int32_t* inv,
                                         cudaStream_t s) {
  const int64_t n = (int64_t)d.T * d.E;
  if (n > 0) (void)launch_pdl(ec_fill_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, inv, n);
  const int rows = d.E * d.c;
  const int m = (rows > d.E + 1 ? rows : d.E + 1);
  (void)launch_pdl(ec_index_kernel, dim3((m + 255) / 256), dim3(256), 0, s, picked, d.E, d.c, d.T, counts, offsets,
                                                  row_src, inv);
  const int esz = (d.dtype == MOE_BF16) ? 2 : 4;
  const int nvec = d.D * esz / 16;
  if (rows > 0 && x_perm)
    (void)launch_pdl(gather_rows_kernel, dim3((rows * 32 + 255) / 256), dim3(256), 0, s, 
        static_cast<const uint4*>(x), d.T, nvec, picked, rows, static_cast<uint4*>(x_perm));
  return cudaGetLastError();
}

}  // namespace moe
