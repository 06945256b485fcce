// Grouped GEMM for the experts' projections on 5th-generation tensor cores (sm_100a).
//
// "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife), section 3
// (SwiGLU expert: hidden = SiLU(x W_gate) * (x W_up), output = hidden W_down) and sections 5/12
// (production systems replace the per-expert loop by token permutation + grouped GEMM);
// "别只比较 Top-k" (ailearn moe-comparison), Execute step (experts run as a Grouped GEMM).
//
// out[r, n] = epi( sum_k A[r, k] * B[g*N + n, k] ) for every row r of group g, where group g owns
// rows [offsets[g], offsets[g+1]) of A.  A is [rows, K] bf16 row-major, B is the stacked
// nn.Linear weights [G*N, K] bf16 row-major (both K-major operands), accumulation is fp32 in
// tensor memory, out is bf16 [rows, N].
//   EPI_SWIGLU: B0 = W_gate, B1 = W_up; one 128x256 MMA tile holds 128 gate columns and the
//               same 128 up columns side by side in TMEM; out = SiLU(gate) * up.
//   EPI_RELU:   out = max(acc, 0) with B0 = W_up.
//   EPI_GELU:   out = acc * (1 + erf(acc / sqrt 2)) / 2 with B0 = W_up.
//   EPI_NONE:   out = acc with B0 = W_down.
//   Also used by the layer backward:
//   EPI_RAW:      SwiGLU operand staging, out = the raw gate | up accumulators (bf16);
//   EPI_NONE_BMN: out = acc with B stored MN-major ([K, N], N contiguous: a weight used as the
//                 right operand of a backward product, read as stored); K rows of group g at
//                 g * bk_group of B0 below k-block kb_split and of B1 above it;
//   EPI_F32:      fp32 out; with `kgroup` the groups run along K instead of M (weight
//                 gradients: group g owns k columns [kgroup[g], kgroup[g+1]) of A [M, Ktot]
//                 and B [N, Ktot] and writes its own [M, N] block), without it k-splits of one
//                 group write fp32 partials (the router product);
//   EPI_F32_TMA:  EPI_F32 with groups along K, written through shared memory: each epilogue
//                 warp stages 32 x 16 fp32 blocks (64-byte swizzle, two 2 KB buffers per warp)
//                 and one lane stores each with a 3-D TMA store (columns, rows, group) that
//                 clips at the group's bounds.  A weight-gradient tile has a short main loop (one
//                 expert's rows) and 128 KB of fp32 output; per-thread row stores would touch 32
//                 rows per instruction and hold the tensor pipe back.
//   An optional second output (out2) receives the raw accumulators of the SwiGLU / activation
//   epilogues as bf16: the pre-activations a training forward saves for the backward.
//
// Design (one persistent CTA per SM, warp-specialised; two tile heights, see grouped_gemm_kernel):
//   warp 0 (one thread)  TMA producer: 128-byte-swizzled K-major boxes of A (128 x 64, one or two
//                        per stage) and B (2 x 128 x 64; MN-major B: 4 x 64 x 64) into a
//                        shared-memory ring, mbarrier complete_tx; no multicast.
//   warp 1 (one thread)  MMA issuer: tcgen05.mma.cta_group::1.kind::f16, M=128 N=256 K=16, fp32
//                        accumulators in TMEM (512 columns); tcgen05.commit frees ring stages and
//                        hands finished accumulators to the epilogue.  Warp 1 also owns the TMEM
//                        allocation.
//   warps 2..            epilogue: tcgen05.ld 32x32b (warp w reads TMEM lanes 32*(w%4)..+31, one
//                        output row per thread), activation, bf16 pack, 16-byte stores of the rows
//                        that belong to the group (rows past the group end are computed from
//                        neighbouring rows and discarded).
//   128-row tiles: 4 stages of 48 KB, two 256-column accumulators so the epilogue of tile i
//   overlaps the main loop of tile i+1.  256-row tiles (the default): two M=128 MMAs per k-step
//   share each B stage, which cuts L2->SMEM bytes per FLOP by a third (the 128-row tile needs
//   ~96 B/clk/SM, more than the L2 can feed at full tensor rate); 3 stages of 64 KB, one
//   512-column accumulator set; a tile with at most 128 live rows runs one half only, so the
//   row waste stays that of 128-row tiles.
// Tiles are enumerated group by group, n-tile by n-tile, with the m-tiles innermost, so the
// CTAs that run at the same time share B tiles through L2 and each weight byte streams from
// HBM about once.  The per-group row counts are read on the device (no host sync).
// Every mbarrier wait is bounded (globaltimer); a wait that gives up records an error code in
// the device error word and makes the CTA drain its in-flight copies and MMAs and exit.
#include <cuda.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "mbar.cuh"
#include "tc_ops.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int MMA_N = 256;
constexpr int MMA_K = 16;
constexpr int ACC_COLS = MMA_N;             // fp32 accumulator columns per tile
constexpr int TMEM_COLS = 2 * ACC_COLS;     // two accumulators
constexpr uint64_t TIMEOUT_NS = 2000000000ull;   // 2 s per wait
constexpr uint64_t DRAIN_NS = 200000000ull;      // 0.2 s to drain after an abort

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A bf16 (bits 7-9 = 1), B bf16
// (bits 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22, M >> 4 at 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            ((uint32_t)(MMA_N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
// The same with M = 64, for a 128-row half that holds at most 64 live rows.  Its accumulator
// rows 16q .. 16q+15 sit in TMEM lanes 32q .. 32q+15 (16 lanes of each lane quarter).
constexpr uint32_t kIdesc64 = (1u << 4) | (1u << 7) | (1u << 10) |
                              ((uint32_t)(MMA_N >> 3) << 17) | ((uint32_t)(64 >> 4) << 24);

struct GemmParams {
  const int32_t* offsets;   // [G+1] device
  __nv_bfloat16* out;       // [rows, N]
  int* err;                 // device error word
  int64_t rows;             // rows allocated in A and out
  int64_t ldo;              // out row pitch (elements)
  int G, N, K;
  int n_out_tile;           // output columns per tile
  int nt;                   // n-tiles per group
  int fault;                // test hook: 1 = CTA 0 arms its first stage without loading it
  int ksplit;               // k-range splits (EPI_F32 only; 1 otherwise)
  int kchunk;               // k-blocks per split
  int64_t split_stride;     // EPI_F32: elements between the partial outputs of two splits
  // groups along K (weight gradients): group g owns k columns [kgroup[g], kgroup[g+1]) of both
  // operands (device array, multiples of the k-block) and writes out + g * out_gstride
  // ([rows, N], fp32 with EPI_F32); nullptr: groups along M (rows of A) as usual
  const int32_t* kgroup;
  int64_t out_gstride;
  // optional second output: the raw accumulators as bf16 (SwiGLU: gate | up blocks of 128 per
  // n-tile, row pitch ldo2 = nt * 256; others: [rows, N]), saved for the backward pass
  __nv_bfloat16* out2;
  int64_t ldo2;
  // MN-major B (EPI_NONE_BMN): k-blocks below kb_split come from tmB0, the rest from tmB1;
  // group g's K rows start at row g * bk_group of either tensor
  int kb_split;
  int bk_group;
  // row gather (groups along M): when set, row r of the grouped operand A is row
  // gather_src[r] / gather_div of the tensor tmA maps (the tokens x, with 1-row boxes), read
  // with 4-row gathers straight into the ring: the grouped copy of the rows is never written
  const int32_t* gather_src;
  int gather_div;
  // adaptive k-split (EPI_NONE, groups along M): when the launch's tiles fill fewer than half
  // of its CTAs, K is split (at most adapt_ks_max ways, within adapt_cap floats of fp32
  // partials [split][offsets[G]][N] at adapt_part) and the split count goes to *adapt_ks for
  // the summing kernel; otherwise bf16 out as usual and *adapt_ks = 1
  float* adapt_part;
  int64_t adapt_cap;
  int adapt_ks_max;
  int* adapt_ks;
  // EPI_F32 with two B tensors: n-tiles from b1_nt on read tmB1 (rows of n-tile n - b1_nt), so
  // one launch computes both the gate and the up product (0: one B tensor)
  int b1_nt;
  // stream-K (EPI_F32, groups along M): the tiles' k-blocks, tile by tile, are cut into equal
  // contiguous ranges, one per CTA; the part of a tile in CTA c's range is the tile's segment
  // c - (first CTA of the tile), written as fp32 partial slot `segment` (split_stride apart).
  // At most sk_slots segments per tile: the CTAs used are limited so that every range holds
  // at least ceil(nkb / (sk_slots - 1)) k-blocks.
  int streamk;
  int sk_slots;
};

// This CTA's stream-K range of k-blocks [lo, hi) of work = tiles * nkb, over g CTAs.
struct SkRange {
  bool on;
  int64_t lo, hi, work;
  int g;
};



// One work item of the persistent schedule.
struct Tile {
  int g, m, n_idx, m_idx, kb0, kb1, split;
  int64_t row0;   // first A row (and output row) of the group
  int kcol0;      // first k column of the group (groups along K)
};

// Work item t (k-split slowest, then group, n-tile, m-tile); g caches the group search.
template <int TBM, int KB>
__device__ __forceinline__ Tile locate(int t, int total, int nkb, int kchunk, const GemmParams& p,
                                       const int* grp_off, const int* tile_pre, int& g) {
  Tile r;
  r.split = t / total;
  const int tile = t - r.split * total;
  if (tile < tile_pre[g]) g = 0;
  while (tile >= tile_pre[g + 1]) ++g;
  r.g = g;
  if (p.kgroup) {
    r.m = (int)p.rows;
    r.row0 = 0;
    r.kcol0 = grp_off[g];
    r.kb0 = 0;
    r.kb1 = (grp_off[g + 1] - grp_off[g]) / KB;
  } else {
    r.m = grp_off[g + 1] - grp_off[g];
    r.row0 = grp_off[g];
    r.kcol0 = 0;
    r.kb0 = r.split * kchunk;
    r.kb1 = min(nkb, r.kb0 + kchunk);
  }
  const int mt = (r.m + TBM - 1) / TBM;
  const int local = tile - tile_pre[g];
  r.n_idx = local / mt;
  r.m_idx = local - r.n_idx * mt;
  return r;
}

// Work item j of this CTA: the tile t = blockIdx.x + j * gridDim.x of the round-robin schedule,
// or under stream-K the j-th tile its range touches, with that segment's k-blocks and slot.
template <int TBM, int KB>
__device__ __forceinline__ bool item_tile(int j, const SkRange& sk, int total_all, int total,
                                          int nkb, int kchunk, const GemmParams& p,
                                          const int* grp_off, const int* tile_pre, int& g,
                                          Tile& tl) {
  if (!sk.on) {
    const int t = (int)blockIdx.x + j * (int)gridDim.x;
    if (t >= total_all) return false;
    tl = locate<TBM, KB>(t, total, nkb, kchunk, p, grp_off, tile_pre, g);
    return true;
  }
  if (sk.hi <= sk.lo) return false;
  const int t = (int)(sk.lo / nkb) + j;
  if (t > (int)((sk.hi - 1) / nkb)) return false;
  tl = locate<TBM, KB>(t, total, nkb, nkb, p, grp_off, tile_pre, g);
  const int64_t base = (int64_t)t * nkb;
  tl.kb0 = (int)((sk.lo > base ? sk.lo : base) - base);
  tl.kb1 = (int)((sk.hi < base + nkb ? sk.hi : base + nkb) - base);
  tl.split = (int)blockIdx.x - streamk_owner(base, sk.work, sk.g);
  return true;
}

// Shared -> global tile store through a 3-D tensor map (x = column, y = row, z = group); the
// copy joins the issuing thread's current bulk group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y,
                                             int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's bulk groups are still reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all of this thread's bulk groups have completed (their writes are done).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the TMA (async proxy).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory matrix descriptor, MN-major operand with 128-byte swizzle: 64 MN-elements
// (128 B) per row, 8-row (K) groups 1024 B apart (stride byte offset), 64-element MN blocks
// 8192 B apart (leading byte offset: one 64 x 64 TMA box each).
__device__ __forceinline__ uint64_t sdesc_mn(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);        // start address
  d |= (uint64_t)(8192 >> 4) << 16;                 // leading byte offset: next MN block
  d |= (uint64_t)(1024 >> 4) << 32;                 // stride byte offset: next 8 K rows
  d |= (uint64_t)1 << 46;                           // descriptor version for tcgen05
  d |= (uint64_t)2 << 61;                           // 128-byte swizzle
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// SiLU(gate) * up of 32 accumulator columns -> 32 bf16 at dst (16-byte aligned).
__device__ __forceinline__ void store_swiglu32(const uint32_t (&gv)[32], const uint32_t (&uv)[32],
                                               __nv_bfloat16* dst) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float g0 = __uint_as_float(gv[2 * i]), g1 = __uint_as_float(gv[2 * i + 1]);
    const float u0 = __uint_as_float(uv[2 * i]), u1 = __uint_as_float(uv[2 * i + 1]);
    const float h0 = __fdividef(g0, 1.0f + __expf(-g0)) * u0;
    const float h1 = __fdividef(g1, 1.0f + __expf(-g1)) * u1;
    pk[i] = pack_bf16(h0, h1);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  d[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  d[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
  d[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
}

// act(acc) of 32 accumulator columns -> 32 bf16 at dst (EPI_RELU, EPI_GELU or EPI_NONE).
template <int EPI>
__device__ __forceinline__ void store_act32(const uint32_t (&v)[32], __nv_bfloat16* dst) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float a0 = __uint_as_float(v[2 * i]), a1 = __uint_as_float(v[2 * i + 1]);
    if (EPI == EPI_RELU) {
      a0 = fmaxf(a0, 0.f);
      a1 = fmaxf(a1, 0.f);
    } else if (EPI == EPI_GELU) {
      a0 = 0.5f * a0 * (1.0f + erff(a0 * 0.70710678118654752f));
      a1 = 0.5f * a1 * (1.0f + erff(a1 * 0.70710678118654752f));
    }
    pk[i] = pack_bf16(a0, a1);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  d[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  d[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
  d[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr)
               : "memory");
}
// TMA box into this CTA's shared memory; completion is counted on the mbarrier at cluster
// address bar_cl, which may be the peer CTA's (the pair's leader).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar_cl, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cl), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b,
                                               uint32_t acc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
// Arrive on the mbarrier at this offset in both CTAs of the pair once the MMAs issued so far
// have completed.
__device__ __forceinline__ void umma_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"((unsigned short)3)
      : "memory");
}
__device__ __forceinline__ void umma_commit_pair_local(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// HALVES = 1: 128-row tiles, 4-stage ring of 48 KB, two 256-column TMEM accumulators (the
//             epilogue of one tile overlaps the next tile's main loop), 4 epilogue warps.
// HALVES = 2: 256-row tiles made of two M=128 MMAs that share every B stage (a third fewer
//             L2->SMEM bytes per FLOP), 3-stage ring of 64 KB, one 512-column accumulator set,
//             8 epilogue warps; a tile with <= 128 live rows loads and multiplies one half only.
// tmB1 is the second B operand (SwiGLU, EPI_RAW, EPI_NONE_BMN) or, for EPI_F32_TMA, the fp32
// output map: [groups][rows][N], boxes of 16 columns x 32 rows, 64-byte swizzle.
// RB: A rows per half (128; 64 for products of a few rows, whose 128-row boxes would be mostly
// rows past the end: half the A bytes per stage, one more stage of weights in flight).
template <int EPI, int HALVES, int KB, int NSTAGES, int RB = BM>
__global__ void __launch_bounds__(64 + 128 * HALVES, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const GemmParams p) {
  constexpr int TBM = RB * HALVES;
  constexpr int TSTAGES = NSTAGES;
  constexpr int HA_BYTES = RB * KB * 2;              // one half of A per stage
  constexpr int TA_BYTES = HALVES * HA_BYTES;
  constexpr int TB_BYTES = MMA_N * KB * 2;           // B per stage
  constexpr int NBUF = HALVES == 1 ? 2 : 1;          // TMEM accumulator buffers
  constexpr int BUF_COLS = HALVES * ACC_COLS;        // columns per buffer
  constexpr int N_EPI = 4 * HALVES;                  // epilogue warps
  // EPI_F32_TMA: two 2 KB staging buffers (32 rows x 16 fp32) per epilogue warp
  constexpr int STG_BYTES = EPI == EPI_F32_TMA ? N_EPI * 2 * 2048 : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + TSTAGES * TA_BYTES;
  const uint32_t sStg = sB + TSTAGES * TB_BYTES;     // 1024-byte aligned (the ring is)
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(smem + TSTAGES * (TA_BYTES + TB_BYTES) + STG_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + TSTAGES;
  uint64_t* tfull = bars + 2 * TSTAGES;
  uint64_t* tempty = tfull + NBUF;
  uint64_t* drain = tempty + NBUF;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* grp_off = reinterpret_cast<int*>(tmem_holder + 2);   // [G+1]
  int* tile_pre = grp_off + (p.G + 1);                      // [G+1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < NBUF; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], N_EPI * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB0)) : "memory");
    if (EPI == EPI_SWIGLU || EPI == EPI_RAW || EPI == EPI_F32_TMA)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB1)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // everything above is set-up of this CTA's own shared memory and tensor memory; the group
  // table and the operands were written by earlier kernels
  pdl_trigger();
  pdl_wait();
  if (warp == 2 && p.kgroup) {
    // groups along K: every group has the same ceil(rows / TBM) * nt tiles
    const int per = (int)((p.rows + TBM - 1) / TBM) * p.nt;
    for (int g = lane; g <= p.G; g += 32) {
      grp_off[g] = p.kgroup[g];
      tile_pre[g] = g * per;
    }
  } else if (warp == 2) {
    // group row starts and the tile prefix (tiles of group g = ceil(rows_g / BM) * nt)
    int carry = 0;
    if (lane == 0) {
      grp_off[0] = p.offsets ? p.offsets[0] : 0;
      tile_pre[0] = 0;
    }
    for (int g0 = 0; g0 < p.G; g0 += 32) {
      const int g = g0 + lane;
      int tiles = 0;
      if (g < p.G) {
        // no offsets array: one group of all allocated rows
        const int lo = p.offsets ? p.offsets[g] : 0;
        const int hi = p.offsets ? p.offsets[g + 1] : (int)p.rows;
        const int m = hi > lo ? hi - lo : 0;
        tiles = ((m + TBM - 1) / TBM) * p.nt;
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
  const int nkb = (p.K + KB - 1) / KB;
  int ksplit = p.ksplit, kchunk = p.kchunk;
  int64_t split_stride = p.split_stride;
  if (EPI == EPI_NONE && p.adapt_ks_max > 1) {
    // the same decision in every thread of every CTA (it depends on the group table only)
    const int64_t live = grp_off[p.G];
    int sk = (total > 0 && 2 * total <= (int)gridDim.x) ? (int)gridDim.x / total : 1;
    sk = min(sk, min(p.adapt_ks_max, nkb));
    while (sk > 1 && (int64_t)sk * live * p.N > p.adapt_cap) --sk;
    if (sk > 1) {
      kchunk = (nkb + sk - 1) / sk;
      sk = (nkb + kchunk - 1) / kchunk;            // every k-range non-empty
    } else {
      sk = 1;
      kchunk = nkb;
    }
    ksplit = sk;
    split_stride = live * p.N;
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.adapt_ks = sk;
  }
  const bool adapt_f32 = EPI == EPI_NONE && ksplit > 1;
  const int total_all = total * ksplit;            // k-splits are the slowest tile index
  SkRange sk{false, 0, 0, 0, 0};
  if (EPI == EPI_F32 && p.streamk) {
    sk.on = true;
    sk.work = (int64_t)total * nkb;
    sk.g = streamk_ctas(sk.work, nkb, p.sk_slots, (int)gridDim.x);
    if ((int)blockIdx.x < sk.g) {
      sk.lo = (int64_t)blockIdx.x * sk.work / sk.g;
      sk.hi = (int64_t)(blockIdx.x + 1) * sk.work / sk.g;
    }
  }

  if (warp == 0 && p.gather_src) {
    // ---------------- TMA producer, gathered rows of A ----------------
    // All 32 lanes walk the schedule.  Lane 0 waits for a free stage, arms it and loads B;
    // lane l loads rows 8 l .. 8 l + 7 of the tile's A block with two 4-row gathers (rows past
    // the group end read token row 0: computed, then discarded by the epilogue).
    constexpr int ROWB = KB * 2;                 // bytes of one A row in a stage
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, issued_par = 0;
    bool ok = true;
    int g = 0;
    Tile tl;
    for (int j = 0; ok && item_tile<TBM, KB>(j, sk, total_all, total, nkb, kchunk, p, grp_off,
                                            tile_pre, g, tl); ++j) {
      const int a_row = (int)tl.row0 + tl.m_idx * TBM;
      const int row_end = (int)tl.row0 + tl.m;
      const int b_row = tl.g * p.N + tl.n_idx * p.n_out_tile;
      const bool two = HALVES == 2 && (tl.m - tl.m_idx * TBM) > RB;
      const bool mine = 8 * lane < (two ? 2 * RB : RB);
      int src[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = a_row + 8 * lane + i;
        src[i] = (mine && r < row_end) ? __ldg(p.gather_src + r) / p.gather_div : 0;
      }
      for (int kb = tl.kb0; kb < tl.kb1; ++kb) {
        const int kx = kb * KB;
        int go = 1;
        if (lane == 0) {
          go = mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, DEVERR_TIMEOUT_TMA,
                         TIMEOUT_NS);
          if (go) mbar_expect_tx(&full[stage], (two ? 2 * HA_BYTES : HA_BYTES) + TB_BYTES);
        }
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) {
          ok = false;
          break;
        }
        const bool withhold = p.fault == 1 && blockIdx.x == 0 && j == 0 &&
                              kb == tl.kb0;     // test hook, as in the tiled producer below
        const uint32_t a_dst = sA + stage * TA_BYTES, b_dst = sB + stage * TB_BYTES;
        if (mine && !withhold) {
          tma_gather4(a_dst + (8 * lane) * ROWB, &tmA, &full[stage], kx, src[0], src[1], src[2],
                      src[3]);
          tma_gather4(a_dst + (8 * lane + 4) * ROWB, &tmA, &full[stage], kx, src[4], src[5],
                      src[6], src[7]);
        }
        if (lane == 0 && !withhold) {
          if (EPI == EPI_SWIGLU || EPI == EPI_RAW) {
            tma_load_2d(b_dst, &tmB0, &full[stage], kx, b_row);
            tma_load_2d(b_dst + TB_BYTES / 2, &tmB1, &full[stage], kx, b_row);
          } else {
            tma_load_2d(b_dst, &tmB0, &full[stage], kx, b_row);
            tma_load_2d(b_dst + TB_BYTES / 2, &tmB0, &full[stage], kx, b_row + 128);
          }
        }
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == TSTAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      // let the copies already in flight land before the CTA exits
      for (int s = 0; s < TSTAGES; ++s)
        if (issued & (1u << s))
          mbar_wait(&full[s], (issued_par >> s) & 1u, abort_flag, p.err, DEVERR_TIMEOUT_TMA,
                    DRAIN_NS, /*honor_abort=*/false);
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_par = 0;     // per stage: has a load, parity of the last one
      bool ok = true;
      int g = 0;
      Tile tl;
      for (int j = 0; ok && item_tile<TBM, KB>(j, sk, total_all, total, nkb, kchunk, p, grp_off,
                                              tile_pre, g, tl); ++j) {
        const int a_row = (int)tl.row0 + tl.m_idx * TBM;
        const bool b1 = EPI == EPI_F32 && p.b1_nt > 0 && tl.n_idx >= p.b1_nt;
        const int b_row = (p.kgroup ? 0 : tl.g * p.N) +
                          (tl.n_idx - (b1 ? p.b1_nt : 0)) * p.n_out_tile;
        const bool two = HALVES == 2 && (tl.m - tl.m_idx * TBM) > RB;
        const int kb0 = tl.kb0, kb1 = tl.kb1;
        for (int kb = kb0; kb < kb1; ++kb) {
          const int kx = tl.kcol0 + kb * KB;
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, DEVERR_TIMEOUT_TMA,
                         TIMEOUT_NS)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&full[stage], (two ? 2 * HA_BYTES : HA_BYTES) + TB_BYTES);
          if (p.fault == 1 && blockIdx.x == 0 && j == 0 && kb == kb0) {
            // test hook: the stage is armed but never loaded, so the MMA issuer's bounded
            // wait on it runs out; nothing is in flight for this stage
            issued |= 1u << stage;
            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
            if (++stage == TSTAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          const uint32_t a_dst = sA + stage * TA_BYTES, b_dst = sB + stage * TB_BYTES;
          tma_load_2d(a_dst, &tmA, &full[stage], kx, a_row);
          if (two) tma_load_2d(a_dst + HA_BYTES, &tmA, &full[stage], kx, a_row + RB);
          if (EPI == EPI_NONE_BMN) {
            // [K, N] boxes of 64 x 64: four N blocks of 64 for this k-block
            const bool hi = kb >= p.kb_split;
            const int krow = tl.g * p.bk_group + (hi ? kb - p.kb_split : kb) * KB;
            const int n0 = tl.n_idx * p.n_out_tile;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_2d(b_dst + j * (TB_BYTES / 4), hi ? &tmB1 : &tmB0, &full[stage], n0 + 64 * j,
                          krow);
          } else if (EPI == EPI_SWIGLU || EPI == EPI_RAW) {
            tma_load_2d(b_dst, &tmB0, &full[stage], kx, b_row);
            tma_load_2d(b_dst + TB_BYTES / 2, &tmB1, &full[stage], kx, b_row);
          } else {
            const CUtensorMap* mb = b1 ? &tmB1 : &tmB0;
            tma_load_2d(b_dst, mb, &full[stage], kx, b_row);
            tma_load_2d(b_dst + TB_BYTES / 2, mb, &full[stage], kx, b_row + 128);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == TSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let the copies already in flight land before the CTA exits
        for (int s = 0; s < TSTAGES; ++s)
          if (issued & (1u << s))
            mbar_wait(&full[s], (issued_par >> s) & 1u, abort_flag, p.err, DEVERR_TIMEOUT_TMA,
                      DRAIN_NS, /*honor_abort=*/false);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0, g = 0;
      Tile tl;
      for (int j = 0; ok && item_tile<TBM, KB>(j, sk, total_all, total, nkb, kchunk, p, grp_off,
                                              tile_pre, g, tl); ++j, ++it) {
        const int m = tl.m, m_idx = tl.m_idx;
        const bool two = HALVES == 2 && (m - m_idx * TBM) > RB;
        const int kb0 = tl.kb0, kb1 = tl.kb1;      // kb0 == kb1: an empty group along K
        // M = 64 for a half with at most 64 live rows
        const int live0 = min(RB, m - m_idx * TBM), live1 = min(RB, m - m_idx * TBM - RB);
        // MN-major B: the transpose-B bit (16) of the instruction descriptor
        const uint32_t bmaj = EPI == EPI_NONE_BMN ? (1u << 16) : 0u;
        const uint32_t idesc0 = (live0 <= 64 ? kIdesc64 : kIdesc) | bmaj;
        const uint32_t idesc1 = (live1 <= 64 ? kIdesc64 : kIdesc) | bmaj;
        const int acc = it % NBUF;
        const uint32_t acc_par = (uint32_t)(it / NBUF) & 1u;
        if (!mbar_wait(&tempty[acc], acc_par ^ 1u, abort_flag, p.err, DEVERR_TIMEOUT_MMA,
                       TIMEOUT_NS)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BUF_COLS);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, DEVERR_TIMEOUT_MMA,
                         TIMEOUT_NS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = sA + stage * TA_BYTES, b0 = sB + stage * TB_BYTES;
#pragma unroll
          for (int k = 0; k < KB / MMA_K; ++k) {
            // K-major: the k-step moves 32 bytes along each row; MN-major: 16 rows of 128 B
            const uint64_t bdesc = EPI == EPI_NONE_BMN ? sdesc_mn(b0 + k * MMA_K * 128)
                                                       : sdesc<KB>(b0 + k * MMA_K * 2);
            const uint32_t accum = (kb > kb0 || k > 0) ? 1u : 0u;
            umma_bf16(d_tmem, sdesc<KB>(a0 + k * MMA_K * 2), bdesc, accum, idesc0);
            if (two)
              umma_bf16(d_tmem + ACC_COLS, sdesc<KB>(a0 + HA_BYTES + k * MMA_K * 2), bdesc,
                        accum, idesc1);
          }
          umma_commit(&empty[stage]);       // frees the stage once these MMAs have read it
          if (++stage == TSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[acc]);   // accumulator ready for the epilogue
      }
      // all MMAs issued by this thread complete before the CTA releases TMEM
      umma_commit(drain);
      mbar_wait(drain, 0u, abort_flag, p.err, DEVERR_TIMEOUT_MMA, ok ? TIMEOUT_NS : DRAIN_NS,
                /*honor_abort=*/false);
    }
  } else {
    // ---------------- epilogue (warps 2 .. 2 + N_EPI) ----------------
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int half = (warp - 2) / 4;         // which 128-row half of the tile
    int g = 0, it = 0;
    uint32_t nstored = 0;                    // EPI_F32_TMA: staged blocks this warp has stored
    Tile tl;
    for (int j = 0; item_tile<TBM, KB>(j, sk, total_all, total, nkb, kchunk, p, grp_off, tile_pre,
                                       g, tl); ++j, ++it) {
      const int m = tl.m, n_idx = tl.n_idx, m_idx = tl.m_idx, split = tl.split;
      const bool zero = tl.kb1 <= tl.kb0;    // no k-blocks (empty group along K): the sum is 0
      const bool two = HALVES == 2 && (m - m_idx * TBM) > RB;
      const int acc = it % NBUF;
      const uint32_t acc_par = (uint32_t)(it / NBUF) & 1u;
      int okw = 1;
      if (lane == 0)
        okw = mbar_wait(&tfull[acc], acc_par, abort_flag, p.err, DEVERR_TIMEOUT_EPI, TIMEOUT_NS);
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      tc_fence_after();
      if (half == 1 && !two) {               // this half was not computed: nothing to drain
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        continue;
      }
      // rows of this half: M = 128 -> lane quarter q holds rows 32q + lane; M = 64 (at most 64
      // live rows) -> rows 16q + lane in the quarter's first 16 lanes
      const int live = min(RB, m - m_idx * TBM - half * RB);
      const bool m64 = live <= 64;
      const int row = half * RB + (m64 ? 16 * q + lane : 32 * q + lane);
      const int r = m_idx * TBM + row;
      const int64_t orow = tl.row0 + r;
      bool valid = r < m && (!m64 || lane < 16);
      if (valid && (orow < 0 || orow >= p.rows)) {
        atomicCAS(p.err, 0, DEVERR_BOUNDS);
        valid = false;
      }
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) +
                             (uint32_t)(acc * BUF_COLS + half * ACC_COLS);
      __nv_bfloat16* orow_ptr = p.out + orow * p.ldo + (int64_t)n_idx * p.n_out_tile;
      if (EPI == EPI_SWIGLU) {
        // two 32-column chunks of gate and up per TMEM wait
#pragma unroll 1
        for (int c = 0; c < 128; c += 64) {
          uint32_t g0[32], u0[32], g1[32], u1[32];
          tmem_ld32(taddr + c, g0);
          tmem_ld32(taddr + 128 + c, u0);
          tmem_ld32(taddr + c + 32, g1);
          tmem_ld32(taddr + 160 + c, u1);
          tmem_wait_ld();
          if (c == 64) {                     // last TMEM read of the tile: release the buffer
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
          }
          const int col = n_idx * p.n_out_tile + c;
          if (valid && col < p.N) store_swiglu32(g0, u0, orow_ptr + c);   // SiLU(g) * u
          if (valid && col + 32 < p.N) store_swiglu32(g1, u1, orow_ptr + c + 32);
          if (p.out2 && valid) {             // pre-activations for the backward pass
            __nv_bfloat16* o2 = p.out2 + orow * p.ldo2 + (int64_t)n_idx * 256 + c;
            if (col < p.N) {
              store_act32<EPI_NONE>(g0, o2);
              store_act32<EPI_NONE>(u0, o2 + 128);
            }
            if (col + 32 < p.N) {
              store_act32<EPI_NONE>(g1, o2 + 32);
              store_act32<EPI_NONE>(u1, o2 + 160);
            }
          }
        }
      } else if (EPI == EPI_RAW) {
        // the raw gate | up accumulators of the tile as bf16: row pitch ldo, tile n at 256 n
        __nv_bfloat16* o = p.out + orow * p.ldo + (int64_t)n_idx * 2 * p.n_out_tile;
#pragma unroll 1
        for (int c = 0; c < MMA_N; c += 128) {
          uint32_t v0[32], v1[32], v2[32], v3[32];
          tmem_ld32(taddr + c, v0);
          tmem_ld32(taddr + c + 32, v1);
          tmem_ld32(taddr + c + 64, v2);
          tmem_ld32(taddr + c + 96, v3);
          tmem_wait_ld();
          if (c == MMA_N - 128) {            // last TMEM read of the tile: release the buffer
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
          }
          const int f = n_idx * p.n_out_tile + (c & 127);   // feature of the chunk's first column
          if (valid && f < p.N) store_act32<EPI_NONE>(v0, o + c);
          if (valid && f + 32 < p.N) store_act32<EPI_NONE>(v1, o + c + 32);
          if (valid && f + 64 < p.N) store_act32<EPI_NONE>(v2, o + c + 64);
          if (valid && f + 96 < p.N) store_act32<EPI_NONE>(v3, o + c + 96);
        }
      } else if (EPI == EPI_F32 || EPI == EPI_F32_TMA) {
        // fp32 partial of this k-split, rows of out32 + split * split_stride (+ the group's
        // output block when groups run along K)
        float* orow32 = reinterpret_cast<float*>(p.out) + split * split_stride +
                        (p.kgroup ? (int64_t)tl.g * p.out_gstride : 0) + orow * p.ldo +
                        (int64_t)n_idx * p.n_out_tile;
        // TMA stores need the warp's 32 rows in its 32 lanes: a tile of at most 64 live rows
        // (M = 64 MMA, 16 rows per lane quarter) keeps the per-thread stores
        const bool staged = EPI == EPI_F32_TMA && !m64;
#pragma unroll 1
        for (int c = 0; c < MMA_N; c += 32) {
          uint32_t v[32];
          if (!zero) {
            tmem_ld32(taddr + c, v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          if (c == MMA_N - 32) {             // last TMEM read of the tile: release the buffer
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
          }
          const int col = n_idx * p.n_out_tile + c;
          // column within its product (two B tensors: the second product's block starts at
          // n-tile b1_nt)
          const int pcol = (EPI == EPI_F32 && p.b1_nt > 0 && n_idx >= p.b1_nt)
                               ? col - p.b1_nt * p.n_out_tile
                               : col;
          if (staged) {
            if (col >= p.N) continue;        // warp-uniform: the chunk lies past the last column
            // two 16-column halves, each staged in buffer (nstored & 1) of this warp (2 KB: 32
            // rows of 64 B) and written by one TMA store; the store that used the buffer two
            // halves ago must have finished reading it
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t buf = sStg + (uint32_t)((((warp - 2) << 1) | (nstored & 1)) << 11);
              if (lane == 0) bulk_wait_read<1>();
              __syncwarp();
              // row `lane`, 16-byte chunk i at chunk position i ^ ((lane / 2) % 4): the 64-byte
              // swizzle the tensor map names (conflict-free: a phase of 8 lanes covers the 8
              // distinct 16-byte bank groups)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint32_t a =
                    buf + (uint32_t)(lane << 6) + (uint32_t)((i ^ ((lane >> 1) & 3)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                             "r"(v[16 * h + 4 * i]), "r"(v[16 * h + 4 * i + 1]),
                             "r"(v[16 * h + 4 * i + 2]), "r"(v[16 * h + 4 * i + 3])
                             : "memory");
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_3d(&tmB1, buf, col + 16 * h, m_idx * TBM + half * RB + 32 * q, tl.g);
                bulk_commit();
              }
              ++nstored;
            }
          } else if (valid && pcol < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(orow32 + c);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      } else if (EPI == EPI_NONE && adapt_f32) {
        // adaptive k-split: this split's fp32 partial, rows of adapt_part + split * stride
        float* orow32 = p.adapt_part + split * split_stride + orow * p.N +
                        (int64_t)n_idx * p.n_out_tile;
#pragma unroll 1
        for (int c = 0; c < MMA_N; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_wait_ld();
          if (c == MMA_N - 32) {             // last TMEM read of the tile: release the buffer
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
          }
          const int col = n_idx * p.n_out_tile + c;
          if (valid && col < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(orow32 + c);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      } else {
        // four 32-column chunks per TMEM wait
#pragma unroll 1
        for (int c = 0; c < MMA_N; c += 128) {
          uint32_t v0[32], v1[32], v2[32], v3[32];
          tmem_ld32(taddr + c, v0);
          tmem_ld32(taddr + c + 32, v1);
          tmem_ld32(taddr + c + 64, v2);
          tmem_ld32(taddr + c + 96, v3);
          tmem_wait_ld();
          if (c == MMA_N - 128) {            // last TMEM read of the tile: release the buffer
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
          }
          const int col = n_idx * p.n_out_tile + c;
          if (valid && col < p.N) store_act32<EPI>(v0, orow_ptr + c);
          if (valid && col + 32 < p.N) store_act32<EPI>(v1, orow_ptr + c + 32);
          if (valid && col + 64 < p.N) store_act32<EPI>(v2, orow_ptr + c + 64);
          if (valid && col + 96 < p.N) store_act32<EPI>(v3, orow_ptr + c + 96);
          if (p.out2 && valid) {             // pre-activations for the backward pass
            __nv_bfloat16* o2 = p.out2 + orow * p.ldo2 + (int64_t)n_idx * p.n_out_tile + c;
            if (col < p.N) store_act32<EPI_NONE>(v0, o2);
            if (col + 32 < p.N) store_act32<EPI_NONE>(v1, o2 + 32);
            if (col + 64 < p.N) store_act32<EPI_NONE>(v2, o2 + 64);
            if (col + 96 < p.N) store_act32<EPI_NONE>(v3, o2 + 96);
          }
        }
      }
    }
    // the TMA stores this warp issued complete before the kernel ends
    if (EPI == EPI_F32_TMA && lane == 0) bulk_wait_all();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ---------------- CTA-pair variant: tcgen05 cta_group::2, 256 x 512 tiles ----------------
//
// A cluster of two CTAs on neighbouring SMs computes each tile of 256 rows x 512 accumulator
// columns with pairs of N=256 MMAs (M=256: CTA r supplies tile rows 128r .. 128r+127 of A; the
// B operand of each MMA is split by rows, 128 per CTA); the leader (r = 0) issues the MMAs,
// which read both CTAs' stages and leave each CTA's 128 rows x 512 fp32 columns in that CTA's
// tensor memory.  Per SM and 64-element k-block the ring then moves 48 KB (128 A rows + 256 B
// rows) for 128 x 512 x 64 multiply-adds: three quarters of the operand bytes per FLOP of a
// 256 x 256 tile, which matters because the TMA/L2 path feeds an SM only ~30 B per clock while
// a 256 x 256 tile needs 44 B per clock at the full tensor rate.  TMEM is full, so the epilogue
// (8 warps: 4 lane quarters x 2 column halves) is not overlapped with the next tile's MMAs.
// A tile with at most 128 live rows runs M=128 MMAs (64 rows per CTA) instead; their
// accumulator holds a CTA's 64 rows in TMEM lanes 0-63 for the MMA's columns [0,128) and again
// in lanes 64-127 for its columns [128,256), both at TMEM columns [0,128) of the MMA.
// MMA j (j = 0, 1) writes TMEM columns [256j, 256j + 256); its B rows, 128 from each CTA, are
//   SwiGLU:    for features f = n0 + 128j + 64r .. +63 of CTA r, 64 W_gate rows then the same
//              64 W_up rows (64-row boxes), so that gate and up of a feature share a TMEM lane
//              in both accumulator layouts: MMA column 128r + x is gate and 128r + 64 + x up
//              of feature n0 + 128j + 64r + x;
//   otherwise: W rows n0 + 256j + 128r .. +127 of CTA r: MMA column c is output column
//              n0 + 256j + c.
// Barriers: full[s] is used on the leader (its producer arms it with both CTAs' bytes, and both
// CTAs' TMA loads complete on it); empty[s] and tfull exist in both CTAs and the leader's
// tcgen05.commit arrives on both; tempty is used on the leader and takes one arrive per
// epilogue warp of both CTAs.  Waits on barriers the peer arrives on acquire at cluster scope.
constexpr uint32_t kIdescPair256 = (1u << 4) | (1u << 7) | (1u << 10) |
                                   ((uint32_t)(MMA_N >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
constexpr uint32_t kIdescPair128 = (1u << 4) | (1u << 7) | (1u << 10) |
                                   ((uint32_t)(MMA_N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
constexpr int kPairEpiWarps = 8;
constexpr int kPairThreads = 64 + 32 * kPairEpiWarps;

template <int EPI, int NSTAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB0,
                         const __grid_constant__ CUtensorMap tmB1, const GemmParams p) {
  constexpr int KB = 64;
  constexpr int TBM = 2 * BM;                      // rows of a pair tile
  constexpr int A_BYTES = BM * KB * 2;             // this CTA's A box per stage
  constexpr int BH_BYTES = 128 * KB * 2;           // one 128-row B box
  constexpr int B_BYTES = 2 * BH_BYTES;            // this CTA's B rows of both MMAs
  constexpr uint32_t STAGE_TX = 2 * (A_BYTES + B_BYTES);   // both CTAs, counted on the leader
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + NSTAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NSTAGES * (A_BYTES + B_BYTES));
  uint64_t* full = bars;
  uint64_t* empty = bars + NSTAGES;
  uint64_t* tfull = bars + 2 * NSTAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* grp_off = reinterpret_cast<int*>(tmem_holder + 2);   // [G+1]
  int* tile_pre = grp_off + (p.G + 1);                      // [G+1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 2 * kPairEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB0)) : "memory");
    if (EPI == EPI_SWIGLU)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB1)) : "memory");
  }
  if (warp == 1) {
    // both CTAs allocate together: the pair's MMAs write the same columns in each
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (warp == 2) {
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
        tiles = ((m + TBM - 1) / TBM) * p.nt;
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
  // barriers initialised and TMEM allocated in both CTAs before either touches the other
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = tile_pre[p.G];
  const int nkb = (p.K + KB - 1) / KB;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_par = 0;
      bool ok = true;
      int g = 0;
      for (int t = pair; t < total && ok; t += n_pairs) {
        if (t < tile_pre[g]) g = 0;
        while (t >= tile_pre[g + 1]) ++g;
        const int m = grp_off[g + 1] - grp_off[g];
        const int mt = (m + TBM - 1) / TBM;
        const int local = t - tile_pre[g];
        const int n_idx = local / mt, m_idx = local - n_idx * mt;
        const bool m128 = m - m_idx * TBM <= BM;        // M=128 MMAs: 64 rows per CTA
        const int a_row = grp_off[g] + m_idx * TBM + (int)rank * (m128 ? 64 : BM);
        // SwiGLU: first feature of this CTA's rows of MMA 0 (MMA 1: + 128); otherwise the
        // first W row of this CTA's rows of MMA 0 (MMA 1: + 256)
        const int b_row0 = g * p.N + n_idx * p.n_out_tile + (int)rank * (EPI == EPI_SWIGLU ? 64 : 128);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait<true>(&empty[stage], phase ^ 1u, abort_flag, p.err, DEVERR_TIMEOUT_TMA,
                               TIMEOUT_NS)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_expect_tx(&full[stage], STAGE_TX);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (!(p.fault == 1 && rank == 0 && pair == 0 && t == pair && kb == 0)) {
            // (test hook: the leader of pair 0 arms its first stage without loading its
            // share, so the MMA issuer's bounded wait on that stage runs out)
            const uint32_t bar = cluster_map(smem_u32(&full[stage]), 0);
            const uint32_t b_dst = sB + stage * B_BYTES;
            tma_load_2d_pair(sA + stage * A_BYTES, &tmA, bar, kb * KB, a_row);
            if (EPI == EPI_SWIGLU) {          // 64-row boxes: gate, up of MMA 0, then MMA 1
              tma_load_2d_pair(b_dst, &tmB0, bar, kb * KB, b_row0);
              tma_load_2d_pair(b_dst + BH_BYTES / 2, &tmB1, bar, kb * KB, b_row0);
              tma_load_2d_pair(b_dst + BH_BYTES, &tmB0, bar, kb * KB, b_row0 + 128);
              tma_load_2d_pair(b_dst + 3 * BH_BYTES / 2, &tmB1, bar, kb * KB, b_row0 + 128);
            } else {
              tma_load_2d_pair(b_dst, &tmB0, bar, kb * KB, b_row0);
              tma_load_2d_pair(b_dst + BH_BYTES, &tmB0, bar, kb * KB, b_row0 + 256);
            }
          }
          if (++stage == NSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        if (rank == 0) {
          // let the copies already in flight land before the CTA moves on
          for (int s = 0; s < NSTAGES; ++s)
            if (issued & (1u << s))
              mbar_wait<true>(&full[s], (issued_par >> s) & 1u, abort_flag, p.err,
                              DEVERR_TIMEOUT_TMA, DRAIN_NS, /*honor_abort=*/false);
        } else {
          // this CTA's copies complete on the leader's barriers: give them a fixed time
          const uint64_t t0 = gtimer();
          while (gtimer() - t0 < DRAIN_NS / 100) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader only) ----------------
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0, g = 0;
      for (int t = pair; t < total && ok; t += n_pairs, ++it) {
        if (t < tile_pre[g]) g = 0;
        while (t >= tile_pre[g + 1]) ++g;
        const int m = grp_off[g + 1] - grp_off[g];
        const int mt = (m + TBM - 1) / TBM;
        const int m_idx = (t - tile_pre[g]) % mt;
        const uint32_t idesc = (m - m_idx * TBM <= BM) ? kIdescPair128 : kIdescPair256;
        if (!mbar_wait<true>(tempty, ((uint32_t)it & 1u) ^ 1u, abort_flag, p.err,
                             DEVERR_TIMEOUT_MMA, TIMEOUT_NS)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait<true>(&full[stage], phase, abort_flag, p.err, DEVERR_TIMEOUT_MMA,
                               TIMEOUT_NS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = sA + stage * A_BYTES, b0 = sB + stage * B_BYTES;
#pragma unroll
          for (int k = 0; k < KB / MMA_K; ++k) {
            const uint64_t adesc = sdesc<KB>(a0 + k * MMA_K * 2);
            const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
            umma_bf16_pair(tmem_base, adesc, sdesc<KB>(b0 + k * MMA_K * 2), accum, idesc);
            umma_bf16_pair(tmem_base + ACC_COLS, adesc,
                           sdesc<KB>(b0 + BH_BYTES + k * MMA_K * 2), accum, idesc);
          }
          umma_commit_both(&empty[stage]);  // frees the stage in both CTAs once read
          if (++stage == NSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit_both(tfull);    // both CTAs' accumulators are ready
      }
      umma_commit_pair_local(drain);
      mbar_wait(drain, 0u, abort_flag, p.err, DEVERR_TIMEOUT_MMA, ok ? TIMEOUT_NS : DRAIN_NS,
                /*honor_abort=*/false);
    }
  } else {
    // ---------------- epilogue (warps 2..9 of both CTAs) ----------------
    // warp (q, j): TMEM lane quarter q = warp % 4 of MMA j's accumulator columns.
    //   M=256: rows 32q + lane of this CTA's 128; SwiGLU features n0 + 128j .. +127 (gate at
    //          MMA columns x and 64 + x for x < 64, 128 + x' and 192 + x' for the next 64),
    //          otherwise output columns n0 + 256j .. +255.
    //   M=128: rows 32(q % 2) + lane of this CTA's 64; quarters 2 and 3 hold the MMA's upper
    //          128 columns: SwiGLU features n0 + 128j + 64(q / 2) .. +63, otherwise output
    //          columns n0 + 256j + 128(q / 2) .. +127.
    const int q = warp & 3;
    const int j = (warp - 2) >> 2;
    int g = 0, it = 0;
    for (int t = pair; t < total; t += n_pairs, ++it) {
      if (t < tile_pre[g]) g = 0;
      while (t >= tile_pre[g + 1]) ++g;
      const int m = grp_off[g + 1] - grp_off[g];
      const int mt = (m + TBM - 1) / TBM;
      const int local = t - tile_pre[g];
      const int n_idx = local / mt, m_idx = local - n_idx * mt;
      int okw = 1;
      if (lane == 0)
        okw = mbar_wait<true>(tfull, (uint32_t)it & 1u, abort_flag, p.err, DEVERR_TIMEOUT_EPI,
                              TIMEOUT_NS);
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      tc_fence_after();
      const uint32_t release = cluster_map(smem_u32(tempty), 0);
      const bool m128 = m - m_idx * TBM <= BM;
      const int r0 = m_idx * TBM + (int)rank * (m128 ? 64 : BM);
      if (r0 >= m) {                                    // no live rows here: nothing to read
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(release);
        continue;
      }
      const int r = r0 + 32 * (m128 ? (q & 1) : q) + lane;
      const int64_t orow = (int64_t)grp_off[g] + r;
      bool valid = r < m;
      if (valid && (orow < 0 || orow >= p.rows)) {
        atomicCAS(p.err, 0, DEVERR_BOUNDS);
        valid = false;
      }
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(j * ACC_COLS);
      __nv_bfloat16* orow_ptr = p.out + orow * p.ldo;
      if (EPI == EPI_SWIGLU) {
        const int nch = m128 ? 2 : 4;
        const int f0 = n_idx * p.n_out_tile + 128 * j + (m128 ? 64 * (q >> 1) : 0);
        // chunks i, i+1 (gate at MMA column 32i (+64 from i = 2), up 64 further) per wait
#pragma unroll 1
        for (int i = 0; i < nch; i += 2) {
          const int gc = 32 * i + (i >= 2 ? 64 : 0);
          uint32_t g0[32], u0[32], g1[32], u1[32];
          tmem_ld32(taddr + gc, g0);
          tmem_ld32(taddr + gc + 64, u0);
          tmem_ld32(taddr + gc + 32, g1);
          tmem_ld32(taddr + gc + 96, u1);
          tmem_wait_ld();
          if (i + 2 >= nch) {                // last TMEM read of the tile: release it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(release);
          }
          const int f = f0 + 32 * i;
          if (valid && f < p.N) store_swiglu32(g0, u0, orow_ptr + f);
          if (valid && f + 32 < p.N) store_swiglu32(g1, u1, orow_ptr + f + 32);
        }
      } else {
        const int nch = m128 ? 4 : 8;
        const int c0 = n_idx * p.n_out_tile + 256 * j + (m128 ? 128 * (q >> 1) : 0);
        // four 32-column chunks per wait
#pragma unroll 1
        for (int i = 0; i < nch; i += 4) {
          uint32_t v0[32], v1[32], v2[32], v3[32];
          tmem_ld32(taddr + 32 * i, v0);
          tmem_ld32(taddr + 32 * i + 32, v1);
          tmem_ld32(taddr + 32 * i + 64, v2);
          tmem_ld32(taddr + 32 * i + 96, v3);
          tmem_wait_ld();
          if (i + 4 >= nch) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(release);
          }
          const int c = c0 + 32 * i;
          if (valid && c < p.N) store_act32<EPI>(v0, orow_ptr + c);
          if (valid && c + 32 < p.N) store_act32<EPI>(v1, orow_ptr + c + 32);
          if (valid && c + 64 < p.N) store_act32<EPI>(v2, orow_ptr + c + 64);
          if (valid && c + 96 < p.N) store_act32<EPI>(v3, orow_ptr + c + 96);
        }
      }
    }
  }
  // neither CTA leaves (or frees TMEM) while the other may still touch its shared or tensor
  // memory: the leader's MMAs read the peer's stages and write its TMEM, the peer's loads and
  // arrives target the leader's barriers
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ---------------- host side ----------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3D fp32 tensor [groups][rows][cols] (dense); box = 16 columns x 32 rows x 1 group, 64-byte
// swizzle (one 64-byte row of the box per swizzle row): the EPI_F32_TMA output.
bool make_map_f32_out(CUtensorMap* m, void* ptr, uint64_t groups, uint64_t rows, uint64_t cols) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {cols, rows, groups};
  const cuuint64_t strides[2] = {cols * 4, rows * cols * 4};
  const cuuint32_t box[3] = {16, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// Tile shape.  Default: 256-row tiles (two M=128 MMAs sharing each B stage: a third fewer L2
// bytes per FLOP than 128-row tiles) with 64-element k-blocks in a 3-stage ring.
// MOE_GEMM_TILE selects another shape for comparison measurements (all are tested):
//   "128"      128-row tiles, 4 stages, double TMEM buffer;
//   "256k32"   256-row tiles with 32-element k-blocks (64-byte swizzle) in a 6-7 stage ring;
//   "pair"     256 x 512 accumulator tiles on a CTA pair (cta_group::2), 4 stages of 48 KB
//              per CTA.
enum GemmTile { TILE_128 = 0, TILE_256 = 1, TILE_256_K32 = 2, TILE_PAIR = 3 };

int g_gemm_fault = 0;       // set through moe_debug_inject (tests of the bounded waits)
constexpr int kRouterMaxSplits = 8;
// -1: no MOE_GEMM_TILE in the environment (the shape is chosen per call, see tile_for).
int gemm_tile_env() {
  static int t = [] {
    const char* v = getenv("MOE_GEMM_TILE");
    if (v && !strcmp(v, "128")) return (int)TILE_128;
    if (v && !strcmp(v, "256")) return (int)TILE_256;
    if (v && !strcmp(v, "256k32")) return (int)TILE_256_K32;
    if (v && !strcmp(v, "pair")) return (int)TILE_PAIR;
    return -1;
  }();
  return t;
}
GemmTile gemm_tile() {
  const int t = gemm_tile_env();
  return t < 0 ? TILE_256 : (GemmTile)t;
}
int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Weights-as-M schedule (gemm_swap.cu), taken for every eligible call when MOE_GEMM_SWAP=1
// (unless MOE_GEMM_TILE names a row-tile shape).  Off by default: it measured slower than the
// row tiles at the DeepSeek-V3 shape (up 2.94 against 2.51 ms, down 1.81 against 1.72 ms) and
// at the Mixtral shape.  An M=128 MMA reads its 4 KB weight slice from shared memory whatever
// its N, so a token tile below ~128 rows needs more than the SM's 128 B per clock of shared
// memory bandwidth; the row tiles always run N = 256.
bool use_swap(int epi, bool grouped, bool out2, bool adapt) {
  static const bool on = [] {
    const char* e = getenv("MOE_GEMM_SWAP");
    return e && !strcmp(e, "1");
  }();
  return on && grouped && !out2 && !adapt && swap_epilogue_ok(epi) && gemm_tile_env() < 0;
}

// Per call.  Groups of at most 192 rows on average (DeepSeek-V3: T k / E = 128, Switch: at most
// the capacity) run 128-row tiles with two TMEM accumulators: they fill a 256-row tile's second
// half only partly and give each tile a short main loop whose epilogue one accumulator set
// cannot hide (V3 down projection 1.70 -> 1.61 ms).  Larger groups compare the two shapes by
// whole waves of persistent CTAs: tiles ~ (a_rows / TBM + n_groups / 2) * nt (each group's last
// tile counted as half full), a 128-row tile costing 0.6 of a 256-row one (half the rows, a
// fifth more time per row: more L2 bytes per FLOP, measured).  The 256-row tiles keep every
// Mixtral projection at T k >= 8192; the down projection (16 output tiles per group) takes the
// 128-row tiles at 1024 and 2048 tokens, where 256-row tiles leave a mostly idle last wave
// (measured: 365 -> 330 us and 531 -> 444 us).
GemmTile tile_for(int64_t a_rows, int n_groups, bool grouped, int nt) {
  const int t = gemm_tile_env();
  if (t >= 0) return (GemmTile)t;
  if (!grouped || n_groups < 1) return TILE_256;
  if (n_groups > 1 && a_rows / n_groups <= 192) return TILE_128;
  const int64_t sms = sm_count();
  const int64_t t256 = ((a_rows + 255) / 256 + n_groups / 2) * nt;
  const int64_t t128 = ((a_rows + 127) / 128 + n_groups / 2) * nt;
  const int64_t w256 = (t256 + sms - 1) / sms, w128 = (t128 + sms - 1) / sms;
  return 6 * w128 < 10 * w256 ? TILE_128 : TILE_256;
}


template <int EPI, int HALVES, int KB, int NSTAGES, int RB = BM>
cudaError_t launch_epi(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                       const GemmParams& p, int grid, size_t smem, cudaStream_t s) {
  auto kern = grouped_gemm_kernel<EPI, HALVES, KB, NSTAGES, RB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(64 + 128 * HALVES), smem, s, a, b0, b1, p);
}

template <int HALVES, int KB, int NSTAGES>
cudaError_t launch_cfg(int epi, const CUtensorMap& a, const CUtensorMap& b0,
                       const CUtensorMap& b1, const GemmParams& p, int grid, size_t smem,
                       cudaStream_t s) {
  switch (epi) {
    case EPI_SWIGLU: return launch_epi<EPI_SWIGLU, HALVES, KB, NSTAGES>(a, b0, b1, p, grid, smem, s);
    case EPI_RELU: return launch_epi<EPI_RELU, HALVES, KB, NSTAGES>(a, b0, b1, p, grid, smem, s);
    case EPI_F32: return launch_epi<EPI_F32, HALVES, KB, NSTAGES>(a, b0, b1, p, grid, smem, s);
    case EPI_GELU: return launch_epi<EPI_GELU, HALVES, KB, NSTAGES>(a, b0, b1, p, grid, smem, s);
    case EPI_RAW: return launch_epi<EPI_RAW, HALVES, KB, NSTAGES>(a, b0, b1, p, grid, smem, s);
    case EPI_NONE_BMN:
      return launch_epi<EPI_NONE_BMN, HALVES, KB, NSTAGES>(a, b0, b1, p, grid, smem, s);
    default: return launch_epi<EPI_NONE, HALVES, KB, NSTAGES>(a, b0, b1, p, grid, smem, s);
  }
}

// Dynamic shared memory of one configuration (ring + barriers + group tables + alignment).
// `staging`: the EPI_F32_TMA store buffers between the ring and the barriers.
size_t gemm_smem(int halves, int kb, int nstages, int n_groups, size_t staging = 0,
                 int rb = BM) {
  const size_t ring = (size_t)nstages * ((size_t)halves * rb * kb * 2 + (size_t)MMA_N * kb * 2);
  return 1024 + ring + staging + (2 * nstages + 5) * 8 + 8 +
         (size_t)2 * (n_groups + 1) * sizeof(int);
}

constexpr int kPairStages = 4;
size_t pair_smem(int nstages, int n_groups) {
  const size_t ring = (size_t)nstages * (3 * (size_t)128 * 64 * 2);   // A box + two B boxes
  return 1024 + ring + (2 * nstages + 3) * 8 + 8 + (size_t)2 * (n_groups + 1) * sizeof(int);
}

// Co-resident CTA pairs of one pair-kernel instance (queried once per device).
template <int EPI>
int pair_slots(size_t smem) {
  constexpr int kMaxDev = 64;
  static int cached[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < kMaxDev && cached[dev] > 0) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sm_count() / 2));
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = smem;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel<EPI, kPairStages>, &cfg) !=
          cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    n = sm_count() / 2;
  }
  if (dev >= 0 && dev < kMaxDev) cached[dev] = n;
  return n;
}

template <int EPI>
cudaError_t launch_pair_epi(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                            const GemmParams& p, int64_t max_tiles, cudaStream_t s) {
  auto kern = grouped_gemm_pair_kernel<EPI, kPairStages>;
  const size_t smem = pair_smem(kPairStages, p.G);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int slots = pair_slots<EPI>(smem);
  const int pairs = (int)(max_tiles < slots ? max_tiles : slots);
  kern<<<counted(2 * pairs), kPairThreads, smem, s>>>(a, b0, b1, p);
  return cudaGetLastError();
}

cudaError_t launch_pair(int epi, const CUtensorMap& a, const CUtensorMap& b0,
                        const CUtensorMap& b1, const GemmParams& p, int64_t max_tiles,
                        cudaStream_t s) {
  switch (epi) {
    case EPI_SWIGLU: return launch_pair_epi<EPI_SWIGLU>(a, b0, b1, p, max_tiles, s);
    case EPI_RELU: return launch_pair_epi<EPI_RELU>(a, b0, b1, p, max_tiles, s);
    case EPI_GELU: return launch_pair_epi<EPI_GELU>(a, b0, b1, p, max_tiles, s);
    default: return launch_pair_epi<EPI_NONE>(a, b0, b1, p, max_tiles, s);
  }
}

}  // namespace

// 2-D bf16 tensor map (declared in tc_ops.cuh).
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
              int kb) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kb, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             kb == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gemm_gather_ok() {
  const GemmTile t = gemm_tile();
  return t == TILE_256 || t == TILE_128;
}

cudaError_t launch_grouped_gemm_bf16(int epi, const void* A, int64_t a_rows, int K,
                                     const void* B0, const void* B1, int n_groups, int N,
                                     const int32_t* offsets, void* out, cudaStream_t s,
                                     void* out2, const int32_t* gather_src, int gather_div,
                                     int64_t src_rows, float* adapt_part, int64_t adapt_cap,
                                     int adapt_ks_max, int* adapt_ks) {
  if (a_rows <= 0 || n_groups <= 0) return cudaSuccess;
  if (gather_src && (!offsets || !gemm_gather_ok() || epi == EPI_NONE_BMN || gather_div < 1 ||
                     src_rows <= 0))
    return cudaErrorInvalidValue;
  const bool adapt = adapt_ks_max > 1;
  if (adapt && (epi != EPI_NONE || !offsets || out2 || gather_src || !adapt_part || !adapt_ks))
    return cudaErrorInvalidValue;
  if (use_swap(epi, offsets != nullptr, out2 != nullptr, adapt))
    return launch_grouped_gemm_swap(epi, A, a_rows, K, B0, B1, n_groups, N, offsets, out, s,
                                    gather_src, gather_div, src_rows, g_gemm_fault);
  alignas(64) CUtensorMap ta, tb0, tb1;
  const uint64_t brows = (uint64_t)n_groups * (uint64_t)N;
  GemmParams p{};
  p.offsets = offsets;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.err = device_error_word();
  p.rows = a_rows;
  p.ldo = N;
  p.G = n_groups;
  p.N = N;
  p.K = K;
  p.n_out_tile = (epi == EPI_SWIGLU || epi == EPI_RAW) ? 128 : 256;
  p.nt = (N + p.n_out_tile - 1) / p.n_out_tile;
  if (epi == EPI_RAW) p.ldo = (int64_t)p.nt * 256;     // gate | up blocks of 128 per n-tile
  p.kgroup = nullptr;
  p.out_gstride = 0;
  p.out2 = static_cast<__nv_bfloat16*>(out2);
  p.ldo2 = (epi == EPI_SWIGLU) ? (int64_t)p.nt * 256 : N;
  p.kb_split = 0;
  p.bk_group = 0;
  p.fault = g_gemm_fault;
  p.ksplit = 1;
  p.kchunk = 1 << 30;
  p.split_stride = 0;
  p.gather_src = gather_src;
  p.gather_div = gather_div;
  p.adapt_part = adapt_part;
  p.adapt_cap = adapt_cap;
  p.adapt_ks_max = adapt ? adapt_ks_max : 0;
  p.adapt_ks = adapt_ks;
  GemmTile tile = tile_for(a_rows, n_groups, offsets != nullptr, p.nt);
  if (adapt && tile == TILE_PAIR) tile = TILE_256;     // the pair kernel has no adaptive split
  const int halves = tile == TILE_128 ? 1 : 2;
  const int kb = tile == TILE_256_K32 ? 32 : 64;
  if (gather_src) {
    // A rows come from the token rows of A itself ([src_rows, K]) by 4-row gathers
    if (!make_map(&ta, A, (uint64_t)src_rows, (uint64_t)K, 1, kb)) return cudaErrorInvalidValue;
  } else if (!make_map(&ta, A, (uint64_t)a_rows, (uint64_t)K, 128, kb)) {
    return cudaErrorInvalidValue;
  }
  if (!make_map(&tb0, B0, brows, (uint64_t)K, 128, kb)) return cudaErrorInvalidValue;
  if (epi == EPI_SWIGLU || epi == EPI_RAW) {
    if (!make_map(&tb1, B1, brows, (uint64_t)K, 128, kb)) return cudaErrorInvalidValue;
  } else {
    tb1 = tb0;
  }
  const int tbm = tile == TILE_PAIR ? 2 * BM : BM * halves;
  const int64_t max_tiles = ((a_rows + tbm - 1) / tbm + n_groups) * (int64_t)p.nt;
  if (tile == TILE_PAIR && offsets && epi != EPI_RAW && !out2 && !gather_src) {
    // 256 x 512 accumulator tiles: 256 SwiGLU features (gate + up) or 512 output columns;
    // the SwiGLU weights go in 64-row boxes
    if (epi == EPI_SWIGLU && (!make_map(&tb0, B0, brows, (uint64_t)K, 64, kb) ||
                              !make_map(&tb1, B1, brows, (uint64_t)K, 64, kb)))
      return cudaErrorInvalidValue;
    p.n_out_tile = (epi == EPI_SWIGLU) ? 256 : 512;
    p.nt = (N + p.n_out_tile - 1) / p.n_out_tile;
    const int64_t pair_tiles = ((a_rows + 2 * BM - 1) / (2 * BM) + n_groups) * (int64_t)p.nt;
    return launch_pair(epi, ta, tb0, tb1, p, pair_tiles, s);
  }
  const int grid = (int)(max_tiles < sm_count() ? max_tiles : sm_count());
  constexpr size_t kMaxSmem = 232448;          // 227 KB of dynamic shared memory per block
  switch (tile) {
    case TILE_128:
      return launch_cfg<1, 64, 4>(epi, ta, tb0, tb1, p, grid, gemm_smem(1, 64, 4, n_groups), s);
    case TILE_256_K32:
      if (gemm_smem(2, 32, 7, n_groups) <= kMaxSmem)
        return launch_cfg<2, 32, 7>(epi, ta, tb0, tb1, p, grid, gemm_smem(2, 32, 7, n_groups), s);
      return launch_cfg<2, 32, 6>(epi, ta, tb0, tb1, p, grid, gemm_smem(2, 32, 6, n_groups), s);
    default:
      return launch_cfg<2, 64, 3>(epi, ta, tb0, tb1, p, grid, gemm_smem(2, 64, 3, n_groups), s);
  }
}

void set_gemm_fault(int kind) { g_gemm_fault = kind; }

cudaError_t launch_grouped_gemm_bf16_bmn(const void* A, int64_t a_rows, int K, const void* B0,
                                         const void* B1, int kb_split, int bk_group,
                                         int n_groups, int N, const int32_t* offsets, void* out,
                                         cudaStream_t s) {
  if (a_rows <= 0 || n_groups <= 0) return cudaSuccess;
  alignas(64) CUtensorMap ta, tb0, tb1;
  const uint64_t brows = (uint64_t)n_groups * (uint64_t)bk_group;
  if (!make_map(&ta, A, (uint64_t)a_rows, (uint64_t)K, 128, 64)) return cudaErrorInvalidValue;
  if (!make_map(&tb0, B0, brows, (uint64_t)N, 64, 64)) return cudaErrorInvalidValue;
  if (B1) {
    if (!make_map(&tb1, B1, brows, (uint64_t)N, 64, 64)) return cudaErrorInvalidValue;
  } else {
    tb1 = tb0;
  }
  GemmParams p{};
  p.offsets = offsets;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.err = device_error_word();
  p.rows = a_rows;
  p.ldo = N;
  p.G = n_groups;
  p.N = N;
  p.K = K;
  p.n_out_tile = 256;
  p.nt = (N + 255) / 256;
  p.fault = g_gemm_fault;
  p.ksplit = 1;
  p.kchunk = 1 << 30;
  p.split_stride = 0;
  p.kgroup = nullptr;
  p.out_gstride = 0;
  p.out2 = nullptr;
  p.ldo2 = 0;
  p.kb_split = kb_split;
  p.bk_group = bk_group;
  const int64_t max_tiles = ((a_rows + 2 * BM - 1) / (2 * BM) + n_groups) * (int64_t)p.nt;
  const int grid = (int)(max_tiles < sm_count() ? max_tiles : sm_count());
  return launch_epi<EPI_NONE_BMN, 2, 64, 3>(ta, tb0, tb1, p, grid, gemm_smem(2, 64, 3, n_groups),
                                            s);
}

// Weight-gradient tile shape.  Default: 256-row tiles (two M=128 MMAs share each B stage, so a
// k-block moves 64 B of operands per MMA clock instead of 96; one accumulator set, the epilogue
// is not overlapped).  MOE_WGRAD_TILE=128 selects 128-row tiles with two TMEM accumulators (the
// epilogue overlaps the next tile; tested, kept for comparison measurements).
bool wgrad_tile_128() {
  static const bool v = [] {
    const char* e = getenv("MOE_WGRAD_TILE");
    return e && !strcmp(e, "128");
  }();
  return v;
}

cudaError_t launch_grouped_gemm_kgroups_f32(const void* A, int M, const void* B, int N, int G,
                                            const int32_t* kgroup, int64_t k_total, float* out,
                                            cudaStream_t s) {
  if (M <= 0 || N <= 0 || G <= 0) return cudaSuccess;
  // The output needs 16-byte aligned rows: N a multiple of 4.
  if (N % 4 || (reinterpret_cast<uintptr_t>(out) & 15)) return cudaErrorInvalidValue;
  constexpr size_t kMaxSmem = 232448;          // 227 KB of dynamic shared memory per block
  const bool t128 = wgrad_tile_128();
  const int halves = t128 ? 1 : 2;
  const size_t staging = (size_t)4 * halves * 2 * 2048;   // two 2 KB buffers per epilogue warp
  // 64-element k-blocks unless the group tables of many experts leave no room for the ring;
  // then 32-element k-blocks (64-byte swizzle) in a deeper ring of smaller stages
  const bool k32 = !t128 && gemm_smem(2, 64, 3, G, staging) > kMaxSmem;
  const int kb = k32 ? 32 : 64;
  alignas(64) CUtensorMap ta, tb, to;
  if (!make_map(&ta, A, (uint64_t)M, (uint64_t)k_total, 128, kb)) return cudaErrorInvalidValue;
  if (!make_map(&tb, B, (uint64_t)N, (uint64_t)k_total, 128, kb)) return cudaErrorInvalidValue;
  if (!make_map_f32_out(&to, out, (uint64_t)G, (uint64_t)M, (uint64_t)N))
    return cudaErrorInvalidValue;
  GemmParams p{};
  p.offsets = nullptr;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.err = device_error_word();
  p.rows = M;
  p.ldo = N;
  p.G = G;
  p.N = N;
  p.K = (int)k_total;
  p.n_out_tile = 256;
  p.nt = (N + 255) / 256;
  p.fault = 0;
  p.ksplit = 1;
  p.kchunk = 1 << 30;
  p.split_stride = 0;
  p.kgroup = kgroup;
  p.out_gstride = (int64_t)M * N;
  p.out2 = nullptr;
  p.ldo2 = 0;
  p.kb_split = 0;
  p.bk_group = 0;
  const int tbm = BM * halves;
  const int64_t tiles = (int64_t)G * ((M + tbm - 1) / tbm) * p.nt;
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  if (t128) {
    if (gemm_smem(1, 64, 4, G, staging) <= kMaxSmem)
      return launch_epi<EPI_F32_TMA, 1, 64, 4>(ta, tb, to, p, grid,
                                               gemm_smem(1, 64, 4, G, staging), s);
    return launch_epi<EPI_F32_TMA, 1, 64, 3>(ta, tb, to, p, grid,
                                             gemm_smem(1, 64, 3, G, staging), s);
  }
  if (!k32)
    return launch_epi<EPI_F32_TMA, 2, 64, 3>(ta, tb, to, p, grid,
                                             gemm_smem(2, 64, 3, G, staging), s);
  return launch_epi<EPI_F32_TMA, 2, 32, 5>(ta, tb, to, p, grid, gemm_smem(2, 32, 5, G, staging),
                                           s);
}

// k-split fp32 partials of a grouped product with groups along M (the small-batch schedule,
// when a handful of executed rows leaves most SMs without a tile): out[s][r][n] = the sum over
// the k-blocks of split s of A[r, k] * B[g * N + n, k] for every row r of group g; split s
// covers k-blocks [s * kchunk, (s + 1) * kchunk), every split non-empty.  out is
// [ksplit][a_rows][N] fp32; only rows below offsets[G] are written.
// A rows per tile of the k-split products: with at most 64 rows in all (the decode schedule
// at up to 32 tokens of top-2), 64-row A boxes and a 5-stage ring (40 KB stages: 160 KB of
// weights in flight per SM instead of 128 KB with 128-row boxes, which are then mostly rows
// past the end that TMA fills without a memory access); otherwise 128 rows, 4 stages.
static int split_rows(int64_t a_rows) { return a_rows <= 64 ? 64 : BM; }

cudaError_t launch_grouped_gemm_f32_splitk(const void* A, int64_t a_rows, int K, const void* B,
                                           int G, int N, const int32_t* offsets, int ksplit,
                                           float* out, cudaStream_t s, int sk_slots) {
  if (a_rows <= 0 || G <= 0 || N <= 0 || ksplit < 1) return cudaSuccess;
  if (sk_slots > 0 && (split_rows(a_rows) != 64 || sk_slots < 2)) return cudaErrorInvalidValue;
  alignas(64) CUtensorMap ta, tb;
  const int rb = split_rows(a_rows);
  if (!make_map(&ta, A, (uint64_t)a_rows, (uint64_t)K, rb, 64)) return cudaErrorInvalidValue;
  if (!make_map(&tb, B, (uint64_t)G * N, (uint64_t)K, 128, 64)) return cudaErrorInvalidValue;
  GemmParams p{};
  p.offsets = offsets;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.err = device_error_word();
  p.rows = a_rows;
  p.ldo = N;
  p.G = G;
  p.N = N;
  p.K = K;
  p.n_out_tile = 256;
  p.nt = (N + 255) / 256;
  p.fault = 0;
  const int nkb = (K + 63) / 64;
  p.kchunk = (nkb + ksplit - 1) / ksplit;
  p.ksplit = splitk_count(K, ksplit);
  p.split_stride = a_rows * (int64_t)N;
  p.kgroup = nullptr;
  p.out_gstride = 0;
  p.out2 = nullptr;
  p.ldo2 = 0;
  p.kb_split = 0;
  p.bk_group = 0;
  p.streamk = sk_slots > 0;
  p.sk_slots = sk_slots;
  const int64_t tiles = ((a_rows + rb - 1) / rb + G) * (int64_t)p.nt * p.ksplit;
  const int grid = p.streamk ? sm_count() : (int)(tiles < sm_count() ? tiles : sm_count());
  if (rb == 64)
    return launch_epi<EPI_F32, 1, 64, 5, 64>(ta, tb, tb, p, grid,
                                             gemm_smem(1, 64, 5, G, 0, 64), s);
  return launch_epi<EPI_F32, 1, 64, 4>(ta, tb, tb, p, grid, gemm_smem(1, 64, 4, G), s);
}

cudaError_t launch_grouped_gemm_f32_splitk2(const void* A, int64_t a_rows, int K, const void* B0,
                                            const void* B1, int G, int N,
                                            const int32_t* offsets, int ksplit, float* out,
                                            cudaStream_t s, int sk_slots) {
  if (a_rows <= 0 || G <= 0 || N <= 0 || ksplit < 1) return cudaSuccess;
  if (sk_slots > 0 && (split_rows(a_rows) != 64 || sk_slots < 2)) return cudaErrorInvalidValue;
  alignas(64) CUtensorMap ta, tb0, tb1;
  const int rb = split_rows(a_rows);
  if (!make_map(&ta, A, (uint64_t)a_rows, (uint64_t)K, rb, 64)) return cudaErrorInvalidValue;
  if (!make_map(&tb0, B0, (uint64_t)G * N, (uint64_t)K, 128, 64)) return cudaErrorInvalidValue;
  if (!make_map(&tb1, B1, (uint64_t)G * N, (uint64_t)K, 128, 64)) return cudaErrorInvalidValue;
  const int half = (N + 255) / 256;               // n-tiles of one product
  GemmParams p{};
  p.offsets = offsets;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.err = device_error_word();
  p.rows = a_rows;
  p.ldo = (int64_t)2 * half * 256;                // [product 0 | product 1], 256-column tiles
  p.G = G;
  p.N = N;
  p.K = K;
  p.n_out_tile = 256;
  p.nt = 2 * half;
  p.b1_nt = half;
  p.fault = 0;
  const int nkb = (K + 63) / 64;
  p.kchunk = (nkb + ksplit - 1) / ksplit;
  p.ksplit = splitk_count(K, ksplit);
  p.split_stride = a_rows * p.ldo;
  p.streamk = sk_slots > 0;
  p.sk_slots = sk_slots;
  const int64_t tiles = ((a_rows + rb - 1) / rb + G) * (int64_t)p.nt * p.ksplit;
  const int grid = p.streamk ? sm_count() : (int)(tiles < sm_count() ? tiles : sm_count());
  if (rb == 64)
    return launch_epi<EPI_F32, 1, 64, 5, 64>(ta, tb0, tb1, p, grid,
                                             gemm_smem(1, 64, 5, G, 0, 64), s);
  return launch_epi<EPI_F32, 1, 64, 4>(ta, tb0, tb1, p, grid, gemm_smem(1, 64, 4, G), s);
}

int gemm_sm_count() { return sm_count(); }

int splitk_count(int K, int ksplit) {
  const int nkb = (K + 63) / 64;
  if (nkb <= 0 || ksplit < 1) return 1;
  const int kchunk = (nkb + ksplit - 1) / ksplit;
  return (nkb + kchunk - 1) / kchunk;
}

// k-splits of the router product: enough (m-tile, split) pairs to cover the SMs, at most
// kRouterMaxSplits, and every split non-empty (ks = ceil(nkb / ceil(nkb / ks))).
int router_gemm_splits(int T, int D) {
  const int mt = (T + BM - 1) / BM;
  const int nkb = (D + 63) / 64;
  int ks = sm_count() / (mt > 0 ? mt : 1);
  if (ks > kRouterMaxSplits) ks = kRouterMaxSplits;
  if (ks > nkb) ks = nkb;
  if (ks < 1) ks = 1;
  const int kchunk = (nkb + ks - 1) / ks;
  return (nkb + kchunk - 1) / kchunk;
}

cudaError_t launch_router_gemm_bf16(const void* x, int T, int D, const void* Wg, int E,
                                    float* partials, int ksplit, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  alignas(64) CUtensorMap ta, tb;
  if (!make_map(&ta, x, (uint64_t)T, (uint64_t)D, 128, 64)) return cudaErrorInvalidValue;
  if (!make_map(&tb, Wg, (uint64_t)E, (uint64_t)D, 128, 64)) return cudaErrorInvalidValue;
  GemmParams p{};
  p.offsets = nullptr;                        // one group: all T token rows
  p.out = reinterpret_cast<__nv_bfloat16*>(partials);
  p.err = device_error_word();
  p.rows = T;
  p.ldo = E;
  p.G = 1;
  p.N = E;
  p.K = D;
  p.n_out_tile = 256;
  p.nt = 1;
  p.fault = 0;
  const int nkb = (D + 63) / 64;
  p.ksplit = ksplit;
  p.kchunk = (nkb + ksplit - 1) / ksplit;
  p.split_stride = (int64_t)T * E;
  p.kgroup = nullptr;
  p.out_gstride = 0;
  p.out2 = nullptr;
  p.ldo2 = 0;
  p.kb_split = 0;
  p.bk_group = 0;
  const int64_t tiles = (int64_t)((T + BM - 1) / BM) * ksplit;
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  return launch_epi<EPI_F32, 1, 64, 4>(ta, tb, tb, p, grid, gemm_smem(1, 64, 4, 1), s);
}

}  // namespace moe
