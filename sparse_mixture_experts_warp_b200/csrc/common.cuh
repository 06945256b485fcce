// Shared device/host helpers of the sm_100a MoE library (no layer arithmetic here).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Device error codes written into the library's device error word.
enum : int {
  DEVERR_NONE = 0,
  DEVERR_TIMEOUT_TMA = 0x101,     // producer gave up waiting for a free stage
  DEVERR_TIMEOUT_MMA = 0x102,     // MMA issuer gave up waiting for operands / accumulator
  DEVERR_TIMEOUT_EPI = 0x103,     // epilogue gave up waiting for an accumulator
  DEVERR_BOUNDS = 0x201,          // a device-side bounds check fired
};

// Address of the library's device error word on the current device.
int* device_error_word();

inline bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Kernels this library has enqueued since it was loaded (every launch site passes its grid
// through counted()).
void note_launch();
template <typename G>
inline G counted(G grid) {
  note_launch();
  return grid;
}

// ---- programmatic dependent launch ----
// The forward path's kernels are launched with programmatic stream serialization: the next
// kernel in the stream may be scheduled while this one finishes (its launch and set-up overlap
// the tail), and every such kernel starts with pdl_trigger() (its dependents may launch) and
// calls pdl_wait() -- which returns once the preceding grid has completed and its memory is
// visible -- before it touches anything an earlier kernel wrote or reads.  Without the launch
// attribute both are no-ops.  MOE_PDL=0 in the environment turns the attribute off.
bool pdl_enabled();
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch of a kernel that calls pdl_wait() before its first dependent access.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
  note_launch();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---- stream-K schedule of the fp32 k-split products (grouped GEMM and its summing kernel) ----
// CTA c of g takes k-blocks [c * work / g, (c + 1) * work / g) of work = tiles * nkb (tile t
// owns [t * nkb, (t + 1) * nkb)).  CTAs used: at most grid, and few enough that every range
// holds ceil(nkb / (slots - 1)) k-blocks or more, so that a tile meets at most `slots` ranges.
__host__ __device__ __forceinline__ int streamk_ctas(int64_t work, int nkb, int slots, int grid) {
  if (work <= 0) return 0;
  const int64_t minr = slots > 1 ? (nkb + slots - 2) / (slots - 1) : nkb;
  int64_t g = work / (minr > 0 ? minr : 1);
  if (g > grid) g = grid;
  return g > 0 ? (int)g : 1;
}
// The CTA whose range holds k-block x.
__host__ __device__ __forceinline__ int streamk_owner(int64_t x, int64_t work, int g) {
  return (int)(((x + 1) * g - 1) / work);
}

// ---- launchers implemented in the .cu files (all enqueue on `s`, return the launch error) ----

// route.cu
cudaError_t launch_router_token_choice(const moe_desc_t& d, const void* x, const void* Wg,
                                       const float* bias, int32_t* ids, float* gates,
                                       float* logits, float* imp_partials, int* n_partials,
                                       float* lpart, cudaStream_t s);
cudaError_t launch_router_expert_choice(const moe_desc_t& d, const void* x, const void* Wg,
                                        float* probs, float* probsT, float* logits,
                                        float* imp_partials, int* n_partials, float* lpart,
                                        cudaStream_t s);
cudaError_t launch_ec_select(const moe_desc_t& d, const float* probsT, int32_t* picked,
                             cudaStream_t s);
cudaError_t launch_importance_reduce(const float* partials, int n_partials, int E, int T,
                                     float* importance, float* entropy, cudaStream_t s);
int router_partials(const moe_desc_t& d);   // rows of the importance partials buffer (upper bound)
bool router_uses_gemm(const moe_desc_t& d);
size_t router_gemm_scratch_bytes(const moe_desc_t& d);   // partial logits of the GEMM router

// Streaming multiprocessors of the current device.
int num_sms();

// permute.cu
int permute_blocks(const moe_desc_t& d);
cudaError_t launch_permute_token_choice(const moe_desc_t& d, const int32_t* ids, const void* x,
                                        void* x_perm, int32_t* counts, int32_t* offsets,
                                        int32_t* row_src, int32_t* inv, int32_t* block_hist,
                                        int32_t cap, cudaStream_t s);
// The grouped copy of the token rows alone (x_perm[row] = x[token of row]), from the
// permutation's inv (token choice) or picked lists (expert choice).
cudaError_t launch_gather_permuted_rows(const moe_desc_t& d, const int32_t* ids,
                                        const int32_t* inv, const void* x, void* x_perm,
                                        cudaStream_t s);
cudaError_t launch_permute_expert_choice(const moe_desc_t& d, const int32_t* picked,
                                         const void* x, void* x_perm, int32_t* counts,
                                         int32_t* offsets, int32_t* row_src, int32_t* inv,
                                         cudaStream_t s);

// gemm_sm100.cu (bf16 grouped GEMM on tcgen05)
enum GemmEpilogue { EPI_SWIGLU = 0, EPI_RELU = 1, EPI_NONE = 2, EPI_F32 = 3, EPI_GELU = 4,
                    EPI_RAW = 5 /* bf16 gate | up accumulators, SwiGLU operand staging */,
                    EPI_NONE_BMN = 6 /* EPI_NONE with an MN-major B operand */,
                    EPI_F32_TMA = 7 /* EPI_F32 written by TMA stores from shared memory */ };
// k-split fp32 partials [ksplit][a_rows][N] of a grouped product (groups along M); the number
// of non-empty splits is ceil(nkb / ceil(nkb / ksplit)) for nkb = ceil(K / 64).
// sk_slots > 0 (a_rows <= 64): stream-K instead of ksplit equal k-ranges per tile: every CTA
// takes an equal contiguous range of the tiles' k-blocks, and the part of a tile in CTA c's
// range is written as partial slot c - (the tile's first CTA), at most sk_slots per tile
// (launch_splitk_streamk sums them).
cudaError_t launch_grouped_gemm_f32_splitk(const void* A, int64_t a_rows, int K, const void* B,
                                           int G, int N, const int32_t* offsets, int ksplit,
                                           float* out, cudaStream_t s, int sk_slots = 0);
// The same for two products that share A (the gate and up products of the decode schedule):
// out[split][row][ldo] with ldo = 2 * ceil(N / 256) * 256, B0's product in columns
// [0, N) and B1's from column ldo / 2.
cudaError_t launch_grouped_gemm_f32_splitk2(const void* A, int64_t a_rows, int K, const void* B0,
                                            const void* B1, int G, int N,
                                            const int32_t* offsets, int ksplit, float* out,
                                            cudaStream_t s, int sk_slots = 0);
int gemm_sm_count();
int splitk_count(int K, int ksplit);   // non-empty splits of K (64-element k-blocks)
// splitk.cu: the sums of k-split partials of the small-batch schedule (rows below *n_rows)
// ld: row pitch of the partials (F when gate and up are separate arrays; the two-product
// layout's ldo otherwise).
cudaError_t launch_splitk_act(int act, const float* pg, const float* pu, int S,
                              int64_t rows, int F, const int32_t* n_rows, void* h,
                              cudaStream_t s, int64_t ld = 0);
cudaError_t launch_splitk_sum(const float* p, int S, int64_t rows, int N,
                              const int32_t* n_rows, void* y, cudaStream_t s);
// The sums of a stream-K product (launch_grouped_gemm_f32_splitk[2] with sk_slots, over the
// grid of gemm_sm_count() CTAs, groups of at most 64 rows): out[r, c] = act(sum over the
// segments of c's tile, in slot order) for the rows r < offsets[G].  Partials [slots][rows][ld];
// two = 1: gate columns at [0, N), up columns at ld / 2 (the two-product layout, n-tiles of the
// up product from ceil(N / 256)), else one product of ceil(N / 256) n-tiles.  act: MOE_ACT_* or
// -1 (no activation: the down projection).
cudaError_t launch_splitk_streamk(int act, const float* part, int slots, int64_t rows, int ld,
                                  int N, int K, int two, const int32_t* offsets, int G,
                                  void* out, cudaStream_t s);
// y[r, n] = sum over *ks splits of P[s][r][n] (split stride *n_rows * N) for r < *n_rows; does
// nothing when *ks == 1 (the product wrote y itself).  rows bounds *n_rows (grid sizing).
cudaError_t launch_splitk_sum_adaptive(const float* p, const int* ks, int64_t rows, int N,
                                       const int32_t* n_rows, void* y, cudaStream_t s);
// With gather_src, A is the token tensor [src_rows, K] and row r of the grouped operand is its
// row gather_src[r] / gather_div (4-row TMA gathers; the grouped copy is never written).
// adapt_ks_max > 1 (EPI_NONE, groups along M, no gather or out2): an adaptive k-split.  When
// the group table on the device gives fewer tiles than half the launch's CTAs, K is split
// (at most adapt_ks_max ways, as many as fill the CTAs and fit adapt_cap floats) into fp32
// partials [split][offsets[G]][N] at adapt_part instead of writing out; the split count goes
// to *adapt_ks (1: out was written), for launch_splitk_sum_adaptive.
cudaError_t launch_grouped_gemm_bf16(int epi, const void* A, int64_t a_rows, int K,
                                     const void* B0, const void* B1, int n_groups, int N,
                                     const int32_t* offsets, void* out, cudaStream_t s,
                                     void* out2 = nullptr, const int32_t* gather_src = nullptr,
                                     int gather_div = 1, int64_t src_rows = 0,
                                     float* adapt_part = nullptr, int64_t adapt_cap = 0,
                                     int adapt_ks_max = 0, int* adapt_ks = nullptr);
bool gemm_gather_ok();   // the selected tile shape can gather A rows
// gemm_swap.cu: the same grouped product with the weights as the MMA's M side and the tokens as
// its N side (tiles of 256 weight rows by up to 256 tokens, N rounded up to 16), for many groups
// of a few hundred rows or fewer; EPI_SWIGLU / EPI_RELU / EPI_GELU / EPI_NONE, bf16 out
// [a_rows, N]; gather_src as above; fault: the bounded-wait test hook.
bool swap_epilogue_ok(int epi);
cudaError_t launch_grouped_gemm_swap(int epi, const void* A, int64_t a_rows, int K,
                                     const void* B0, const void* B1, int n_groups, int N,
                                     const int32_t* offsets, void* out, cudaStream_t s,
                                     const int32_t* gather_src, int gather_div, int64_t src_rows,
                                     int fault);

// Router product on the same engine: one group of T rows, N = E, fp32 partial logits of
// ksplit k-ranges in partials[ksplit][T][E] (E % 32 == 0, E <= 256).
int router_gemm_splits(int T, int D);
cudaError_t launch_router_gemm_bf16(const void* x, int T, int D, const void* Wg, int E,
                                    float* partials, int ksplit, cudaStream_t s);

// out = A B per group along M with B stored MN-major ([K, N], N contiguous; the layout of
// nn.Linear weights used as the right operand of a backward product): group g reads its K rows
// at g * bk_group of B0 for k-blocks below kb_split and of B1 above it (B1 may be null).
cudaError_t launch_grouped_gemm_bf16_bmn(const void* A, int64_t a_rows, int K, const void* B0,
                                         const void* B1, int kb_split, int bk_group,
                                         int n_groups, int N, const int32_t* offsets, void* out,
                                         cudaStream_t s);
// out[g] = A[:, K_g] B[:, K_g]^T (fp32 [M, N] per group) for groups along K: group g owns the
// k columns [kgroup[g], kgroup[g+1]) of A [M, k_total] and B [N, k_total] (bf16, K-major,
// kgroup a device array of multiples of 64).
cudaError_t launch_grouped_gemm_kgroups_f32(const void* A, int M, const void* B, int N, int G,
                                            const int32_t* kgroup, int64_t k_total, float* out,
                                            cudaStream_t s);
// backward.cu (layer backward with the selection fixed: memory-bound pieces)
int backward_dwg_chunks(int T);
cudaError_t launch_pad_offsets(const int32_t* offsets, int E, int32_t* pad_off, cudaStream_t s);
cudaError_t launch_gather_dy(const void* dout, const void* y, const int32_t* row_src,
                             const float* gates, const int32_t* offsets, int E, int K, int D,
                             int64_t rows_max, void* dY, float* dgates, cudaStream_t s);
cudaError_t launch_act_backward(int act, const void* dH, const void* gu, int64_t ldg,
                                const int32_t* offsets, int E, int F, int64_t rows_max,
                                void* dAB, cudaStream_t s, void* h_out = nullptr);
cudaError_t launch_transpose(const void* src, int64_t src_bstride, int R, int C, int64_t lds,
                             void* dst, int64_t dst_bstride, int64_t ldd, int dcol0, int batch,
                             cudaStream_t s);
cudaError_t launch_transpose_pad(const void* src, int64_t lds, int C, const int32_t* offsets,
                                 const int32_t* pad_off, int E, int64_t pad_cols, void* dst,
                                 int64_t ldd, cudaStream_t s);
cudaError_t launch_router_backward(const moe_desc_t& d, const float* logits, const int32_t* ids,
                                   const float* gates, const float* dgates, const int32_t* inv,
                                   const float* f, float aux_grad, float* ds, cudaStream_t s);
cudaError_t launch_dx(const void* dX, const int32_t* inv, const float* ds, const void* Wg, int T,
                      int D, int E, int K, void* dx, cudaStream_t s, const void* dXs = nullptr,
                      int n_add = 0);
cudaError_t launch_dwg(const float* ds, const void* x, int T, int D, int E, float* part,
                       float* dWg, cudaStream_t s);

// Test hook of the grouped GEMM's bounded waits (see moe_debug_inject).
void set_gemm_fault(int kind);

// backward_f32.cu (fp32 layer backward on CUDA cores)
size_t backward_f32_workspace(const moe_desc_t& d, int64_t rows);
cudaError_t launch_backward_f32(const moe_desc_t& d, const moe_layer_views_t& v,
                                const float* x, const float* Wg, const float* W_gate,
                                const float* W_up, const float* W_down,
                                const moe_bwd_shared_t* sh, const float* dout, float aux_grad,
                                float* dx, float* dWg, float* dW_gate, float* dW_up,
                                float* dW_down, void* ws, cudaStream_t s);

// ffn_simt.cu (fp32 experts)
cudaError_t launch_ffn_up_f32(int act, const float* a, int64_t a_rows, int D, int F,
                              const int32_t* offsets, int n_groups, const float* Wgate,
                              const float* Wup, float* h, cudaStream_t s);
cudaError_t launch_ffn_down_f32(const float* h, int64_t a_rows, int D, int F,
                                const int32_t* offsets, int n_groups, const float* Wdown,
                                float* y, cudaStream_t s);

// combine.cu
// Inputs of the balance statistics (moe_balance_stats): counts / offsets from the permutation,
// importance / entropy from the router, outputs f [E] and *st.
struct StatsArgs {
  const int32_t* counts;
  const int32_t* offsets;
  const float* importance;
  const float* entropy;
  int E, n_routes;
  float alpha;
  float* f;
  moe_stats_t* st;
};
StatsArgs stats_args(const moe_desc_t& d, const int32_t* counts, const int32_t* offsets,
                     const float* importance, const float* entropy, float* f,
                     moe_stats_t* stats);
// The down projection's device-side k-split left unsummed: fp32 partials [*ks][live][D] at
// part (live = min(*n_rows, rows)); when *ks <= 1 the product wrote y itself.
struct SplitRows {
  const float* part;
  const int* ks;
  const int32_t* n_rows;
  int64_t rows;
  void* y;          // [rows, D] bf16, filled by launch_combine
};
// with_stats: block 0 of the combine also computes the balance statistics (the layer step's
// last two stages in one launch; every input of the statistics was written by earlier kernels).
// split: the combine first forms each kept row of y from the partials (the sum and bf16
// rounding of launch_splitk_sum_adaptive, in split order), writes it to y and uses it.
cudaError_t launch_combine(const moe_desc_t& d, const void* y, const int32_t* inv,
                           const float* gates, const void* y_shared, void* out,
                           cudaStream_t s, const StatsArgs* with_stats = nullptr,
                           const SplitRows* split = nullptr);
cudaError_t launch_balance_stats(const moe_desc_t& d, const int32_t* counts,
                                 const int32_t* offsets, const float* importance,
                                 const float* entropy, float* f, moe_stats_t* stats,
                                 cudaStream_t s);

}  // namespace moe
