/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts FFN layer, forward pass.
 *
 * The layer, as the pages define it (Gate -> Dispatch -> Expert compute -> Combine):
 *   "Top-k 路由（Top-k Routing）" (compassingai), "Top-k 路由的完整生命週期" and
 *   "門控函式的數學形式" Steps 1-3;
 *   "别只比较 Top-k" (ailearn moe-comparison), "评分、Top-k、合并权重和实际执行是四个连续但
 *   不同的步骤" (Score -> Select -> Merge -> Execute);
 *   "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡" (f3dlife),
 *   sections 3-8.
 *
 * Conventions shared by every entry point
 *   - All pointers named as device buffers are device pointers of the current CUDA device;
 *     the caller allocates and owns them.  The library allocates, frees and synchronises
 *     nothing (the one exception, moe_get_device_error, says so).  Work is enqueued on the
 *     given stream and is asynchronous.
 *   - Tensors are dense row-major.  Weights use the nn.Linear layout [out, in]:
 *     W_g [E, D]; W_gate, W_up [E, F, D]; W_down [E, D, F]; shared [S, Fs, D] / [S, D, Fs].
 *   - dtype MOE_BF16: activations and weights are bf16 (fp32 accumulation, bf16 out);
 *     dtype MOE_F32: everything is fp32.  Router logits, probabilities and gates are fp32.
 *   - Every device buffer handed in must be 16-byte aligned.
 *   - Arguments are checked on the host before anything is launched: a bad argument returns
 *     MOE_ERR_INVALID_ARG, a valid but unimplemented combination MOE_ERR_UNSUPPORTED, a too
 *     small workspace MOE_ERR_WORKSPACE, a failed launch MOE_ERR_CUDA.  Device-side waits are
 *     bounded: a wait that gives up records MOE_ERR_TIMEOUT in a device error word, read
 *     with moe_get_device_error.
 *   - Limits: 1 <= E <= 256; token choice 1 <= k <= min(E, 32); expert choice 1 <= c <= T;
 *     T * max(k, E) < 2^31.  bf16: D, F and F_shared multiples of 64.  fp32: D multiple of 4.
 *   - An empty batch (T = 0, token choice) is valid: moe_layer_forward, moe_route, moe_combine
 *     and moe_balance_stats check their arguments and return MOE_OK without launching anything
 *     or writing any output (views and statistics keep their previous contents); moe_permute
 *     writes zero counts and offsets; the expert products have no rows to compute.
 *
 * Environment switches, read once per process.  The defaults are the paths measured fastest on
 * B200; each switch keeps another tested path reachable for comparison measurements:
 *   MOE_ROUTER=tc|fast|gemm|simt   router kernel (default: mma.sync for E <= 8 with
 *                                  D = 256 * (4..16), else the tcgen05 router, else SIMT)
 *   MOE_GEMM_TILE=128|256|256k32|pair  one grouped-GEMM tile shape for every call (default:
 *                                  chosen per call by group size and whole waves of SMs)
 *   MOE_GEMM_SWAP=1                grouped GEMMs with the weights as the MMA's M side
 *   MOE_GATHER_FUSION=1            the layer's up projection gathers the token rows itself
 *   MOE_DECODE_SPLITK=0            no k-split schedule for few executed rows
 *   MOE_STREAMK=0                  equal k-ranges instead of stream-K in that schedule
 *   MOE_ADAPTIVE_SPLIT=0           no device-side k-split of a capacity-limited down product
 *   MOE_PERMUTE_CLUSTER=0          no one-cluster permutation index kernel
 *   MOE_PDL=0                      no programmatic dependent launch between kernels
 *   MOE_WGRAD_TILE=128             128-row weight-gradient tiles (default 256)
 *   MOE_BWD_WEIGHT_TRANSPOSE=1     the backward's dgrad products read transposed weight copies
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t;   /* same type as cudaStream_t; NULL = legacy default stream */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_WORKSPACE = 3,
    MOE_ERR_CUDA = 4,
    MOE_ERR_TIMEOUT = 5,
    MOE_ERR_DEVICE = 6
} moe_status_t;

enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 };   /* affinity */
enum { MOE_TOKEN_CHOICE = 0, MOE_EXPERT_CHOICE = 1 };    /* who selects */
enum { MOE_GATE_RENORM = 0, MOE_GATE_RAW = 1 };          /* merge weights */
enum { MOE_DROPLESS = 0, MOE_CAPACITY_DROP = 1 };        /* overflow policy */
enum { MOE_ACT_SWIGLU = 0, MOE_ACT_RELU = 1, MOE_ACT_GELU = 2 };   /* expert FFN */
enum { MOE_F32 = 0, MOE_BF16 = 1 };                      /* operand dtype */

/* Problem statement of one layer call.
 *   T tokens, D hidden, E routed experts, F expert width;
 *   k  : token choice, experts per token ("Top-k 路由" gate Step 2);
 *   c  : expert choice, tokens per expert ("Top-k 路由" Token-Choice vs Expert-Choice table);
 *   n_shared, F_shared : always-on shared experts (moe-comparison family table, DeepSeek rows);
 *   score    : softmax over experts, or sigmoid affinity (moe-comparison "Score");
 *   gate     : RENORM g_j = p_j / sum_sel p (Tiny MoE section 4), RAW g = p (Switch, top-1);
 *              under sigmoid, RENORM uses the raw affinities, never the selection bias;
 *   overflow : DROPLESS, or CAPACITY_DROP with C = ceil(capacity_factor * T * k / E) slots per
 *              expert, evaluated in double ("Top-k 路由" capacity factor formula); the first C
 *              assignments of an expert in (token, slot) order keep a slot, later ones add 0;
 *   aux_alpha: alpha of the balance loss alpha * E * sum_e f_e P_e;
 *   n_group, topk_group : group-limited token choice (talentme M4-080 routing variant (c):
 *              groups first, then experts inside them; moe-comparison "Group/node limited" row,
 *              DeepSeek-V3: 256 experts on 8 nodes, a token's top-8 on at most 4).  The experts
 *              are split into n_group contiguous groups of E / n_group; a group scores its
 *              largest selection key and each token keeps its topk_group best groups (ties to the
 *              lower group index) before the top-k.  n_group <= 1 or topk_group == n_group:
 *              no limit.  Limits: n_group <= 32 and divides E, E / n_group a power of two
 *              <= 32 or a multiple of 32, 1 <= topk_group <= n_group, topk_group * E / n_group
 *              >= k; token choice only. */
typedef struct moe_desc {
    int32_t T, D, E, F;
    int32_t k;
    int32_t c;
    int32_t n_shared, F_shared;
    int32_t score, select, gate, overflow, act, dtype;
    float capacity_factor;
    float aux_alpha;
    int32_t n_group, topk_group;
} moe_desc_t;

/* Scalars of the balance statistics (written to device memory by moe_balance_stats). */
typedef struct moe_stats {
    float aux;             /* alpha * E * sum_e f_e * P_e */
    float max_over_mean;   /* max_e count_e / mean_e count_e (nominal counts) */
    int32_t n_routes;      /* T*k (token choice) or E*c (expert choice) */
    int32_t n_kept;        /* rows the experts execute */
    int32_t n_dropped;     /* n_routes - n_kept */
    int32_t reserved;
    float entropy;         /* mean over tokens of -sum_e p log p (NaN when not given) */
    float count_p95;       /* 95th / 99th percentile of the per-expert counts, linear */
    float count_p99;       /*   interpolation between order statistics */
    float reserved2;
} moe_stats_t;

/* Device views into a moe_layer_forward workspace (see moe_layer_views). */
typedef struct moe_layer_views {
    int32_t* expert_ids;   /* TC [T,k] expert per slot, descending key; EC [E,c] token ids, ascending */
    float* gates;          /* TC [T,k] merge weights;  EC [T,E] softmax probabilities */
    float* logits;         /* [T,E] fp32 router logits */
    float* importance;     /* [E]   P_e */
    float* entropy;        /* [1]   mean router entropy over tokens */
    int32_t* counts;       /* [E]   nominal assignments per expert */
    int32_t* offsets;      /* [E+1] first row of each expert in the grouped buffers */
    int32_t* row_src;      /* [A]   assignment id of each row: t*k+j (TC) or t*E+e (EC) */
    int32_t* inv;          /* TC [T*k], EC [T*E]: row of each assignment, -1 if dropped / not picked */
    void* x_perm;          /* [A, D]  token rows grouped by expert (not written by a
                                         moe_layer_forward that gathers, see moe_gather_fusion) */
    void* h;               /* [A, F]  expert hidden activations */
    void* y;               /* [A, D]  expert outputs, grouped */
    void* y_shared;        /* [S, T, D] shared expert outputs (NULL when S = 0) */
    void* h_shared;        /* [T, Fs] shared expert hidden (NULL when S = 0) */
    int32_t* shared_offsets; /* [2] = {0, T} */
    float* f;              /* [E] load f_e */
    moe_stats_t* stats;    /* one moe_stats_t */
    void* scratch;         /* scratch for the step entry points */
    size_t scratch_bytes;
    int64_t rows;          /* A: rows allocated for the grouped buffers */
} moe_layer_views_t;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status_t status);

/* Library version as a static string. */
const char* moe_version(void);

/* A, the upper bound on rows the experts execute: T*k (dropless), min(T*k, E*C) (capacity
 * drop), E*c (expert choice).  Grouped buffers (x_perm, h, y, row_src) need A rows. */
moe_status_t moe_rows_max(const moe_desc_t* desc, int64_t* rows);

/* C, the slots per expert under MOE_CAPACITY_DROP (0 otherwise). */
moe_status_t moe_capacity(const moe_desc_t* desc, int32_t* capacity);

/* Bytes of scratch that moe_route, moe_permute and moe_balance_stats need, and the routed
 * experts' k-split partials of moe_expert_up_ws / moe_expert_down_ws (a few executed rows). */
moe_status_t moe_scratch_size(const moe_desc_t* desc, size_t* bytes);

/* Bytes of workspace moe_layer_forward needs (every intermediate plus scratch). */
moe_status_t moe_workspace_size(const moe_desc_t* desc, size_t* bytes);

/* Carves `ws` (moe_workspace_size bytes, 256-byte aligned) into the views above.  Host only. */
moe_status_t moe_layer_views(const moe_desc_t* desc, void* ws, size_t ws_bytes,
                             moe_layer_views_t* views);

/* Score + Select + merge weights.
 * "Top-k 路由" gate Steps 1-2; Tiny MoE section 4; moe-comparison "Score"/"Select"/"Merge".
 *   Kernels: bf16 with E <= 8 and D a multiple of 256 in [1024, 4096]: an mma.sync router;
 *   other bf16 with D % 64 == 0 and E <= 256: the tcgen05 router product in CTA clusters fused
 *   with the selection; otherwise a CUDA-core router.  Every path takes the same decisions from
 *   its fp32 logits (MOE_ROUTER=tc|fast|gemm|simt in the environment selects one).
 *   x [T,D], Wg [E,D] (dtype); sel_bias [E] fp32 or NULL (added to sigmoid affinities for
 *   selection only).
 *   Token choice: expert_ids [T,k], gates [T,k]; slot j holds the j-th largest key (the logit
 *   under softmax, sigmoid + bias under sigmoid), ties to the lower expert id.
 *   Expert choice: expert_ids [E,c] = each expert's c most probable tokens (ties to the lower
 *   token id) in ascending order; gates [T,E] = softmax probabilities (merge weights).
 *   logits [T,E] (fp32) and importance [E] (P_e = mean_t of the softmax probabilities, or of
 *   the sigmoid affinities normalised over experts) and entropy [1] (mean over tokens of
 *   -sum_e p log p of those probabilities; moe-comparison monitoring list) are optional (NULL).
 *   scratch: moe_scratch_size bytes. */
moe_status_t moe_route(const moe_desc_t* desc, const void* x, const void* Wg,
                       const float* sel_bias, int32_t* expert_ids, float* gates,
                       float* logits, float* importance, float* entropy,
                       void* scratch, size_t scratch_bytes, moe_stream_t stream);

/* Dispatch: counting-sort permutation of assignments into expert-contiguous rows.
 * Tiny MoE section 5 (torch.where gives, per expert, its (token, slot) pairs in row-major
 * order); "Top-k 路由" capacity factor; moe-comparison capacity/overflow table.
 *   counts [E] nominal assignments; offsets [E+1] exclusive scan of kept rows;
 *   row_src [A] assignment id per row; inv [T*k] (TC) / [T*E] (EC) row per assignment or -1;
 *   x_perm [A, D] (dtype) rows gathered from x; x_perm = NULL computes the indices only (the
 *   rows are then read by moe_expert_up_gather).  Rows of one expert are ordered by (token,
 *   slot).  All outputs are deterministic.  scratch: moe_scratch_size bytes. */
moe_status_t moe_permute(const moe_desc_t* desc, const int32_t* expert_ids, const void* x,
                         void* x_perm, int32_t* counts, int32_t* offsets, int32_t* row_src,
                         int32_t* inv, void* scratch, size_t scratch_bytes, moe_stream_t stream);

/* moe_permute without scratch, for callers that cannot allocate device memory (a plugin handed
 * only its input and output buffers by an engine whose allocator owns the device memory, or
 * host code that must not call cudaMalloc at that point).  The pages have no counterpart: this
 * is a property of the library, not of the method.
 *   Same arguments, outputs and results as moe_permute, minus scratch.  Its scratch is a fixed
 *   file-scope device array of MOE_PERMUTE_NOALLOC_MAX_INTS int32 (256 KiB), held until exit on
 *   every GPU where the library's module is loaded.  Token choice needs ceil(T*k/1024)*E of
 *   them; larger problems return MOE_ERR_UNSUPPORTED before any pointer is examined and before
 *   anything is launched.  Allocates nothing (no cudaMalloc, cudaFree or allocating library
 *   call).
 *   The first call in each CUDA context looks up the array's device address
 *   (cudaGetSymbolAddress) with that context current and caches it under the context's unique
 *   id, so a device reset is followed by a fresh look-up: make that first call before any
 *   stream capture.  Under lazy module loading that first call is also when the array is
 *   committed to the GPU: make it before the caller reserves the GPU's memory (a GPU with no
 *   room left gives MOE_ERR_CUDA).
 *   All calls share the array and each overwrites the last one's contents; calls whose work
 *   overlaps on the GPU (other streams, other threads) race on it -- serialise them. */
#define MOE_PERMUTE_NOALLOC_MAX_INTS 65536
moe_status_t moe_permute_noalloc(const moe_desc_t* desc, const int32_t* expert_ids,
                                 const void* x, void* x_perm, int32_t* counts, int32_t* offsets,
                                 int32_t* row_src, int32_t* inv, moe_stream_t stream);

/* Expert compute on grouped rows (Tiny MoE section 3, SwiGLU: down(SiLU(x W_gate^T) * x W_up^T);
 * the classic two-matrix FFN D -> F -> D: down(ReLU(x W_up^T)) or down(GELU(x W_up^T)) with the
 * exact GELU(z) = z * (1 + erf(z / sqrt 2)) / 2).  Group g owns rows [offsets[g], offsets[g+1]) of `a`
 * (offsets is a device array of n_groups+1 ints, read on the device).
 *   a [a_rows, D], h [a_rows, F], y [a_rows, D] (dtype; h, y rows outside the groups are not
 *   written).  W_gate (NULL for ReLU / GELU), W_up [n_groups, F, D], W_down [n_groups, D, F].
 *   D comes from desc; act and dtype too.  For routed experts: n_groups = E, F = desc->F,
 *   a = x_perm, a_rows = moe_rows_max.  For a shared expert: n_groups = 1, F = F_shared,
 *   a = x, a_rows = T, offsets = {0, T}.
 * moe_expert_up writes h, moe_expert_down reads h and writes y; moe_expert_ffn does both. */
moe_status_t moe_expert_up(const moe_desc_t* desc, int32_t n_groups, int32_t F,
                           const void* a, int64_t a_rows, const int32_t* offsets,
                           const void* W_gate, const void* W_up, void* h, moe_stream_t stream);
moe_status_t moe_expert_down(const moe_desc_t* desc, int32_t n_groups, int32_t F,
                             const void* h, int64_t a_rows, const int32_t* offsets,
                             const void* W_down, void* y, moe_stream_t stream);
moe_status_t moe_expert_ffn(const moe_desc_t* desc, int32_t n_groups, int32_t F,
                            const void* a, int64_t a_rows, const int32_t* offsets,
                            const void* W_gate, const void* W_up, const void* W_down,
                            void* h, void* y, moe_stream_t stream);

/* moe_expert_up that reads its rows straight from the tokens: Tiny MoE section 12.1's fusion of
 * the token permutation into the grouped GEMM.  Row r of the grouped operand is token
 * row_src[r] / K of x (K = k for token choice, E for expert choice; row_src from moe_permute,
 * which then needs no x_perm); the up projection's A tiles are loaded with 4-row TMA gathers,
 * so the grouped copy of x is never written or read.  Same results as moe_permute with x_perm
 * followed by moe_expert_up on it.  x [T, D] bf16; a_rows = moe_rows_max; bf16 only, and the
 * default or 128-row GEMM tile (MOE_ERR_UNSUPPORTED otherwise). */
moe_status_t moe_expert_up_gather(const moe_desc_t* desc, int32_t n_groups, int32_t F,
                                  const void* x, const int32_t* row_src, int64_t a_rows,
                                  const int32_t* offsets, const void* W_gate, const void* W_up,
                                  void* h, moe_stream_t stream);

/* Whether moe_layer_forward uses that fusion for this desc (*on = 1): MOE_GATHER_FUSION=1 in the
 * environment (it is off by default: measured slower than the tiled loads of x_perm, whose
 * write it saves), bf16, more than 16 grouped rows (fewer take the small-batch schedule on
 * x_perm).  Host only. */
moe_status_t moe_gather_fusion(const moe_desc_t* desc, int32_t* on);

/* moe_expert_up / moe_expert_down with a scratch area for the small-batch (decode) schedule
 * ("别只比较 Top-k" expert-work account: a small decode batch leaves each expert's products
 * with very few rows, so they stream the weights).  Same arguments and results (up to fp32
 * summation order), plus scratch (device, 16-byte aligned, scratch_bytes long; may be NULL with
 * scratch_bytes = 0).  bf16 only: when the fused grouped product would keep fewer than 80% of
 * the SMs busy (a_rows <= 256 for the down product, <= 16 for the up product; active groups
 * bounded by min(n_groups, a_rows)), the product is split along K into 2..8 parts whose fp32
 * partials go to scratch and are summed in a fixed order (deterministic) before the activation
 * and the bf16 rounding; SwiGLU's gate and up products run as one launch.  With at most 64 rows,
 * a split whose tiles x k-ranges exceed the SM count runs stream-K instead (every SM an equal
 * contiguous share of all tiles' k-blocks, at most 8 partial slots per tile, summed in slot
 * order); MOE_STREAMK=0 keeps equal k-ranges per tile.
 * moe_expert_down_ws also splits on the device: for a desc under a capacity limit whose fewest
 * possible executed rows would give fewer output tiles than a B200 has SMs, the grouped GEMM
 * reads the group table and, when its tiles fill fewer than half of its CTAs, splits K (at most
 * 8 ways, fp32 partials of the executed rows within at most 24 MB of scratch) and a second
 * kernel sums them in split order; otherwise it writes y directly.  When scratch is too small
 * for the partials, or MOE_DECODE_SPLITK=0 (both schedules) / MOE_ADAPTIVE_SPLIT=0 (the
 * device-side one) is set in the environment, the fused product runs.  moe_scratch_size covers
 * the routed experts' partials; moe_layer_forward uses these schedules for the routed experts
 * (the shared experts keep the fused products). */
moe_status_t moe_expert_up_ws(const moe_desc_t* desc, int32_t n_groups, int32_t F,
                              const void* a, int64_t a_rows, const int32_t* offsets,
                              const void* W_gate, const void* W_up, void* h, void* scratch,
                              size_t scratch_bytes, moe_stream_t stream);
moe_status_t moe_expert_down_ws(const moe_desc_t* desc, int32_t n_groups, int32_t F,
                                const void* h, int64_t a_rows, const int32_t* offsets,
                                const void* W_down, void* y, void* scratch, size_t scratch_bytes,
                                moe_stream_t stream);

/* Merge: out[t] = sum_j gates[t,j] * y[inv[t,j]] + sum_s y_shared[s,t], fp32 accumulation in
 * slot order, no atomics; inv = -1 contributes 0.  "Top-k 路由" Combine; Tiny MoE section 6.
 *   y [A, D] (dtype); inv, gates as produced by moe_permute / moe_route (K = k, or E under
 *   expert choice); y_shared [n_shared, T, D] or NULL; out [T, D] (dtype). */
moe_status_t moe_combine(const moe_desc_t* desc, const void* y, const int32_t* inv,
                         const float* gates, const void* y_shared, void* out,
                         moe_stream_t stream);

/* Balance statistics ("Top-k 路由" load-balancing loss; Tiny MoE section 8; moe-comparison
 * [9,4,2,1] imbalance example and its monitoring list): f_e = counts_e / n_routes,
 * aux = alpha * E * sum f_e P_e, max/mean of counts, kept and dropped routes, the 95th/99th
 * percentiles of the per-expert counts, and the router entropy when `entropy` (a device scalar
 * written by moe_route) is given.  counts [E] and offsets [E+1] from moe_permute, importance
 * [E] from moe_route; f [E] and one moe_stats_t are written. */
moe_status_t moe_balance_stats(const moe_desc_t* desc, const int32_t* counts,
                               const int32_t* offsets, const float* importance,
                               const float* entropy, float* f, moe_stats_t* stats,
                               moe_stream_t stream);

/* The whole layer: route -> permute -> expert_ffn (+ shared experts) -> combine -> stats,
 * enqueued on one stream with no host synchronisation.  Intermediates live in `ws`
 * (moe_workspace_size bytes); moe_layer_views gives their addresses.  The last two steps run
 * as one launch (the combine's first block computes the statistics); f and the moe_stats_t in
 * `ws` equal, bit for bit, what moe_balance_stats computes from the same views.  When the down
 * projection splits K on the device (moe_expert_down_ws) and the layer has no shared experts
 * and k <= 2, the combine sums the split partials into y itself; y and out are the same, bit
 * for bit, as with the separate summing pass.
 *   x [T,D], Wg [E,D], sel_bias [E] or NULL, routed weights as above, shared weights
 *   [S,Fs,D], [S,Fs,D], [S,D,Fs] (NULL when S = 0), out [T,D]. */
moe_status_t moe_layer_forward(const moe_desc_t* desc, const void* x, const void* Wg,
                               const float* sel_bias, const void* W_gate, const void* W_up,
                               const void* W_down, const void* Ws_gate, const void* Ws_up,
                               const void* Ws_down, void* out, void* ws, size_t ws_bytes,
                               moe_stream_t stream);

/* Shared experts' weights and gradient outputs for moe_layer_backward_ex (see below). */
typedef struct moe_bwd_shared {
    const void* Ws_gate;   /* [S, Fs, D] bf16, as given to moe_layer_forward */
    const void* Ws_up;     /* [S, Fs, D] */
    const void* Ws_down;   /* [S, D, Fs] */
    float* dWs_gate;       /* [S, Fs, D] fp32, overwritten */
    float* dWs_up;         /* [S, Fs, D] fp32, overwritten */
    float* dWs_down;       /* [S, D, Fs] fp32, overwritten */
} moe_bwd_shared_t;

/* Backward of moe_layer_forward with the selection held fixed ("Top-k 路由" section
 * "門控網路的梯度流": the selected experts' gate scores carry the gradient, unselected experts
 * none; Tiny MoE section 9: task loss + weight x aux loss, fixed expert indices).
 * Loss L = <dout, out> + aux_grad * aux; the routing, permutation, logits, gates, h, y
 * and f of the forward call are read from its workspace `fwd_ws` (same desc and inputs).
 *   Outputs: dx [T, D] (the layer dtype); dWg [E, D], dW_gate and dW_up [E, F, D] (dW_gate NULL unless
 *   SwiGLU), dW_down [E, D, F], all fp32, overwritten.  The selection-only bias gets no
 *   gradient.  Merge weights: softmax over the selected logits (RENORM) or the softmax value
 *   (RAW); sigmoid affinities likewise; the balance loss reaches the logits through P.
 *   bwd_ws: moe_backward_workspace_size bytes, 256-byte aligned.
 *   flags: MOE_BWD_PREACT_SAVED when moe_layer_forward_train wrote the expert
 *   pre-activations into this bwd_ws for this forward (the backward then skips recomputing
 *   them with a third up projection); 0 otherwise.
 * Token choice or expert choice (the merge weight of a picked (token, expert) pair is its
 * softmax probability, so its logit gradient is the softmax Jacobian applied to the pairs' dg;
 * the picked sets are held fixed like the top-k).  Layers with shared experts use
 * moe_layer_backward_ex.  bf16 layers run the products on the tensor-core grouped GEMM (bf16
 * operands, fp32 accumulation); fp32 layers (Tiny MoE section 9 trains in fp32) run them in
 * fp32 on CUDA cores, always recompute the pre-activations (flags ignored) and write dx in
 * fp32. */
enum { MOE_BWD_PREACT_SAVED = 1 };
moe_status_t moe_backward_workspace_size(const moe_desc_t* desc, size_t* bytes);
moe_status_t moe_layer_backward(const moe_desc_t* desc, const void* x, const void* Wg,
                                const void* W_gate, const void* W_up, const void* W_down,
                                const void* dout, float aux_grad, void* fwd_ws,
                                size_t fwd_ws_bytes, void* dx, float* dWg, float* dW_gate,
                                float* dW_up, float* dW_down, void* bwd_ws,
                                size_t bwd_ws_bytes, int32_t flags, moe_stream_t stream);

/* moe_layer_backward for any layer, shared experts included ("别只比较 Top-k" family table,
 * DeepSeek rows: always-on shared experts on the direct path with weight 1, so each sees dout on
 * every token).  `shared` (NULL when n_shared = 0) holds their weights and receives their
 * gradients: dWs_down[i] = dout^T h_i, dWs_gate[i] = da_i^T x, dWs_up[i] = db_i^T x, and their
 * input gradients are added into dx.  Their pre-activations are recomputed.  The other
 * arguments, results and limits are those of moe_layer_backward; bwd_ws is
 * moe_backward_workspace_size bytes of the same desc. */
moe_status_t moe_layer_backward_ex(const moe_desc_t* desc, const void* x, const void* Wg,
                                   const void* W_gate, const void* W_up, const void* W_down,
                                   const moe_bwd_shared_t* shared, const void* dout,
                                   float aux_grad, void* fwd_ws, size_t fwd_ws_bytes, void* dx,
                                   float* dWg, float* dW_gate, float* dW_up, float* dW_down,
                                   void* bwd_ws, size_t bwd_ws_bytes, int32_t flags,
                                   moe_stream_t stream);

/* moe_layer_forward (same limits as moe_layer_backward) that also stores the routed expert
 * pre-activations (SwiGLU gate and up, or the ReLU/GELU input) into bwd_ws, for a following
 * moe_layer_backward with MOE_BWD_PREACT_SAVED.  Results and the workspace `ws` are those of
 * moe_layer_forward.  Layers with shared experts and fp32 layers: MOE_ERR_UNSUPPORTED (run
 * moe_layer_forward, then the backward with flags 0). */
moe_status_t moe_layer_forward_train(const moe_desc_t* desc, const void* x, const void* Wg,
                                     const float* sel_bias, const void* W_gate,
                                     const void* W_up, const void* W_down, void* out, void* ws,
                                     size_t ws_bytes, void* bwd_ws, size_t bwd_ws_bytes,
                                     moe_stream_t stream);

/* Expert parallelism ("Top-k 路由" section "通訊拓撲：All-to-All": rows go to the device that
 * holds their expert and their outputs come back, two All-to-All exchanges per layer;
 * "别只比较 Top-k", "两次 All-to-All 是常见 dispatcher 的前向合同").  G ranks, rank r holds the
 * Eg = E / G experts [r Eg, (r+1) Eg).  A rank's permuted rows are already grouped by expert,
 * so the rows for rank r are the contiguous range of its experts' rows.
 *
 * moe_ep_plan (host only, no GPU needed) turns the row counts into the exchange plan.
 *   rows_send [G*Eg]: this rank's rows per expert (kept rows, offsets[e+1] - offsets[e]),
 *     entry r*Eg + e for expert r*Eg + e.
 *   rows_recv [G*Eg]: rows_recv[s*Eg + e] = rows source rank s sends for local expert e (its
 *     rows_send entry r*Eg + e, received through a count exchange).
 *   Outputs (caller arrays): send_rows / send_offsets [G] and recv_rows / recv_offsets [G]
 *   (rows per peer and their start, in rows, in the send buffer = the permuted rows and in the
 *   source-major receive buffer); local_offsets [Eg+1], the expert-major layout the grouped
 *   GEMM runs on (local expert e: its rows from source 0, then 1, ...); block (s, e) at index
 *   s*Eg + e: block_recv (start in the receive buffer), block_local (start in the local
 *   layout), block_rows; *max_block_rows.  Negative counts or G*Eg > 65536 give
 *   MOE_ERR_INVALID_ARG.
 * moe_ep_reorder moves row blocks on `stream`: dst[dst_start[b] + i] = src[src_start[b] + i]
 *   for i < block_rows[b], rows of desc->D elements of desc->dtype; the three block arrays are
 *   device arrays of n_blocks int64; 16-byte aligned src and dst.  Receive buffer -> local
 *   layout with (block_recv, block_local); back with the two swapped. */
moe_status_t moe_ep_plan(int32_t G, int32_t Eg, const int32_t* rows_send,
                         const int32_t* rows_recv, int64_t* send_rows, int64_t* send_offsets,
                         int64_t* recv_rows, int64_t* recv_offsets, int32_t* local_offsets,
                         int64_t* block_recv, int64_t* block_local, int64_t* block_rows,
                         int64_t* max_block_rows);
moe_status_t moe_ep_reorder(const moe_desc_t* desc, int32_t n_blocks, const int64_t* src_start,
                            const int64_t* dst_start, const int64_t* block_rows,
                            int64_t max_block_rows, const void* src, void* dst,
                            moe_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word that kernels set when
 * a bounded wait gives up (MOE_ERR_TIMEOUT) or a device-side check fires (MOE_ERR_DEVICE).
 * *code receives the raw word (0 = none).  Returns MOE_OK when the word was 0. */
moe_status_t moe_get_device_error(moe_stream_t stream, int32_t* code);

/* Number of kernels this library has enqueued since it was loaded (all entry points, all
 * streams).  Host counter; useful to attribute launches in a timed region. */
int64_t moe_kernel_launches(void);

/* Test hook for the bounded device waits (failure detection without a GPU fault).  fault = 1:
 * in every following bf16 expert projection, CTA 0 of the grouped GEMM arms its first ring
 * stage without loading it, so the MMA issuer's bounded wait runs out (about 2 s); the CTA
 * records MOE_ERR_TIMEOUT in the device error word, drains what is in flight, frees its tensor
 * memory and exits, the other CTAs finish, and the context stays usable.  fault = 0 restores
 * normal operation.  Not for production use: the affected call's outputs are incomplete.
 * Host state only (not thread-safe); returns MOE_ERR_INVALID_ARG for other values. */
moe_status_t moe_debug_inject(int32_t fault);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
