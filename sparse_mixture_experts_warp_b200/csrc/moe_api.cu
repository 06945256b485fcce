// C ABI of the sm_100a sparse MoE FFN layer: argument validation, workspace carving and the
// launch chain.  The layer follows "Top-k 路由（Top-k Routing）" (compassingai), lifecycle
// Gate -> Dispatch -> Expert compute -> Combine, and "别只比较 Top-k" (ailearn
// moe-comparison), Score -> Select -> Merge -> Execute.  No entry point allocates, frees or
// synchronises (moe_get_device_error excepted); all work goes on the caller's stream.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "common.cuh"

namespace moe {

static __device__ int g_device_error = 0;

static std::atomic<int64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

bool pdl_enabled() {
  static const bool v = [] {
    const char* e = getenv("MOE_PDL");
    return !(e && e[0] == '0');
  }();
  return v;
}

int* device_error_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

namespace {

constexpr size_t kAlign = 256;
inline size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

moe_status_t validate(const moe_desc_t* d) {
  if (!d) return MOE_ERR_INVALID_ARG;
  if (d->T < 0 || d->D <= 0 || d->E <= 0 || d->F <= 0) return MOE_ERR_INVALID_ARG;
  if (d->score != MOE_SCORE_SOFTMAX && d->score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (d->select != MOE_TOKEN_CHOICE && d->select != MOE_EXPERT_CHOICE) return MOE_ERR_INVALID_ARG;
  if (d->gate != MOE_GATE_RENORM && d->gate != MOE_GATE_RAW) return MOE_ERR_INVALID_ARG;
  if (d->overflow != MOE_DROPLESS && d->overflow != MOE_CAPACITY_DROP) return MOE_ERR_INVALID_ARG;
  if (d->act != MOE_ACT_SWIGLU && d->act != MOE_ACT_RELU && d->act != MOE_ACT_GELU)
    return MOE_ERR_INVALID_ARG;
  if (d->dtype != MOE_F32 && d->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (d->n_shared < 0 || (d->n_shared > 0 && d->F_shared <= 0)) return MOE_ERR_INVALID_ARG;
  if (d->E > 256) return MOE_ERR_UNSUPPORTED;
  if (d->select == MOE_TOKEN_CHOICE) {
    if (d->k < 1 || d->k > d->E) return MOE_ERR_INVALID_ARG;
    if (d->k > 32) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)d->T * d->k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
    if (d->overflow == MOE_CAPACITY_DROP && !(d->capacity_factor > 0.f)) return MOE_ERR_INVALID_ARG;
  } else {
    if (d->c < 1 || d->c > d->T) return MOE_ERR_INVALID_ARG;
    if (d->score != MOE_SCORE_SOFTMAX) return MOE_ERR_UNSUPPORTED;
    if (d->overflow != MOE_DROPLESS) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)d->T * d->E >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  }
  if (!(d->aux_alpha >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (d->n_group < 0 || d->topk_group < 0) return MOE_ERR_INVALID_ARG;
  if (d->n_group > 1) {
    if (d->select != MOE_TOKEN_CHOICE) return MOE_ERR_UNSUPPORTED;
    if (d->E % d->n_group || d->topk_group < 1 || d->topk_group > d->n_group)
      return MOE_ERR_INVALID_ARG;
    const int size = d->E / d->n_group;
    if ((int64_t)d->topk_group * size < d->k) return MOE_ERR_INVALID_ARG;
    const bool pow2 = (size & (size - 1)) == 0;
    if (d->n_group > 32 || !((pow2 && size <= 32) || size % 32 == 0)) return MOE_ERR_UNSUPPORTED;
  }
  if (d->dtype == MOE_BF16) {
    if (d->D % 64 || d->F % 64) return MOE_ERR_UNSUPPORTED;
    if (d->n_shared > 0 && d->F_shared % 64) return MOE_ERR_UNSUPPORTED;
  } else {
    if (d->D % 4) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

int32_t capacity_of(const moe_desc_t* d) {
  if (d->select != MOE_TOKEN_CHOICE || d->overflow != MOE_CAPACITY_DROP) return 0;
  const double c = ceil((double)d->capacity_factor * (double)d->T * (double)d->k / (double)d->E);
  return (int32_t)c;
}

int64_t rows_of(const moe_desc_t* d) {
  if (d->select == MOE_EXPERT_CHOICE) return (int64_t)d->E * d->c;
  const int64_t A = (int64_t)d->T * d->k;
  if (d->overflow == MOE_CAPACITY_DROP) {
    const int64_t cap = (int64_t)d->E * capacity_of(d);
    return cap < A ? cap : A;
  }
  return A;
}

size_t esize(const moe_desc_t* d) { return d->dtype == MOE_BF16 ? 2 : 4; }

size_t route_scratch(const moe_desc_t* d) {
  size_t b = up((size_t)router_partials(*d) * (d->E + 1) * sizeof(float));
  if (d->select == MOE_EXPERT_CHOICE) b += up((size_t)d->E * d->T * sizeof(float));
  b += up(router_gemm_scratch_bytes(*d));
  return b;
}
size_t permute_scratch(const moe_desc_t* d) {
  if (d->select == MOE_EXPERT_CHOICE) return 0;
  return up((size_t)(permute_blocks(*d) > 0 ? permute_blocks(*d) : 1) * d->E * sizeof(int32_t));
}
// Small-batch (decode) schedule of the routed experts.  With few executed rows the grouped
// GEMM has fewer tiles than SMs (one token of the Mixtral layer: 2 experts x 16 output tiles of
// the down projection for 148 SMs), so the products are split along K into fp32 partials in
// the step scratch (free once the permutation is done) and summed by splitk.cu.  At most
// kMaxSplits splits; the up projection only for A <= kSplitUpRows, the down projection for
// A <= kSplitDownRows.  MOE_DECODE_SPLITK=0 turns the schedule off (comparison measurements).
constexpr int kMaxSplits = 8;
constexpr int64_t kSplitUpRows = 16, kSplitDownRows = 256;

bool decode_splitk_enabled() {
  static const bool v = [] {
    const char* e = getenv("MOE_DECODE_SPLITK");
    return !(e && e[0] == '0');
  }();
  return v;
}

// With at most kStreamKRows rows (64-row tiles: one per group) a split product whose S equal
// k-ranges per tile would take more than one wave of CTAs runs stream-K instead: every SM takes
// an equal contiguous share of all tiles' k-blocks, so no partly filled last wave leaves SMs
// idle; up to kMaxSplits partial slots per tile.  Mixtral width, one token: gate + up 94 -> 87
// us (448 equal ranges over 148 SMs before); the down product (128 ranges, one wave) keeps its
// equal ranges (stream-K measured 49 -> 51 us there).  MOE_STREAMK=0 keeps the equal ranges
// everywhere (comparison measurements).
constexpr int64_t kStreamKRows = 64;
constexpr int kStreamKGroups = 1024;
bool streamk_enabled() {
  static const bool v = [] {
    const char* e = getenv("MOE_STREAMK");
    return !(e && e[0] == '0');
  }();
  return v;
}

// Adaptive k-split of the down projection.  Under a capacity limit the executed rows can be
// far fewer than the host's bound (a few popular experts, each at its capacity: the Switch
// layer runs 413 of 8192 possible rows on 9 of 128 experts), and the down projection's tiles
// then leave most SMs idle.  The grouped GEMM reads the group table on the device and, when
// its tiles fill fewer than half of the CTAs, splits K into fp32 partials that
// launch_splitk_sum_adaptive sums.  Used where the smallest possible row count gives fewer
// tiles than a B200 has SMs (148), the only case in which a launch can be under-filled;
// MOE_ADAPTIVE_SPLIT=0 turns it off (comparison measurements).
constexpr int kSmBound = 148;
constexpr size_t kAdaptCapBytes = (size_t)24 << 20;   // partials of any split that fills the SMs

bool adaptive_split_enabled() {
  static const bool v = [] {
    const char* e = getenv("MOE_ADAPTIVE_SPLIT");
    return !(e && e[0] == '0');
  }();
  return v;
}

// Fewest rows the routed experts can execute: every token on the same k experts, each kept up
// to its capacity; expert choice always E * c.
int64_t min_rows_of(const moe_desc_t* d) {
  if (d->select == MOE_EXPERT_CHOICE) return (int64_t)d->E * d->c;
  const int64_t A = (int64_t)d->T * d->k;
  if (d->overflow != MOE_CAPACITY_DROP) return A;
  const int64_t cap = capacity_of(d);
  const int64_t m = (int64_t)d->k * (d->T < cap ? d->T : cap);
  return m < A ? m : A;
}

bool adaptive_down(const moe_desc_t* d) {
  if (d->dtype != MOE_BF16 || !decode_splitk_enabled() || !adaptive_split_enabled()) return false;
  if (rows_of(d) <= kSplitDownRows) return false;     // the small-batch schedule splits already
  const int64_t min_tiles = ((min_rows_of(d) + 255) / 256) * (((int64_t)d->D + 255) / 256);
  return min_tiles < kSmBound;
}

// fp32 partials (at most kAdaptCapBytes) and the split count after them
size_t adaptive_part_bytes(const moe_desc_t* d) {
  const size_t full = (size_t)kMaxSplits * rows_of(d) * d->D * sizeof(float);
  return up(full < kAdaptCapBytes ? full : kAdaptCapBytes);
}
size_t adaptive_bytes(const moe_desc_t* d) {
  return adaptive_down(d) ? adaptive_part_bytes(d) + kAlign : 0;
}

size_t splitk_up_bytes(const moe_desc_t* d, int64_t A) {     // one product's partials
  return up((size_t)kMaxSplits * A * ((int64_t)(d->F + 255) / 256 * 256) * sizeof(float));
}
size_t splitk_scratch(const moe_desc_t* d) {
  if (d->dtype != MOE_BF16) return 0;
  const int64_t A = rows_of(d);
  size_t b = 0;
  if (A <= kSplitDownRows) b = up((size_t)kMaxSplits * A * d->D * sizeof(float));
  if (A <= kSplitUpRows) {
    const size_t u = (d->act == MOE_ACT_SWIGLU ? 2 : 1) * splitk_up_bytes(d, A);
    if (u > b) b = u;
  }
  const size_t ad = adaptive_bytes(d);
  return ad > b ? ad : b;
}

size_t scratch_bytes(const moe_desc_t* d) {
  size_t a = route_scratch(d);
  const size_t b = permute_scratch(d), c = splitk_scratch(d);
  if (b > a) a = b;
  if (c > a) a = c;
  return a + kAlign;
}

// Fraction of the SM slots that a persistent launch of `units` equal work items keeps busy.
double sm_fill(int64_t units, int sms) {
  const int64_t waves = (units + sms - 1) / sms;
  return waves > 0 ? (double)units / (double)(waves * sms) : 0.0;
}

// Split count for a product of `units` output tiles over K: 1 when the unsplit launch fills
// at least 80% of the SM slots; otherwise the (effective) count in 2..kMaxSplits, each split
// at least 4 k-blocks, that fills the most slots (fewer splits unless 2 points better).
int choose_splits(int64_t units, int K, int sms) {
  const int nkb = (K + 63) / 64;
  double best_fill = sm_fill(units, sms);
  if (units <= 0 || best_fill >= 0.8) return 1;
  int best = 1;
  for (int S = 2; S <= kMaxSplits && S * 4 <= nkb; ++S) {
    const int se = splitk_count(K, S);
    const double f = sm_fill(units * se, sms);
    if (f > best_fill + 0.02) {
      best_fill = f;
      best = se;
    }
  }
  return best;
}

// Workspace layout of moe_layer_forward; with base == nullptr only the size is computed.
size_t carve(const moe_desc_t* d, uint8_t* base, moe_layer_views_t* v) {
  const int64_t T = d->T, E = d->E, A = rows_of(d);
  const bool ec = d->select == MOE_EXPERT_CHOICE;
  const int64_t K = ec ? E : d->k;
  const size_t es = esize(d);
  size_t off = 0;
  auto take = [&](size_t bytes) -> void* {
    void* p = base ? base + off : nullptr;
    off += up(bytes ? bytes : 1);
    return p;
  };
  moe_layer_views_t w;
  memset(&w, 0, sizeof(w));
  w.logits = static_cast<float*>(take(T * E * 4));
  w.expert_ids = static_cast<int32_t*>(take((ec ? E * d->c : T * K) * 4));
  w.gates = static_cast<float*>(take(T * K * 4));
  w.importance = static_cast<float*>(take(E * 4));
  w.entropy = static_cast<float*>(take(4));
  w.counts = static_cast<int32_t*>(take(E * 4));
  w.offsets = static_cast<int32_t*>(take((E + 1) * 4));
  w.row_src = static_cast<int32_t*>(take(A * 4));
  w.inv = static_cast<int32_t*>(take(T * K * 4));
  w.x_perm = take(A * d->D * es);
  w.h = take(A * d->F * es);
  w.y = take(A * d->D * es);
  if (d->n_shared > 0) {
    w.h_shared = take(T * d->F_shared * es);
    w.y_shared = take((int64_t)d->n_shared * T * d->D * es);
    w.shared_offsets = static_cast<int32_t*>(take(2 * 4));
  }
  w.f = static_cast<float*>(take(E * 4));
  w.stats = static_cast<moe_stats_t*>(take(sizeof(moe_stats_t)));
  const size_t sb = scratch_bytes(d);
  w.scratch = take(sb);
  w.scratch_bytes = sb;
  w.rows = A;
  if (v) *v = w;
  return off;
}

inline moe_status_t cuda_status(cudaError_t e) {
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

__global__ void set_offsets_kernel(int32_t* o, int T) {
  pdl_trigger();
  pdl_wait();
  o[0] = 0;
  o[1] = T;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace too small or misaligned";
    case MOE_ERR_CUDA: return "CUDA launch error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

moe_status_t moe_rows_max(const moe_desc_t* d, int64_t* rows) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (!rows) return MOE_ERR_INVALID_ARG;
  *rows = rows_of(d);
  return MOE_OK;
}

moe_status_t moe_capacity(const moe_desc_t* d, int32_t* c) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (!c) return MOE_ERR_INVALID_ARG;
  *c = capacity_of(d);
  return MOE_OK;
}

moe_status_t moe_scratch_size(const moe_desc_t* d, size_t* bytes) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = scratch_bytes(d);
  return MOE_OK;
}

moe_status_t moe_workspace_size(const moe_desc_t* d, size_t* bytes) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = carve(d, nullptr, nullptr);
  return MOE_OK;
}

moe_status_t moe_layer_views(const moe_desc_t* d, void* ws, size_t ws_bytes,
                             moe_layer_views_t* v) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (!ws || !v) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return MOE_ERR_WORKSPACE;
  if (ws_bytes < carve(d, nullptr, nullptr)) return MOE_ERR_WORKSPACE;
  carve(d, static_cast<uint8_t*>(ws), v);
  return MOE_OK;
}

moe_status_t moe_route(const moe_desc_t* d, const void* x, const void* Wg, const float* sel_bias,
                       int32_t* expert_ids, float* gates, float* logits, float* importance,
                       float* entropy, void* scratch, size_t scratch_bytes_,
                       moe_stream_t stream) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (d->T == 0) return MOE_OK;
  if (!x || !Wg || !expert_ids || !gates || !scratch) return MOE_ERR_INVALID_ARG;
  if (!is_aligned16(x) || !is_aligned16(Wg)) return MOE_ERR_INVALID_ARG;
  if (scratch_bytes_ < scratch_bytes(d)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* sc = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(scratch) + kAlign - 1) &
                                           ~(uintptr_t)(kAlign - 1));
  float* partials = reinterpret_cast<float*>(sc);
  const size_t pbytes = up((size_t)router_partials(*d) * (d->E + 1) * sizeof(float));
  const size_t tbytes = d->select == MOE_EXPERT_CHOICE ? up((size_t)d->E * d->T * sizeof(float)) : 0;
  float* lpart = router_uses_gemm(*d) ? reinterpret_cast<float*>(sc + pbytes + tbytes) : nullptr;
  int np = 0;
  cudaError_t e;
  if (d->select == MOE_TOKEN_CHOICE) {
    e = launch_router_token_choice(*d, x, Wg, d->score == MOE_SCORE_SIGMOID ? sel_bias : nullptr,
                                   expert_ids, gates, logits, partials, &np, lpart, s);
  } else {
    float* probsT = reinterpret_cast<float*>(sc + pbytes);
    e = launch_router_expert_choice(*d, x, Wg, gates, probsT, logits, partials, &np, lpart, s);
    if (e == cudaSuccess) e = launch_ec_select(*d, probsT, expert_ids, s);
  }
  if (e == cudaSuccess && (importance || entropy))
    e = launch_importance_reduce(partials, np, d->E, d->T, importance, entropy, s);
  return cuda_status(e);
}

moe_status_t moe_permute(const moe_desc_t* d, const int32_t* expert_ids, const void* x,
                         void* x_perm, int32_t* counts, int32_t* offsets, int32_t* row_src,
                         int32_t* inv, void* scratch, size_t scratch_bytes_,
                         moe_stream_t stream) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  // x_perm == NULL: indices only (the rows are gathered later, by moe_expert_up_gather)
  if (!expert_ids || !x || !counts || !offsets || !row_src || !inv) return MOE_ERR_INVALID_ARG;
  if (!is_aligned16(x) || (x_perm && !is_aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (d->select == MOE_TOKEN_CHOICE) {
    if (!scratch || scratch_bytes_ < scratch_bytes(d)) return MOE_ERR_WORKSPACE;
    int32_t* hist = reinterpret_cast<int32_t*>(
        (reinterpret_cast<uintptr_t>(scratch) + kAlign - 1) & ~(uintptr_t)(kAlign - 1));
    e = launch_permute_token_choice(*d, expert_ids, x, x_perm, counts, offsets, row_src, inv,
                                    hist, capacity_of(d), s);
  } else {
    e = launch_permute_expert_choice(*d, expert_ids, x, x_perm, counts, offsets, row_src, inv, s);
  }
  return cuda_status(e);
}

static moe_status_t check_ffn(const moe_desc_t* d, int32_t G, int32_t F, const void* a,
                              int64_t a_rows, const int32_t* offsets) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (G < 1 || G > 1024 || F <= 0 || a_rows < 0 || !a || !offsets) return MOE_ERR_INVALID_ARG;
  if (!is_aligned16(a)) return MOE_ERR_INVALID_ARG;
  if (d->dtype == MOE_BF16 && (F % 64)) return MOE_ERR_UNSUPPORTED;
  if (a_rows >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t moe_expert_up(const moe_desc_t* d, int32_t G, int32_t F, const void* a,
                           int64_t a_rows, const int32_t* offsets, const void* W_gate,
                           const void* W_up, void* h, moe_stream_t stream) {
  moe_status_t st = check_ffn(d, G, F, a, a_rows, offsets);
  if (st != MOE_OK) return st;
  if (!W_up || !h || (d->act == MOE_ACT_SWIGLU && !W_gate)) return MOE_ERR_INVALID_ARG;
  if (!is_aligned16(W_up) || !is_aligned16(h) || (W_gate && !is_aligned16(W_gate)))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (d->dtype == MOE_BF16) {
    if (d->act == MOE_ACT_SWIGLU)
      e = launch_grouped_gemm_bf16(EPI_SWIGLU, a, a_rows, d->D, W_gate, W_up, G, F, offsets, h, s);
    else
      e = launch_grouped_gemm_bf16(d->act == MOE_ACT_GELU ? EPI_GELU : EPI_RELU, a, a_rows, d->D,
                                   W_up, nullptr, G, F, offsets, h, s);
  } else {
    e = launch_ffn_up_f32(d->act, static_cast<const float*>(a), a_rows, d->D, F, offsets, G,
                          static_cast<const float*>(W_gate), static_cast<const float*>(W_up),
                          static_cast<float*>(h), s);
  }
  return cuda_status(e);
}

moe_status_t moe_expert_down(const moe_desc_t* d, int32_t G, int32_t F, const void* h,
                             int64_t a_rows, const int32_t* offsets, const void* W_down, void* y,
                             moe_stream_t stream) {
  moe_status_t st = check_ffn(d, G, F, h, a_rows, offsets);
  if (st != MOE_OK) return st;
  if (!W_down || !y) return MOE_ERR_INVALID_ARG;
  if (!is_aligned16(W_down) || !is_aligned16(y)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (d->dtype == MOE_BF16)
    e = launch_grouped_gemm_bf16(EPI_NONE, h, a_rows, F, W_down, nullptr, G, d->D, offsets, y, s);
  else
    e = launch_ffn_down_f32(static_cast<const float*>(h), a_rows, d->D, F, offsets, G,
                            static_cast<const float*>(W_down), static_cast<float*>(y), s);
  return cuda_status(e);
}

moe_status_t moe_expert_ffn(const moe_desc_t* d, int32_t G, int32_t F, const void* a,
                            int64_t a_rows, const int32_t* offsets, const void* W_gate,
                            const void* W_up, const void* W_down, void* h, void* y,
                            moe_stream_t stream) {
  moe_status_t st = moe_expert_up(d, G, F, a, a_rows, offsets, W_gate, W_up, h, stream);
  if (st != MOE_OK) return st;
  return moe_expert_down(d, G, F, h, a_rows, offsets, W_down, y, stream);
}

// Off unless MOE_GATHER_FUSION=1: the gathering up projection is correct but measured slower
// than writing x_perm and loading it with tiled boxes (its A stages take 64 four-row gathers
// instead of two tiled boxes).
static bool gather_fusion_enabled() {
  static const bool v = [] {
    const char* s = getenv("MOE_GATHER_FUSION");
    return s && s[0] == '1';
  }();
  return v;
}

moe_status_t moe_gather_fusion(const moe_desc_t* d, int32_t* on) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (!on) return MOE_ERR_INVALID_ARG;
  *on = (d->dtype == MOE_BF16 && gather_fusion_enabled() && gemm_gather_ok() &&
         rows_of(d) > kSplitUpRows)
            ? 1
            : 0;
  return MOE_OK;
}

moe_status_t moe_expert_up_gather(const moe_desc_t* d, int32_t G, int32_t F, const void* x,
                                  const int32_t* row_src, int64_t a_rows,
                                  const int32_t* offsets, const void* W_gate, const void* W_up,
                                  void* h, moe_stream_t stream) {
  moe_status_t st = check_ffn(d, G, F, x, a_rows, offsets);
  if (st != MOE_OK) return st;
  if (d->dtype != MOE_BF16 || !gemm_gather_ok()) return MOE_ERR_UNSUPPORTED;
  if (!row_src || !W_up || !h || (d->act == MOE_ACT_SWIGLU && !W_gate))
    return MOE_ERR_INVALID_ARG;
  if (!is_aligned16(W_up) || !is_aligned16(h) || (W_gate && !is_aligned16(W_gate)))
    return MOE_ERR_INVALID_ARG;
  if (d->T == 0 || a_rows == 0) return MOE_OK;
  const int div = d->select == MOE_EXPERT_CHOICE ? d->E : d->k;
  const bool glu = d->act == MOE_ACT_SWIGLU;
  const int epi = glu ? EPI_SWIGLU : (d->act == MOE_ACT_GELU ? EPI_GELU : EPI_RELU);
  return cuda_status(launch_grouped_gemm_bf16(epi, x, a_rows, d->D, glu ? W_gate : W_up,
                                              glu ? W_up : nullptr, G, F, offsets, h,
                                              reinterpret_cast<cudaStream_t>(stream), nullptr,
                                              row_src, div, d->T));
}

// ---- the small-batch (decode) schedule: k-split products, see kMaxSplits ----

// Scratch of at least `need` bytes at a 256-byte boundary inside [scratch, +bytes), or null.
static float* splitk_space(void* scratch, size_t bytes, size_t need) {
  if (!scratch) return nullptr;
  const uintptr_t b = reinterpret_cast<uintptr_t>(scratch);
  const uintptr_t a = (b + kAlign - 1) & ~(uintptr_t)(kAlign - 1);
  if (a - b > bytes || bytes - (a - b) < need) return nullptr;
  return reinterpret_cast<float*>(a);
}

moe_status_t moe_expert_up_ws(const moe_desc_t* d, int32_t G, int32_t F, const void* a,
                              int64_t a_rows, const int32_t* offsets, const void* W_gate,
                              const void* W_up, void* h, void* scratch, size_t scratch_bytes,
                              moe_stream_t stream) {
  moe_status_t st = check_ffn(d, G, F, a, a_rows, offsets);
  if (st != MOE_OK) return st;
  const bool glu = d->act == MOE_ACT_SWIGLU;
  int S = 1;
  if (d->dtype == MOE_BF16 && decode_splitk_enabled() && a_rows > 0 && a_rows <= kSplitUpRows &&
      h && W_up && is_aligned16(W_up) && is_aligned16(h) &&
      (!glu || (W_gate && is_aligned16(W_gate)))) {
    // fused: SwiGLU tiles hold 128 features (gate and up side by side), others 256 columns;
    // split: gate and up are separate products of 256-column tiles
    // split: SwiGLU's gate and up products in one launch of 256-column tiles (n-tiles of W_up
    // after those of W_gate), others one product
    const int sms = gemm_sm_count();
    const int64_t active = a_rows < G ? a_rows : G;
    const int64_t fused = active * ((F + (glu ? 127 : 255)) / (glu ? 128 : 256));
    const int64_t units = active * ((F + 255) / 256) * (glu ? 2 : 1);
    const double fill_fused = sm_fill(fused, sms);
    if (units >= sms) {
      // at least a full wave of split tiles already: two k-ranges when the fused product
      // fills its last wave poorly.  Fewer, longer weight streams per tile measured faster
      // than the fullest last wave (Mixtral width, gate + up: 1 token 0.165 -> 0.153 ms with
      // 2 instead of 5 k-ranges, 2 tokens 0.293 -> 0.269 ms; 3 to 8 ranges all slower)
      if (fill_fused < 0.8 && d->D / 64 >= 8) S = 2;
    } else {
      const int c = choose_splits(units, d->D, sms);
      if (c > 1 && fill_fused < 0.8 && sm_fill(units * c, sms) > fill_fused + 0.05) S = c;
    }
  }
  // partial rows: [gate | up] blocks of ceil(F / 256) * 256 columns each (SwiGLU), F otherwise
  const int64_t fpad = (int64_t)(F + 255) / 256 * 256;
  const int64_t ld = glu ? 2 * fpad : F;
  // at most 64 rows, and S equal k-ranges per tile would take more than one wave of CTAs:
  // stream-K over all SMs (every CTA an equal share of the tiles' k-blocks, up to kMaxSplits
  // partial slots per tile), so that no partly filled last wave remains
  const int64_t split_units =
      (int64_t)(a_rows < G ? a_rows : G) * ((F + 255) / 256) * (glu ? 2 : 1);
  const bool sk = S > 1 && streamk_enabled() && a_rows <= kStreamKRows && F % 4 == 0 &&
                  G <= kStreamKGroups && split_units * S > gemm_sm_count();
  const int slots = sk ? kMaxSplits : S;
  float* part = S > 1 ? splitk_space(scratch, scratch_bytes,
                                     (size_t)slots * a_rows * ld * sizeof(float))
                      : nullptr;
  if (!part)
    return moe_expert_up(d, G, F, a, a_rows, offsets, W_gate, W_up, h, stream);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = glu ? launch_grouped_gemm_f32_splitk2(a, a_rows, d->D, W_gate, W_up, G, F,
                                                         offsets, S, part, s, sk ? slots : 0)
                      : launch_grouped_gemm_f32_splitk(a, a_rows, d->D, W_up, G, F, offsets, S,
                                                       part, s, sk ? slots : 0);
  if (e == cudaSuccess && sk)
    e = launch_splitk_streamk(d->act, part, slots, a_rows, (int)ld, F, d->D, glu ? 1 : 0,
                              offsets, G, h, s);
  else if (e == cudaSuccess)
    e = launch_splitk_act(d->act, part, glu ? part + fpad : part, S, a_rows, F, offsets + G, h, s,
                          ld);
  return cuda_status(e);
}

// defer != nullptr: when the device-side k-split runs, its partials are left for the combine
// (described in *defer; defer->part stays null otherwise).
static moe_status_t down_ws_impl(const moe_desc_t* d, int32_t G, int32_t F, const void* h,
                                 int64_t a_rows, const int32_t* offsets, const void* W_down,
                                 void* y, void* scratch, size_t scratch_bytes,
                                 moe_stream_t stream, SplitRows* defer);

moe_status_t moe_expert_down_ws(const moe_desc_t* d, int32_t G, int32_t F, const void* h,
                                int64_t a_rows, const int32_t* offsets, const void* W_down,
                                void* y, void* scratch, size_t scratch_bytes,
                                moe_stream_t stream) {
  return down_ws_impl(d, G, F, h, a_rows, offsets, W_down, y, scratch, scratch_bytes, stream,
                      nullptr);
}

static moe_status_t down_ws_impl(const moe_desc_t* d, int32_t G, int32_t F, const void* h,
                                 int64_t a_rows, const int32_t* offsets, const void* W_down,
                                 void* y, void* scratch, size_t scratch_bytes,
                                 moe_stream_t stream, SplitRows* defer) {
  moe_status_t st = check_ffn(d, G, F, h, a_rows, offsets);
  if (st != MOE_OK) return st;
  int S = 1;
  if (d->dtype == MOE_BF16 && decode_splitk_enabled() && a_rows > 0 &&
      a_rows <= kSplitDownRows && W_down && y && is_aligned16(W_down) && is_aligned16(y)) {
    const int64_t active = a_rows < G ? a_rows : G;
    S = choose_splits(active * ((d->D + 255) / 256), F, gemm_sm_count());
  }
  const int64_t split_units = (int64_t)(a_rows < G ? a_rows : G) * ((d->D + 255) / 256);
  const bool sk = S > 1 && streamk_enabled() && a_rows <= kStreamKRows && d->D % 4 == 0 &&
                  G <= kStreamKGroups && split_units * S > gemm_sm_count();
  const int slots = sk ? kMaxSplits : S;
  float* part = S > 1 ? splitk_space(scratch, scratch_bytes,
                                     (size_t)slots * a_rows * d->D * sizeof(float))
                      : nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!part && adaptive_down(d) && W_down && y && is_aligned16(W_down) && is_aligned16(y) &&
      d->D % 4 == 0) {
    float* ap = splitk_space(scratch, scratch_bytes, adaptive_part_bytes(d) + kAlign);
    if (ap) {
      const size_t pb = adaptive_part_bytes(d);
      int* ks = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(ap) + pb);
      cudaError_t e = launch_grouped_gemm_bf16(EPI_NONE, h, a_rows, F, W_down, nullptr, G, d->D,
                                               offsets, y, s, nullptr, nullptr, 1, 0, ap,
                                               (int64_t)(pb / sizeof(float)), kMaxSplits, ks);
      if (e == cudaSuccess && defer) {
        *defer = SplitRows{ap, ks, offsets + G, a_rows, nullptr};
        return MOE_OK;
      }
      if (e == cudaSuccess) e = launch_splitk_sum_adaptive(ap, ks, a_rows, d->D, offsets + G, y, s);
      return cuda_status(e);
    }
  }
  if (!part) return moe_expert_down(d, G, F, h, a_rows, offsets, W_down, y, stream);
  cudaError_t e = launch_grouped_gemm_f32_splitk(h, a_rows, F, W_down, G, d->D, offsets, S, part,
                                                 s, sk ? slots : 0);
  // (the decode split keeps its own summing kernel: with a handful of tokens the combine is a
  // warp or two, and the sum needs the whole GPU's loads in flight; measured at one token:
  // 0.160 against 0.183 ms with the sum inside the combine)
  if (e == cudaSuccess && sk)
    e = launch_splitk_streamk(-1, part, slots, a_rows, d->D, d->D, F, 0, offsets, G, y, s);
  else if (e == cudaSuccess)
    e = launch_splitk_sum(part, S, a_rows, d->D, offsets + G, y, s);
  return cuda_status(e);
}

moe_status_t moe_combine(const moe_desc_t* d, const void* y, const int32_t* inv,
                         const float* gates, const void* y_shared, void* out,
                         moe_stream_t stream) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (!y || !inv || !gates || !out) return MOE_ERR_INVALID_ARG;
  if (!is_aligned16(y) || !is_aligned16(out) || (y_shared && !is_aligned16(y_shared)))
    return MOE_ERR_INVALID_ARG;
  if (y_shared && d->n_shared == 0) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine(*d, y, inv, gates, y_shared, out,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_balance_stats(const moe_desc_t* d, const int32_t* counts, const int32_t* offsets,
                               const float* importance, const float* entropy, float* f,
                               moe_stats_t* stats, moe_stream_t stream) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (!counts || !offsets || !importance || !f || !stats) return MOE_ERR_INVALID_ARG;
  if (d->select == MOE_TOKEN_CHOICE ? d->T * d->k == 0 : d->E * d->c == 0) return MOE_OK;
  return cuda_status(launch_balance_stats(*d, counts, offsets, importance, entropy, f, stats,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

static moe_status_t forward_impl(const moe_desc_t* d, const void* x, const void* Wg,
                                 const float* sel_bias, const void* W_gate, const void* W_up,
                                 const void* W_down, const void* Ws_gate, const void* Ws_up,
                                 const void* Ws_down, void* out, void* ws, size_t ws_bytes,
                                 void* preact, moe_stream_t stream);

moe_status_t moe_layer_forward(const moe_desc_t* d, const void* x, const void* Wg,
                               const float* sel_bias, const void* W_gate, const void* W_up,
                               const void* W_down, const void* Ws_gate, const void* Ws_up,
                               const void* Ws_down, void* out, void* ws, size_t ws_bytes,
                               moe_stream_t stream) {
  return forward_impl(d, x, Wg, sel_bias, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, out,
                      ws, ws_bytes, nullptr, stream);
}

// preact != nullptr (bf16 token choice, from moe_layer_forward_train): the routed up
// projection also stores its raw accumulators there for the backward pass.
static moe_status_t forward_impl(const moe_desc_t* d, const void* x, const void* Wg,
                                 const float* sel_bias, const void* W_gate, const void* W_up,
                                 const void* W_down, const void* Ws_gate, const void* Ws_up,
                                 const void* Ws_down, void* out, void* ws, size_t ws_bytes,
                                 void* preact, moe_stream_t stream) {
  moe_layer_views_t v;
  moe_status_t st = moe_layer_views(d, ws, ws_bytes, &v);
  if (st != MOE_OK) return st;
  if (!x || !Wg || !W_up || !W_down || !out) return MOE_ERR_INVALID_ARG;
  if (d->act == MOE_ACT_SWIGLU && !W_gate) return MOE_ERR_INVALID_ARG;
  if (d->n_shared > 0 && (!Ws_gate || !Ws_up || !Ws_down)) return MOE_ERR_INVALID_ARG;
  if (d->T == 0) return MOE_OK;
  st = moe_route(d, x, Wg, sel_bias, v.expert_ids, v.gates, v.logits, v.importance, v.entropy,
                 v.scratch, v.scratch_bytes, stream);
  if (st != MOE_OK) return st;
  // with enough rows (bf16), the up projection gathers the token rows itself and the
  // permutation writes indices only
  int32_t gather = 0;
  if (!preact) moe_gather_fusion(d, &gather);
  st = moe_permute(d, v.expert_ids, x, gather ? nullptr : v.x_perm, v.counts, v.offsets,
                   v.row_src, v.inv, v.scratch, v.scratch_bytes, stream);
  if (st != MOE_OK) return st;
  // without shared experts the combine sums a device-side k-split of the down projection
  // itself (one launch fewer)
  SplitRows split{};
  SplitRows* defer = d->n_shared == 0 ? &split : nullptr;
  if (gather) {
    st = moe_expert_up_gather(d, d->E, d->F, x, v.row_src, v.rows, v.offsets, W_gate, W_up, v.h,
                              stream);
    if (st == MOE_OK)
      st = down_ws_impl(d, d->E, d->F, v.h, v.rows, v.offsets, W_down, v.y, v.scratch,
                        v.scratch_bytes, stream, defer);
  } else if (preact) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool glu = d->act == MOE_ACT_SWIGLU;
    cudaError_t e = launch_grouped_gemm_bf16(
        glu ? EPI_SWIGLU : (d->act == MOE_ACT_GELU ? EPI_GELU : EPI_RELU), v.x_perm, v.rows,
        d->D, glu ? W_gate : W_up, glu ? W_up : nullptr, d->E, d->F, v.offsets, v.h, s, preact);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    st = moe_expert_down(d, d->E, d->F, v.h, v.rows, v.offsets, W_down, v.y, stream);
  } else {
    // the step scratch is free once the permutation is done: the small-batch schedule's
    // partials go there
    st = moe_expert_up_ws(d, d->E, d->F, v.x_perm, v.rows, v.offsets, W_gate, W_up, v.h,
                          v.scratch, v.scratch_bytes, stream);
    if (st == MOE_OK)
      st = down_ws_impl(d, d->E, d->F, v.h, v.rows, v.offsets, W_down, v.y, v.scratch,
                        v.scratch_bytes, stream, defer);
  }
  if (st != MOE_OK) return st;
  if (d->n_shared > 0) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    (void)launch_pdl(set_offsets_kernel, dim3(1), dim3(1), 0, s, v.shared_offsets, d->T);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    // shared experts always use SwiGLU
    moe_desc_t ds = *d;
    ds.act = MOE_ACT_SWIGLU;
    const size_t es = esize(d);
    const int64_t wstride_up = (int64_t)d->F_shared * d->D * es;
    for (int i = 0; i < d->n_shared; ++i) {
      const uint8_t* gw = static_cast<const uint8_t*>(Ws_gate) + i * wstride_up;
      const uint8_t* uw = static_cast<const uint8_t*>(Ws_up) + i * wstride_up;
      const uint8_t* dw = static_cast<const uint8_t*>(Ws_down) + i * wstride_up;
      uint8_t* ys = static_cast<uint8_t*>(v.y_shared) + (int64_t)i * d->T * d->D * es;
      st = moe_expert_ffn(&ds, 1, d->F_shared, x, d->T, v.shared_offsets, gw, uw, dw, v.h_shared,
                          ys, stream);
      if (st != MOE_OK) return st;
    }
  }
  // the combine's first block also computes the balance statistics (the stages of
  // moe_combine and moe_balance_stats in one launch)
  if (!is_aligned16(out)) return MOE_ERR_INVALID_ARG;
  const StatsArgs sa = stats_args(*d, v.counts, v.offsets, v.importance, v.entropy, v.f, v.stats);
  return cuda_status(launch_combine(*d, v.y, v.inv, v.gates,
                                    d->n_shared > 0 ? v.y_shared : nullptr, out,
                                    reinterpret_cast<cudaStream_t>(stream), &sa,
                                    split.part ? &split : nullptr));
}

// ---------------- backward ----------------

namespace {

struct BwdViews {
  int32_t* pad_off;
  void *dY, *gu, *dH, *dAB, *dXp, *WdT, *WguT, *dYT, *hT, *xpT, *dABT;
  float *dgates, *ds, *dwg_part;
  int64_t ldg, nab, pad_cols;
  // shared experts (n_shared > 0): one group of all T tokens each
  int32_t* pad_off_s;
  void *gu_s, *dH_s, *dAB_s, *h_s, *dXs, *doutT, *xT, *hT_s, *dABT_s;
  int64_t ldg_s, pad_cols_s;
};

bool bwd_weight_transpose() {
  static const bool v = [] {
    const char* s = getenv("MOE_BWD_WEIGHT_TRANSPOSE");
    return s && s[0] == '1';
  }();
  return v;
}

moe_status_t check_backward(const moe_desc_t* d) {
  moe_status_t st = validate(d);
  if (st != MOE_OK) return st;
  if (d->E > 256) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Backward workspace layout; with base == nullptr only the size is computed.  fp32 layers use
// their own layout (backward_f32.cu); only its size is returned here.
size_t carve_bwd(const moe_desc_t* d, uint8_t* base, BwdViews* v) {
  if (d->dtype == MOE_F32) {
    memset(v, 0, sizeof *v);
    return backward_f32_workspace(*d, rows_of(d));
  }
  const int64_t T = d->T, D = d->D, E = d->E, F = d->F, A = rows_of(d);
  const bool glu = d->act == MOE_ACT_SWIGLU;
  v->ldg = glu ? (F + 127) / 128 * 256 : F;
  v->nab = glu ? 2 * F : F;
  v->pad_cols = (A + 64 * E + 63) / 64 * 64;
  size_t off = 0;
  auto take = [&](size_t bytes) -> void* {
    void* p = base ? base + off : nullptr;
    off += up(bytes);
    return p;
  };
  const int64_t K = d->select == MOE_EXPERT_CHOICE ? E : d->k;
  v->pad_off = static_cast<int32_t*>(take((E + 1) * 4));
  v->dY = take(A * D * 2);
  v->dgates = static_cast<float*>(take(T * K * 4));
  v->gu = take(A * v->ldg * 2);
  v->dH = take(A * F * 2);
  v->dAB = take(A * v->nab * 2);
  v->dXp = take(A * D * 2);
  v->ds = static_cast<float*>(take(T * E * 4));
  const bool tw = bwd_weight_transpose();
  v->WdT = take(tw ? E * F * D * 2 : 0);
  v->WguT = take(tw ? E * D * v->nab * 2 : 0);
  v->dYT = take(D * v->pad_cols * 2);
  v->hT = take(F * v->pad_cols * 2);
  v->xpT = take(D * v->pad_cols * 2);
  v->dABT = take(v->nab * v->pad_cols * 2);
  v->dwg_part = static_cast<float*>(take((size_t)backward_dwg_chunks(d->T) * E * D * 4));
  const int64_t S = d->n_shared, Fs = d->F_shared;
  v->ldg_s = S ? (Fs + 127) / 128 * 256 : 0;
  v->pad_cols_s = S ? (T + 63) / 64 * 64 : 0;
  const int64_t pcs = v->pad_cols_s;
  v->pad_off_s = static_cast<int32_t*>(take(S ? 2 * 4 : 0));
  v->gu_s = take(S ? T * v->ldg_s * 2 : 0);
  v->dH_s = take(S ? T * Fs * 2 : 0);
  v->dAB_s = take(S ? T * 2 * Fs * 2 : 0);
  v->h_s = take(S ? T * Fs * 2 : 0);
  v->dXs = take(S * T * D * 2);
  v->doutT = take(S ? D * pcs * 2 : 0);
  v->xT = take(S ? D * pcs * 2 : 0);
  v->hT_s = take(S ? Fs * pcs * 2 : 0);
  v->dABT_s = take(S ? 2 * Fs * pcs * 2 : 0);
  return off;
}

// The shared experts' backward ("别只比较 Top-k" family table, DeepSeek rows: always-on shared
// experts on the direct path, weight 1): for expert i, with the recomputed pre-activations
// a | b = x [Ws_gate[i] ; Ws_up[i]]^T, dH = dout Ws_down[i], [da | db] and h from the SwiGLU
// derivative, dXs[i] = [da | db] [Ws_gate[i] ; Ws_up[i]], dWs_down[i] = dout^T h,
// dWs_gate[i] = da^T x, dWs_up[i] = db^T x (fp32, groups along K of one group).
cudaError_t shared_backward(const moe_desc_t* d, const moe_layer_views_t& v, const BwdViews& b,
                            const void* x, const moe_bwd_shared_t* sh, const void* dout,
                            cudaStream_t s) {
  const int T = d->T, D = d->D, Fs = d->F_shared, S = d->n_shared;
  const int64_t pcs = b.pad_cols_s;
  const int64_t wst = (int64_t)Fs * D;           // elements per shared weight matrix
  cudaError_t e = launch_pad_offsets(v.shared_offsets, 1, b.pad_off_s, s);
  if (e == cudaSuccess)
    e = launch_transpose_pad(dout, D, D, v.shared_offsets, b.pad_off_s, 1, pcs, b.doutT, pcs, s);
  if (e == cudaSuccess)
    e = launch_transpose_pad(x, D, D, v.shared_offsets, b.pad_off_s, 1, pcs, b.xT, pcs, s);
  for (int i = 0; i < S && e == cudaSuccess; ++i) {
    const __nv_bfloat16* wg = static_cast<const __nv_bfloat16*>(sh->Ws_gate) + i * wst;
    const __nv_bfloat16* wu = static_cast<const __nv_bfloat16*>(sh->Ws_up) + i * wst;
    const __nv_bfloat16* wd = static_cast<const __nv_bfloat16*>(sh->Ws_down) + i * wst;
    void* dxs = static_cast<__nv_bfloat16*>(b.dXs) + (int64_t)i * T * D;
    e = launch_grouped_gemm_bf16(EPI_RAW, x, T, D, wg, wu, 1, Fs, v.shared_offsets, b.gu_s, s);
    if (e == cudaSuccess)
      e = launch_grouped_gemm_bf16_bmn(dout, T, D, wd, nullptr, D / 64, D, 1, Fs,
                                       v.shared_offsets, b.dH_s, s);
    if (e == cudaSuccess)
      e = launch_act_backward(MOE_ACT_SWIGLU, b.dH_s, b.gu_s, b.ldg_s, v.shared_offsets, 1, Fs,
                              T, b.dAB_s, s, b.h_s);
    if (e == cudaSuccess)
      e = launch_grouped_gemm_bf16_bmn(b.dAB_s, T, 2 * Fs, wg, wu, Fs / 64, Fs, 1, D,
                                       v.shared_offsets, dxs, s);
    if (e == cudaSuccess)
      e = launch_transpose_pad(b.h_s, Fs, Fs, v.shared_offsets, b.pad_off_s, 1, pcs, b.hT_s, pcs,
                               s);
    if (e == cudaSuccess)
      e = launch_grouped_gemm_kgroups_f32(b.doutT, D, b.hT_s, Fs, 1, b.pad_off_s, pcs,
                                          sh->dWs_down + i * wst, s);
    if (e == cudaSuccess)
      e = launch_transpose_pad(b.dAB_s, 2 * Fs, 2 * Fs, v.shared_offsets, b.pad_off_s, 1, pcs,
                               b.dABT_s, pcs, s);
    if (e == cudaSuccess)
      e = launch_grouped_gemm_kgroups_f32(b.dABT_s, Fs, b.xT, D, 1, b.pad_off_s, pcs,
                                          sh->dWs_gate + i * wst, s);
    if (e == cudaSuccess)
      e = launch_grouped_gemm_kgroups_f32(static_cast<const __nv_bfloat16*>(b.dABT_s) +
                                              (int64_t)Fs * pcs,
                                          Fs, b.xT, D, 1, b.pad_off_s, pcs,
                                          sh->dWs_up + i * wst, s);
  }
  return e;
}

}  // namespace

moe_status_t moe_backward_workspace_size(const moe_desc_t* d, size_t* bytes) {
  moe_status_t st = check_backward(d);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  BwdViews v;
  *bytes = carve_bwd(d, nullptr, &v);
  return MOE_OK;
}

moe_status_t moe_layer_forward_train(const moe_desc_t* d, const void* x, const void* Wg,
                                     const float* sel_bias, const void* W_gate,
                                     const void* W_up, const void* W_down, void* out, void* ws,
                                     size_t ws_bytes, void* bwd_ws, size_t bwd_ws_bytes,
                                     moe_stream_t stream) {
  moe_status_t st = check_backward(d);
  if (st != MOE_OK) return st;
  // shared experts and fp32 layers: moe_layer_forward, then the backward with flags 0
  if (d->n_shared > 0 || d->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  BwdViews b;
  if (!bwd_ws || bwd_ws_bytes < carve_bwd(d, nullptr, &b)) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(bwd_ws) % kAlign) != 0) return MOE_ERR_WORKSPACE;
  carve_bwd(d, static_cast<uint8_t*>(bwd_ws), &b);
  return forward_impl(d, x, Wg, sel_bias, W_gate, W_up, W_down, nullptr, nullptr, nullptr, out,
                      ws, ws_bytes, b.gu, stream);
}

moe_status_t moe_layer_backward(const moe_desc_t* d, const void* x, const void* Wg,
                                const void* W_gate, const void* W_up, const void* W_down,
                                const void* dout, float aux_grad, void* fwd_ws,
                                size_t fwd_ws_bytes, void* dx, float* dWg, float* dW_gate,
                                float* dW_up, float* dW_down, void* bwd_ws,
                                size_t bwd_ws_bytes, int32_t flags, moe_stream_t stream) {
  return moe_layer_backward_ex(d, x, Wg, W_gate, W_up, W_down, nullptr, dout, aux_grad, fwd_ws,
                               fwd_ws_bytes, dx, dWg, dW_gate, dW_up, dW_down, bwd_ws,
                               bwd_ws_bytes, flags, stream);
}

moe_status_t moe_layer_backward_ex(const moe_desc_t* d, const void* x, const void* Wg,
                                   const void* W_gate, const void* W_up, const void* W_down,
                                   const moe_bwd_shared_t* shared, const void* dout,
                                   float aux_grad, void* fwd_ws, size_t fwd_ws_bytes, void* dx,
                                   float* dWg, float* dW_gate, float* dW_up, float* dW_down,
                                   void* bwd_ws, size_t bwd_ws_bytes, int32_t flags,
                                   moe_stream_t stream) {
  moe_status_t st = check_backward(d);
  if (st != MOE_OK) return st;
  const int S = d->n_shared;
  if (S > 0) {
    if (!shared || !shared->Ws_gate || !shared->Ws_up || !shared->Ws_down ||
        !shared->dWs_gate || !shared->dWs_up || !shared->dWs_down)
      return MOE_ERR_INVALID_ARG;
    for (const void* p : {shared->Ws_gate, shared->Ws_up, shared->Ws_down,
                          (const void*)shared->dWs_gate, (const void*)shared->dWs_up,
                          (const void*)shared->dWs_down})
      if (!is_aligned16(p)) return MOE_ERR_INVALID_ARG;
  }
  moe_layer_views_t v;
  st = moe_layer_views(d, fwd_ws, fwd_ws_bytes, &v);
  if (st != MOE_OK) return st;
  const bool glu = d->act == MOE_ACT_SWIGLU;
  if (!x || !Wg || !W_up || !W_down || !dout || !dx || !dWg || !dW_up || !dW_down || !bwd_ws)
    return MOE_ERR_INVALID_ARG;
  if (glu && (!W_gate || !dW_gate)) return MOE_ERR_INVALID_ARG;
  for (const void* p : {x, Wg, W_up, W_down, dout, (const void*)dx, (const void*)dWg,
                        (const void*)dW_up, (const void*)dW_down})
    if (!is_aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (glu && (!is_aligned16(W_gate) || !is_aligned16(dW_gate))) return MOE_ERR_INVALID_ARG;
  if (!(aux_grad == aux_grad)) return MOE_ERR_INVALID_ARG;      // NaN
  if (flags & ~MOE_BWD_PREACT_SAVED) return MOE_ERR_INVALID_ARG;
  BwdViews b;
  if (bwd_ws_bytes < carve_bwd(d, nullptr, &b)) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(bwd_ws) % kAlign) != 0) return MOE_ERR_WORKSPACE;
  carve_bwd(d, static_cast<uint8_t*>(bwd_ws), &b);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d->dtype == MOE_F32)
    return cuda_status(launch_backward_f32(
        *d, v, static_cast<const float*>(x), static_cast<const float*>(Wg),
        static_cast<const float*>(W_gate), static_cast<const float*>(W_up),
        static_cast<const float*>(W_down), shared, static_cast<const float*>(dout), aux_grad,
        static_cast<float*>(dx), dWg, dW_gate, dW_up, dW_down, bwd_ws, s));
  const int T = d->T, D = d->D, E = d->E, F = d->F;
  const int K = d->select == MOE_EXPERT_CHOICE ? E : d->k;
  const int64_t A = v.rows;
  const int nab = (int)b.nab;
  const int Fs = d->F_shared;
  if (T == 0) {
    // no tokens: every gradient is zero
    cudaError_t e = cudaMemsetAsync(dWg, 0, (size_t)E * D * 4, s);
    if (e == cudaSuccess && glu) e = cudaMemsetAsync(dW_gate, 0, (size_t)E * F * D * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dW_up, 0, (size_t)E * F * D * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dW_down, 0, (size_t)E * D * F * 4, s);
    const size_t sb = (size_t)S * Fs * D * 4;
    if (e == cudaSuccess && S) e = cudaMemsetAsync(shared->dWs_gate, 0, sb, s);
    if (e == cudaSuccess && S) e = cudaMemsetAsync(shared->dWs_up, 0, sb, s);
    if (e == cudaSuccess && S) e = cudaMemsetAsync(shared->dWs_down, 0, sb, s);
    return cuda_status(e);
  }
  // the grouped copy of x (a forward with the gathering up projection does not write it)
  cudaError_t e = launch_gather_permuted_rows(*d, v.expert_ids, v.inv, x, v.x_perm, s);
  if (e == cudaSuccess) e = launch_pad_offsets(v.offsets, E, b.pad_off, s);
  // dY = g dout on the executed rows, dg = <dout, y>
  if (e == cudaSuccess)
    e = launch_gather_dy(dout, v.y, v.row_src, v.gates, v.offsets, E, K, D, A, b.dY, b.dgates, s);
  // pre-activations (SwiGLU gate | up blocks, or z = x W_up^T): saved by
  // moe_layer_forward_train, else recomputed
  if (e == cudaSuccess && !(flags & MOE_BWD_PREACT_SAVED))
    e = glu ? launch_grouped_gemm_bf16(EPI_RAW, v.x_perm, A, D, W_gate, W_up, E, F, v.offsets,
                                       b.gu, s)
            : launch_grouped_gemm_bf16(EPI_NONE, v.x_perm, A, D, W_up, nullptr, E, F, v.offsets,
                                       b.gu, s);
  // dH = dY W_down and dX = [da | db] [W_gate ; W_up]: the weights are the right operands
  // in their stored layout ([K, N], MN-major B); MOE_BWD_WEIGHT_TRANSPOSE=1 selects the
  // alternative that first transposes them into K-major copies
  const bool transpose = bwd_weight_transpose();
  if (e == cudaSuccess && transpose) {
    e = launch_transpose(W_down, (int64_t)D * F, D, F, F, b.WdT, (int64_t)F * D, D, 0, E, s);
    if (e == cudaSuccess)
      e = launch_grouped_gemm_bf16(EPI_NONE, b.dY, A, D, b.WdT, nullptr, E, F, v.offsets, b.dH,
                                   s);
  } else if (e == cudaSuccess) {
    e = launch_grouped_gemm_bf16_bmn(b.dY, A, D, W_down, nullptr, D / 64, D, E, F, v.offsets,
                                     b.dH, s);
  }
  // activation backward -> [da | db] (SwiGLU) or dz
  if (e == cudaSuccess)
    e = launch_act_backward(d->act, b.dH, b.gu, b.ldg, v.offsets, E, F, A, b.dAB, s);
  if (e == cudaSuccess && transpose) {
    if (glu)
      e = launch_transpose(W_gate, (int64_t)F * D, F, D, D, b.WguT, (int64_t)D * nab, nab, 0, E,
                           s);
    if (e == cudaSuccess)
      e = launch_transpose(W_up, (int64_t)F * D, F, D, D, b.WguT, (int64_t)D * nab, nab,
                           glu ? F : 0, E, s);
    if (e == cudaSuccess)
      e = launch_grouped_gemm_bf16(EPI_NONE, b.dAB, A, nab, b.WguT, nullptr, E, D, v.offsets,
                                   b.dXp, s);
  } else if (e == cudaSuccess) {
    e = launch_grouped_gemm_bf16_bmn(b.dAB, A, nab, glu ? W_gate : W_up, glu ? W_up : nullptr,
                                     F / 64, F, E, D, v.offsets, b.dXp, s);
  }
  // router: ds, then dx = sum_j dX[inv] + ds W_g and dW_g = ds^T x
  if (e == cudaSuccess)
    e = launch_router_backward(*d, v.logits, v.expert_ids, v.gates, b.dgates, v.inv, v.f,
                               aux_grad, b.ds, s);
  // shared experts: one group of all T tokens each, weight 1, so dY_s = dout; their input
  // gradients dXs[i] go into dx with the routed ones
  if (e == cudaSuccess && S > 0)
    e = shared_backward(d, v, b, x, shared, dout, s);
  if (e == cudaSuccess)
    e = launch_dx(b.dXp, v.inv, b.ds, Wg, T, D, E, K, dx, s, S > 0 ? b.dXs : nullptr, S);
  if (e == cudaSuccess) e = launch_dwg(b.ds, x, T, D, E, b.dwg_part, dWg, s);
  // weight gradients: groups along K over the experts' row blocks, transposed and padded
  const int64_t pc = b.pad_cols;
  if (e == cudaSuccess) e = launch_transpose_pad(b.dY, D, D, v.offsets, b.pad_off, E, pc, b.dYT, pc, s);
  if (e == cudaSuccess) e = launch_transpose_pad(v.h, F, F, v.offsets, b.pad_off, E, pc, b.hT, pc, s);
  if (e == cudaSuccess)
    e = launch_grouped_gemm_kgroups_f32(b.dYT, D, b.hT, F, E, b.pad_off, pc, dW_down, s);
  if (e == cudaSuccess)
    e = launch_transpose_pad(v.x_perm, D, D, v.offsets, b.pad_off, E, pc, b.xpT, pc, s);
  if (e == cudaSuccess)
    e = launch_transpose_pad(b.dAB, nab, nab, v.offsets, b.pad_off, E, pc, b.dABT, pc, s);
  if (e == cudaSuccess && glu)
    e = launch_grouped_gemm_kgroups_f32(b.dABT, F, b.xpT, D, E, b.pad_off, pc, dW_gate, s);
  if (e == cudaSuccess)
    e = launch_grouped_gemm_kgroups_f32(static_cast<const __nv_bfloat16*>(b.dABT) +
                                            (glu ? (int64_t)F * pc : 0),
                                        F, b.xpT, D, E, b.pad_off, pc, dW_up, s);
  return cuda_status(e);
}

int64_t moe_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

moe_status_t moe_debug_inject(int32_t fault) {
  if (fault != 0 && fault != 1) return MOE_ERR_INVALID_ARG;
  set_gemm_fault(fault);
  return MOE_OK;
}

moe_status_t moe_get_device_error(moe_stream_t stream, int32_t* code) {
  int* w = device_error_word();
  if (!w) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (code) *code = v;
  if (v == 0) return MOE_OK;
  return (v >= 0x100 && v < 0x200) ? MOE_ERR_TIMEOUT : MOE_ERR_DEVICE;
}

}  // extern "C"
