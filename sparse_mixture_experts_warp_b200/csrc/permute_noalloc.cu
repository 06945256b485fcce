// moe_permute_noalloc: the dispatch permutation for callers that cannot allocate device memory.
//
// Some callers are handed only their input and output buffers and have no way to obtain
// scratch space: a plugin running inside an inference engine or framework whose allocator owns
// all device memory and forbids side allocations, or host code that must not call cudaMalloc
// at that point of its run (cudaMalloc synchronises the device and may fail once memory is
// reserved).  moe_permute needs a small caller-provided scratch buffer (per-block expert
// histograms); this variant keeps that scratch in a fixed, file-scope device array instead and
// allocates nothing.
//
// The array lives in this library's module, held on every GPU where that module is loaded until
// the process exits.  Under lazy module loading (the default of recent CUDA releases) the module,
// and with it the array, is committed to a GPU at the first call there, so make that first call
// before the engine reserves its device memory; if the GPU has no room left then, the call
// returns MOE_ERR_CUDA.
//
// Host code cannot use the array's name as a device address (in host code it names a host-side
// stand-in).  So the first call in each CUDA context, with that context current, looks the
// address up with cudaGetSymbolAddress and caches it under the context's unique id (cuCtxGetId):
// a device reset or a re-created primary context is a new context with a new id, and its first
// call looks the address up again instead of reusing a stale one.  Because that first call does
// this set-up, make it before any stream capture.
//
// Every call shares the one array and overwrites what the previous call left there (each
// histogram entry is written before it is read, so no clearing is needed).  Two calls whose
// work overlaps on the GPU -- on different streams, or from different threads -- race on the
// array and give wrong results; serialise them.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

static __device__ __align__(256) int32_t g_permute_scratch[MOE_PERMUTE_NOALLOC_MAX_INTS];

// The driver's cuCtxGetCurrent / cuCtxGetId, reached through the runtime (the library links
// only the CUDA runtime).  Null when the driver does not provide them: the address is then
// looked up on every call.
typedef CUresult (*ctx_get_current_fn)(CUcontext*);
typedef CUresult (*ctx_get_id_fn)(CUcontext, unsigned long long*);
ctx_get_current_fn g_ctx_get_current = nullptr;
ctx_get_id_fn g_ctx_get_id = nullptr;
std::once_flag g_entry_once;

void resolve_entry_points() {
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_current = reinterpret_cast<ctx_get_current_fn>(f);
  f = nullptr;
  if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_id = reinterpret_cast<ctx_get_id_fn>(f);
}

// Unique id of the current context (false when there is none yet or the driver lacks the call).
bool current_context_id(unsigned long long* id) {
  std::call_once(g_entry_once, resolve_entry_points);
  if (!g_ctx_get_current || !g_ctx_get_id) return false;
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return g_ctx_get_id(ctx, id) == CUDA_SUCCESS;
}

constexpr int kCacheEntries = 64;
struct ScratchEntry {
  unsigned long long ctx_id;
  int32_t* ptr;
};
std::mutex g_scratch_mu;
ScratchEntry g_cache[kCacheEntries] = {};
int g_cache_used = 0;
int g_cache_next = 0;

// Device address of g_permute_scratch in the current context (looked up once per context).
cudaError_t static_scratch(int32_t** out) {
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (have_id) {
    for (int i = 0; i < g_cache_used; ++i)
      if (g_cache[i].ctx_id == id) {
        *out = g_cache[i].ptr;
        return cudaSuccess;
      }
  }
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);   // makes the context current
  if (e != cudaSuccess) return e;
  if (!have_id) have_id = current_context_id(&id);
  if (have_id) {
    int slot = g_cache_used < kCacheEntries ? g_cache_used++ : g_cache_next;
    if (g_cache_used == kCacheEntries) g_cache_next = (slot + 1) % kCacheEntries;
    g_cache[slot] = ScratchEntry{id, static_cast<int32_t*>(p)};
  }
  *out = static_cast<int32_t*>(p);
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_permute_noalloc(const moe_desc_t* d, const int32_t* expert_ids,
                                            const void* x, void* x_perm, int32_t* counts,
                                            int32_t* offsets, int32_t* row_src, int32_t* inv,
                                            moe_stream_t stream) {
  int64_t rows = 0;
  moe_status_t st = moe_rows_max(d, &rows);          // validates the descriptor
  if (st != MOE_OK) return st;
  // the size limit first: an oversized problem is refused whatever pointers it came with
  if (d->select == MOE_TOKEN_CHOICE &&
      (int64_t)moe::permute_blocks(*d) * d->E > MOE_PERMUTE_NOALLOC_MAX_INTS)
    return MOE_ERR_UNSUPPORTED;
  if (!expert_ids || !x || !x_perm || !counts || !offsets || !row_src || !inv)
    return MOE_ERR_INVALID_ARG;
  if (!moe::is_aligned16(x) || !moe::is_aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (d->select == MOE_TOKEN_CHOICE) {
    int32_t cap = 0;
    st = moe_capacity(d, &cap);
    if (st != MOE_OK) return st;
    int32_t* hist = nullptr;
    e = moe::static_scratch(&hist);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = moe::launch_permute_token_choice(*d, expert_ids, x, x_perm, counts, offsets, row_src,
                                         inv, hist, cap, s);
  } else {
    // expert choice needs no scratch
    e = moe::launch_permute_expert_choice(*d, expert_ids, x, x_perm, counts, offsets, row_src,
                                          inv, s);
  }
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
