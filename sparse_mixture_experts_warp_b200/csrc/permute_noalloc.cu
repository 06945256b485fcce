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
// The array lives in this library's module: every GPU that loads the library holds its
// MOE_PERMUTE_NOALLOC_MAX_INTS int32 (256 KiB) until the process exits.  Host code cannot use
// the array's name as a device address (in host code it names a host-side stand-in), so the
// first call on each device, with that device current, looks the address up with
// cudaGetSymbolAddress and caches it; later calls on that device reuse it.  Because that first
// call does this set-up, make it before any stream capture.
//
// Every call shares the one array and overwrites what the previous call left there (each
// histogram entry is written before it is read, so no clearing is needed).  Two calls whose
// work overlaps on the GPU -- on different streams, or from different threads -- race on the
// array and give wrong results; serialise them.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

static __device__ __align__(256) int32_t g_permute_scratch[MOE_PERMUTE_NOALLOC_MAX_INTS];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
int32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_permute_scratch on the current device (looked up once per device).
cudaError_t static_scratch(int32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
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
  if (!expert_ids || !x || !x_perm || !counts || !offsets || !row_src || !inv)
    return MOE_ERR_INVALID_ARG;
  if (!moe::is_aligned16(x) || !moe::is_aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (d->select == MOE_TOKEN_CHOICE) {
    const int64_t need = (int64_t)moe::permute_blocks(*d) * d->E;
    if (need > MOE_PERMUTE_NOALLOC_MAX_INTS) return MOE_ERR_UNSUPPORTED;
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
