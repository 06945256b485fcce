// Expert parallelism: the exchange plan and the row-block reorder around the All-to-All.
//
// "Top-k 路由（Top-k Routing）" (compassingai), "通訊拓撲：All-to-All": with the experts spread
// over devices, every device sends each token row to the device that holds its expert and gets
// the outputs back, two All-to-All exchanges per layer.  "别只比较 Top-k" (ailearn
// moe-comparison), "两次 All-to-All 是常见 dispatcher 的前向合同": dispatch before the experts,
// combine after them, with the volume set by the rows that leave the device.
//
// Layout.  G ranks; rank r holds the Eg = E / G consecutive experts [r Eg, (r+1) Eg).  After the
// permutation a rank's rows are grouped by expert in ascending expert order, so the rows bound
// for rank r are one contiguous range of that buffer: the send side needs no reordering.  The
// receive buffer is source-major ([source][local expert][rows]); the grouped GEMM wants
// expert-major rows ([local expert][source][rows]), which is the order the single-device layer
// would give the same experts over the ranks' batches laid end to end (rows of an expert by
// ascending token, tokens of rank 0 first).  The plan names the G x Eg row blocks of both
// layouts; moe_ep_reorder moves the blocks one way and, with the roles swapped, back.
#include "common.cuh"

namespace moe {
namespace {

// One CTA column per block (blockIdx.x), its rows strided over blockIdx.y; one warp per row,
// 16-byte vector copies.
__global__ void ep_reorder_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                  int nvec, const int64_t* __restrict__ src_start,
                                  const int64_t* __restrict__ dst_start,
                                  const int64_t* __restrict__ rows) {
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n = rows[b];
  const int64_t s0 = src_start[b], d0 = dst_start[b];
  for (int64_t i = (int64_t)blockIdx.y * (blockDim.x >> 5) + warp; i < n;
       i += (int64_t)gridDim.y * (blockDim.x >> 5)) {
    const uint4* s = src + (s0 + i) * nvec;
    uint4* d = dst + (d0 + i) * nvec;
    for (int v = lane; v < nvec; v += 32) d[v] = __ldg(s + v);
  }
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_ep_plan(int32_t G, int32_t Eg, const int32_t* rows_send,
                                    const int32_t* rows_recv, int64_t* send_rows,
                                    int64_t* send_offsets, int64_t* recv_rows,
                                    int64_t* recv_offsets, int32_t* local_offsets,
                                    int64_t* block_recv, int64_t* block_local,
                                    int64_t* block_rows, int64_t* max_block_rows) {
  if (G < 1 || Eg < 1 || (int64_t)G * Eg > 65536) return MOE_ERR_INVALID_ARG;
  if (!rows_send || !rows_recv || !send_rows || !send_offsets || !recv_rows || !recv_offsets ||
      !local_offsets || !block_recv || !block_local || !block_rows || !max_block_rows)
    return MOE_ERR_INVALID_ARG;
  const int64_t n = (int64_t)G * Eg;
  for (int64_t i = 0; i < n; ++i)
    if (rows_send[i] < 0 || rows_recv[i] < 0) return MOE_ERR_INVALID_ARG;
  // send side: destination r takes this rank's rows of experts [r Eg, (r+1) Eg), in order
  int64_t off = 0;
  for (int r = 0; r < G; ++r) {
    int64_t c = 0;
    for (int e = 0; e < Eg; ++e) c += rows_send[(int64_t)r * Eg + e];
    send_offsets[r] = off;
    send_rows[r] = c;
    off += c;
  }
  // receive side, source-major: source s sends its rows of local experts 0..Eg-1 in order
  off = 0;
  for (int s = 0; s < G; ++s) {
    int64_t c = 0;
    for (int e = 0; e < Eg; ++e) {
      block_recv[(int64_t)s * Eg + e] = off + c;
      c += rows_recv[(int64_t)s * Eg + e];
    }
    recv_offsets[s] = off;
    recv_rows[s] = c;
    off += c;
  }
  const int64_t total = off;
  if (total >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
  // local, expert-major: expert e gathers its blocks from sources 0..G-1 in order
  int64_t loc = 0, mx = 0;
  for (int e = 0; e < Eg; ++e) {
    local_offsets[e] = (int32_t)loc;
    for (int s = 0; s < G; ++s) {
      const int64_t b = (int64_t)s * Eg + e;
      block_local[b] = loc;
      block_rows[b] = rows_recv[b];
      loc += rows_recv[b];
      if (rows_recv[b] > mx) mx = rows_recv[b];
    }
  }
  local_offsets[Eg] = (int32_t)loc;
  *max_block_rows = mx;
  return MOE_OK;
}

extern "C" moe_status_t moe_ep_reorder(const moe_desc_t* d, int32_t n_blocks,
                                       const int64_t* src_start, const int64_t* dst_start,
                                       const int64_t* block_rows, int64_t max_block_rows,
                                       const void* src, void* dst, moe_stream_t stream) {
  if (!d || d->D <= 0 || (d->dtype != MOE_BF16 && d->dtype != MOE_F32)) return MOE_ERR_INVALID_ARG;
  if (n_blocks < 0 || n_blocks > 65535 || max_block_rows < 0) return MOE_ERR_INVALID_ARG;
  if (n_blocks == 0 || max_block_rows == 0) return MOE_OK;
  if (!src_start || !dst_start || !block_rows || !src || !dst) return MOE_ERR_INVALID_ARG;
  const size_t row_bytes = (size_t)d->D * (d->dtype == MOE_BF16 ? 2 : 4);
  if (row_bytes % 16 || !moe::is_aligned16(src) || !moe::is_aligned16(dst))
    return MOE_ERR_UNSUPPORTED;
  const int warps = 8;
  int64_t ys = (max_block_rows + warps - 1) / warps;
  if (ys > 65535) ys = 65535;
  const dim3 grid((unsigned)n_blocks, (unsigned)ys);
  moe::ep_reorder_kernel<<<moe::counted(grid), warps * 32, 0,
                           reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), (int)(row_bytes / 16),
      src_start, dst_start, block_rows);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
