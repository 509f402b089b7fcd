// Expert parallelism: the device-side bookkeeping of a dispatch / combine
// between W ranks that each hold E / W of the routed experts.
//
// Qwen3.8-Flash-Next-RAZOR-96B-A6B-NVFP4 card, serving example: the model is
// served with tensor parallelism and expert parallelism over eight GPUs.  The
// forward is unchanged; only where an expert's rows are computed moves.  Rank
// d owns experts [d * E/W, (d+1) * E/W).  After the permutation a rank's
// rows are grouped by expert in ascending order, so they are already grouped
// by destination rank: rank d receives rows offsets[d E/W] ..
// offsets[(d+1) E/W] - 1.  moe_ep_plan gives each row the local index of its
// expert at the destination and counts the rows per destination;
// moe_gather_rows moves whole 16-bit rows by an index (x rows into the send
// order, and the experts' outputs back into the received order).
#include "common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) k_ep_plan(const int32_t* __restrict__ offsets, int E, int W, int rows,
                                                 int32_t* __restrict__ row_local_expert, int32_t* __restrict__ send_counts) {
  const int El = E / W;
  if (blockIdx.x == 0)
    for (int d = threadIdx.x; d < W; d += blockDim.x) send_counts[d] = offsets[(d + 1) * El] - offsets[d * El];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows) return;
  // the expert of permuted row i: the last e with offsets[e] <= i (empty
  // experts share their offset with the next expert)
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= i) lo = mid; else hi = mid - 1;
  }
  row_local_expert[i] = lo - (lo / El) * El;
}

// out[r] = src[index[r]] for 16-byte pieces of whole rows; an index outside
// [0, src_rows) writes a zero row and is recorded in the status word.
__global__ void __launch_bounds__(256) k_gather_rows_checked(const uint4* __restrict__ src, int src_rows,
                                                             const int32_t* __restrict__ index, int rows, int chunks,
                                                             uint4* __restrict__ out, int* status) {
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int t = index[r];
  uint4* dst = out + size_t(r) * chunks;
  if (t < 0 || t >= src_rows) {
    if (lane == 0) report(status, MOE_ERR_INVALID_ARG);
    for (int c = lane; c < chunks; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* s = src + size_t(t) * chunks;
  for (int c = lane; c < chunks; c += 32) dst[c] = __ldg(s + c);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_ep_plan(const int32_t* expert_offsets, int E, int world, int rows, int32_t* row_local_expert,
                           int32_t* send_counts, void* stream) {
  MOE_REQUIRE(E >= 1 && world >= 1 && E % world == 0, MOE_ERR_UNSUPPORTED,
              "moe_ep_plan: E=%d must be a positive multiple of world=%d", E, world);
  MOE_REQUIRE(rows >= 0, MOE_ERR_INVALID_ARG, "moe_ep_plan: rows=%d", rows);
  MOE_REQUIRE(expert_offsets && send_counts && (rows == 0 || row_local_expert), MOE_ERR_INVALID_ARG,
              "moe_ep_plan: null pointer");
  const int blocks = rows > 0 ? (rows + 255) / 256 : 1;
  k_ep_plan<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(expert_offsets, E, world, rows, row_local_expert,
                                                                  send_counts);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

extern "C" int moe_gather_rows(const void* src, int src_rows, int H, const int32_t* index, int rows, void* out,
                               void* stream) {
  MOE_REQUIRE(src_rows >= 0 && rows >= 0 && H > 0 && H % 8 == 0, MOE_ERR_UNSUPPORTED,
              "moe_gather_rows: need rows >= 0 and H %% 8 == 0 (H=%d)", H);
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(src && index && out, MOE_ERR_INVALID_ARG, "moe_gather_rows: null pointer");
  MOE_REQUIRE(aligned16(src) && aligned16(out), MOE_ERR_INVALID_ARG, "moe_gather_rows: rows not 16-byte aligned");
  k_gather_rows_checked<<<(rows * 32 + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), src_rows, index, rows, H / 8, static_cast<uint4*>(out), device_status_ptr());
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}
