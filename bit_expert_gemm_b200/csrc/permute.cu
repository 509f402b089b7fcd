// Deterministic permutation of (token, slot) assignments by expert.
//
// Every token selects an expert at most once, so "ascending token order
// inside an expert" is a property of the set {t : e in S_t}.  The kernels
// build that set as a bitmask per expert (one bit per token), then
//   count[e]        = popcount of the expert's mask          (histogram)
//   offsets         = exclusive scan of count                (scan)
//   row of (t, e)   = offsets[e] + popcount(mask[e] bits < t) (scatter)
// which needs no atomic slot claims and gives the same rows on every run.
#include "common.cuh"

namespace moe {

__global__ void __launch_bounds__(256) k_perm_setbits(const int32_t* __restrict__ idx, int n, int E, int W,
                                                      uint32_t* __restrict__ mask, int ks, int* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int e = idx[i];
  const int t = i / ks;
  if (e < 0 || e >= E) {
    report(status, MOE_ERR_INVALID_ARG);
    return;
  }
  atomicOr(mask + size_t(e) * W + (t >> 5), 1u << (t & 31));
}

// One block per expert: popcount prefix over the expert's words.
__global__ void __launch_bounds__(256) k_perm_expert_scan(const uint32_t* __restrict__ mask, int W,
                                                          int32_t* __restrict__ wordpre, int32_t* __restrict__ count) {
  griddep_wait();  // the mask comes from the kernel before (programmatic dependent launch in route_permute)
  griddep_launch_dependents();
  const int e = blockIdx.x;
  const uint32_t* m = mask + size_t(e) * W;
  int32_t* pre = wordpre + size_t(e) * W;
  const int per = (W + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * per;
  int local = 0;
  for (int w = w0; w < w0 + per && w < W; ++w) local += __popc(m[w]);
  __shared__ int warp_tot[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int i = 0; i < warp; ++i) base += warp_tot[i];
  int run = base + incl - local;
  for (int w = w0; w < w0 + per && w < W; ++w) {
    pre[w] = run;
    run += __popc(m[w]);
  }
  if (threadIdx.x == blockDim.x - 1) count[e] = run;
}

// One block of 1024 threads: exclusive scan of count[0..E) -> offsets[0..E].
__global__ void __launch_bounds__(1024) k_perm_offsets(const int32_t* __restrict__ count, int E,
                                                       int32_t* __restrict__ offsets) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int warp_tot[32];
  const int i = threadIdx.x;
  const int v = i < E ? count[i] : 0;
  const int lane = i & 31, warp = i >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_tot[w];
  if (i < E) offsets[i] = base + incl - v;
  if (i == E - 1) offsets[E] = base + incl;
}

__global__ void __launch_bounds__(256) k_perm_scatter(const int32_t* __restrict__ idx, int n, int ks, int E, int W,
                                                      const uint32_t* __restrict__ mask,
                                                      const int32_t* __restrict__ wordpre,
                                                      const int32_t* __restrict__ offsets,
                                                      int32_t* __restrict__ row_token,
                                                      int32_t* __restrict__ slot_row) {
  griddep_wait();
  griddep_launch_dependents();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int e = idx[i];
  const int t = i / ks;
  if (e < 0 || e >= E) {
    slot_row[i] = -1;
    return;
  }
  const size_t wi = size_t(e) * W + (t >> 5);
  const uint32_t below = mask[wi] & ((1u << (t & 31)) - 1u);
  const int pos = offsets[e] + wordpre[wi] + __popc(below);
  row_token[pos] = t;
  slot_row[i] = pos;
}

// Gathers rows: out[r] = x[row_token[r]] (16-bit rows of H elements); one
// warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) k_gather_rows(const uint4* __restrict__ x, const int32_t* __restrict__ row_token,
                                                     int rows, int chunks, uint4* __restrict__ out) {
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int t = row_token[r];
  const uint4* src = x + size_t(t) * chunks;
  uint4* dst = out + size_t(r) * chunks;
  for (int c = lane; c < chunks; c += 32) dst[c] = __ldg(src + c);
}

size_t permute_ws_bytes(int T, int E) {
  const size_t W = (size_t(T) + 31) / 32;
  WsCounter c;
  c.take<uint32_t>(size_t(E) * W);
  c.take<int32_t>(size_t(E) * W);
  c.take<int32_t>(size_t(E));
  return c.used;
}

int permute(const int32_t* topk_idx, int T, int ks, int E, int32_t* offsets, int32_t* row_token, int32_t* slot_row,
            void* ws, size_t ws_bytes, cudaStream_t stream) {
  const int W = (T + 31) / 32;
  WsCarver carve(ws, ws_bytes);
  uint32_t* mask = carve.take<uint32_t>(size_t(E) * W);
  int32_t* wordpre = carve.take<int32_t>(size_t(E) * W);
  int32_t* count = carve.take<int32_t>(size_t(E));
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_permute: workspace of %zu bytes is too small (need %zu)", ws_bytes,
              permute_ws_bytes(T, E));
  const int n = T * ks;
  int* status = device_status_ptr();
  MOE_CHECK_CUDA(cudaMemsetAsync(mask, 0, size_t(E) * W * sizeof(uint32_t), stream));
  if (n > 0) {
    k_perm_setbits<<<(n + 255) / 256, 256, 0, stream>>>(topk_idx, n, E, W, mask, ks, status);
    MOE_CHECK_CUDA(cudaGetLastError());
  }
  k_perm_expert_scan<<<E, 256, 0, stream>>>(mask, W, wordpre, count);
  MOE_CHECK_CUDA(cudaGetLastError());
  k_perm_offsets<<<1, 1024, 0, stream>>>(count, E, offsets);
  MOE_CHECK_CUDA(cudaGetLastError());
  if (n > 0) {
    k_perm_scatter<<<(n + 255) / 256, 256, 0, stream>>>(topk_idx, n, ks, E, W, mask, wordpre, offsets, row_token,
                                                        slot_row);
    MOE_CHECK_CUDA(cudaGetLastError());
  }
  return MOE_OK;
}

// The permutation from an expert bitmask already built (route_permute: the
// top-k kernel sets the bits): per-expert scan, offsets, scatter, each a
// programmatic dependent of the kernel before.  mask, wordpre [E * W], count [E]
// from the permutation workspace.
int permute_from_mask(const int32_t* topk_idx, int T, int ks, int E, const uint32_t* mask, int32_t* wordpre,
                      int32_t* count, int32_t* offsets, int32_t* row_token, int32_t* slot_row, cudaStream_t stream) {
  const int W = (T + 31) / 32;
  const int n = T * ks;
  MOE_CHECK_CUDA(launch_pdl(k_perm_expert_scan, dim3(E), dim3(256), 0, stream, mask, W, wordpre, count));
  MOE_CHECK_CUDA(launch_pdl(k_perm_offsets, dim3(1), dim3(1024), 0, stream, static_cast<const int32_t*>(count), E,
                            offsets));
  if (n > 0)
    MOE_CHECK_CUDA(launch_pdl(k_perm_scatter, dim3((n + 255) / 256), dim3(256), 0, stream, topk_idx, n, ks, E, W, mask,
                              static_cast<const int32_t*>(wordpre), static_cast<const int32_t*>(offsets), row_token,
                              slot_row));
  return MOE_OK;
}

int gather_rows(const void* x, const int32_t* row_token, int rows, int H, void* out, cudaStream_t stream) {
  if (rows == 0) return MOE_OK;
  const int chunks = H / 8;
  k_gather_rows<<<(rows * 32 + 255) / 256, 256, 0, stream>>>(static_cast<const uint4*>(x), row_token, rows, chunks,
                                                             static_cast<uint4*>(out));
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // namespace moe
