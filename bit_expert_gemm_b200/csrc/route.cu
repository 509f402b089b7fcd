// Router logits, softmax over all experts, top-k and renormalised weights.
//
// Logits: for large T the tcgen05 grouped GEMM (one group, FP32 output with
// the bias added in its epilogue); for small T a CUDA-core kernel in which
// each block stages a few router rows in shared memory and its warps take the
// tokens, so every router row is read from HBM once.  Top-k: one warp per
// token (route.cuh).
#include "common.cuh"
#include "gemm_sm100.cuh"
#include "route.cuh"

namespace moe {

template <typename T16>
__global__ void __launch_bounds__(256) k_router_small(const T16* __restrict__ x, const T16* __restrict__ wr,
                                                      const float* __restrict__ bias, int T, int H, int E,
                                                      float* __restrict__ logits) {
  extern __shared__ __align__(16) uint8_t route_smem[];
  router_block_logits<T16>(x, wr, bias, T, H, E, blockIdx.x * kRouterEB, reinterpret_cast<uint4*>(route_smem),
                           logits);
}

// One warp per token.  NV = values per lane (E <= 32 * NV).
template <int NV>
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ logits, int T, int E, int k, int ks,
                                              int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                              float* __restrict__ topk_logit) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  topk_token<NV>(logits + size_t(t) * E, E, k, ks, threadIdx.x & 31, topk_idx + size_t(t) * ks,
                 topk_w + size_t(t) * k, topk_logit ? topk_logit + size_t(t) * ks : nullptr);
}

// k_topk that also sets the permutation's expert bitmask (one bit per
// (expert, token), mask [E][W] zeroed beforehand): lane j of token t marks
// its selection.  Launched as a programmatic dependent of the router GEMM.
template <int NV>
__global__ void __launch_bounds__(256) k_topk_bits(const float* __restrict__ logits, int T, int E, int k, int ks,
                                                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                                   float* __restrict__ topk_logit, uint32_t* __restrict__ mask, int W,
                                                   int* status) {
  griddep_wait();
  griddep_launch_dependents();
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  topk_token<NV>(logits + size_t(t) * E, E, k, ks, lane, topk_idx + size_t(t) * ks, topk_w + size_t(t) * k,
                 topk_logit ? topk_logit + size_t(t) * ks : nullptr);
  if (lane < ks) {
    const int e = topk_idx[size_t(t) * ks + lane];  // this lane's own selection, written just above
    if (e >= 0 && e < E) atomicOr(mask + size_t(e) * W + (t >> 5), 1u << (t & 31));
    else report(status, MOE_ERR_INVALID_ARG);
  }
}

size_t route_ws_bytes(int T, int E) {
  WsCounter c;
  c.take<float>(size_t(T) * E);
  return c.used;
}

// logits [T, E] FP32 = x w_router^T + bias: the tcgen05 GEMM for T >= 256
// (E % 64 == 0), else k_router_small.
static int router_logits(const void* x, int T, int H, const void* w_router, const float* bias, int E, int dtype,
                         float* logits, cudaStream_t stream) {
  const bool use_tc = T >= 256 && E % 64 == 0;
  if (use_tc) {
    GemmArgs a{};
    a.group_offsets = nullptr;
    a.G = 1;
    a.rows = T;
    a.K = H;
    a.n_out = E;
    a.b_rows_per_group = E;
    a.up_offset = 0;
    a.out = logits;
    a.ldo = E;
    a.out_fp32 = 1;
    a.bias = bias;
    a.bf16 = dtype == MOE_DTYPE_BF16;
    a.status = device_status_ptr();
    a.limit_ns = wait_limit_ns();
    const int bn = E % 256 == 0 ? 256 : (E % 128 == 0 ? 128 : 64);
    return launch_grouped_gemm(x, T, w_router, E, a, EPI_STORE, bn, stream);
  }
  const int blocks = (E + kRouterEB - 1) / kRouterEB;
  const size_t smem = size_t(kRouterEB) * H * 2;
  if (dtype == MOE_DTYPE_BF16) {
    if (smem > 48 * 1024)
      MOE_CHECK_CUDA(cudaFuncSetAttribute(k_router_small<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          int(smem)));
    k_router_small<__nv_bfloat16><<<blocks, 256, smem, stream>>>(static_cast<const __nv_bfloat16*>(x),
                                                                 static_cast<const __nv_bfloat16*>(w_router), bias, T,
                                                                 H, E, logits);
  } else {
    if (smem > 48 * 1024)
      MOE_CHECK_CUDA(cudaFuncSetAttribute(k_router_small<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          int(smem)));
    k_router_small<__half><<<blocks, 256, smem, stream>>>(static_cast<const __half*>(x),
                                                          static_cast<const __half*>(w_router), bias, T, H, E, logits);
  }
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

int route_topk(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
               int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, void* ws, size_t ws_bytes,
               cudaStream_t stream) {
  WsCarver carve(ws, ws_bytes);
  float* logits = carve.take<float>(size_t(T) * E);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_route_topk: workspace of %zu bytes is too small (need %zu)", ws_bytes,
              route_ws_bytes(T, E));
  const int ks = k + extra;
  int rc = router_logits(x, T, H, w_router, bias, E, dtype, logits, stream);
  if (rc) return rc;
  const int blocks = (T * 32 + 255) / 256;
  const int nv = (E + 31) / 32;
#define MOE_TOPK(NV) \
  k_topk<NV><<<blocks, 256, 0, stream>>>(logits, T, E, k, ks, topk_idx, topk_w, topk_logit)
  if (nv <= 1) MOE_TOPK(1);
  else if (nv <= 2) MOE_TOPK(2);
  else if (nv <= 4) MOE_TOPK(4);
  else if (nv <= 8) MOE_TOPK(8);
  else if (nv <= 16) MOE_TOPK(16);
  else MOE_TOPK(32);
#undef MOE_TOPK
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

// route_topk whose top-k kernel also sets the permutation's expert bitmask
// (mask [E][W], W = ceil(T / 32) words, zeroed here before the router runs).
int route_topk_bits(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
                    int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, void* ws, size_t ws_bytes,
                    uint32_t* mask, cudaStream_t stream) {
  WsCarver carve(ws, ws_bytes);
  float* logits = carve.take<float>(size_t(T) * E);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_route_permute: workspace of %zu bytes is too small", ws_bytes);
  const int ks = k + extra;
  const int W = (T + 31) / 32;
  MOE_CHECK_CUDA(cudaMemsetAsync(mask, 0, size_t(E) * W * sizeof(uint32_t), stream));
  int rc = router_logits(x, T, H, w_router, bias, E, dtype, logits, stream);
  if (rc) return rc;
  const dim3 grid((T * 32 + 255) / 256);
  const int nv = (E + 31) / 32;
  int* status = device_status_ptr();
#define MOE_TOPKB(NV)                                                                                                 \
  MOE_CHECK_CUDA(launch_pdl(k_topk_bits<NV>, grid, dim3(256), 0, stream, static_cast<const float*>(logits), T, E, k, \
                            ks, topk_idx, topk_w, topk_logit, mask, W, status))
  if (nv <= 1) MOE_TOPKB(1);
  else if (nv <= 2) MOE_TOPKB(2);
  else if (nv <= 4) MOE_TOPKB(4);
  else if (nv <= 8) MOE_TOPKB(8);
  else if (nv <= 16) MOE_TOPKB(16);
  else MOE_TOPKB(32);
#undef MOE_TOPKB
  return MOE_OK;
}

}  // namespace moe
