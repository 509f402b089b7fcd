// Router logits, softmax over all experts, top-k and renormalised weights.
//
// Logits: for large T the tcgen05 grouped GEMM (one group, FP32 output with
// the bias added in its epilogue); for small T a warp-per-expert GEMV that
// streams each router row once.  Top-k: one warp per token, each lane holds
// E/32 logits; k+extra rounds of a warp arg-max with ties to the lower index.
// Because softmax is monotone and the selected weights are renormalised over
// the selection, w_j = exp(l_j - l_max) / sum_S exp(l_i - l_max) equals
// softmax(l)_j / sum_S softmax(l)_i, so only the selected logits are needed.
#include <float.h>

#include "common.cuh"
#include "gemm_sm100.cuh"

namespace moe {

template <typename T16>
__global__ void __launch_bounds__(256) k_router_gemv(const T16* __restrict__ x, const T16* __restrict__ wr,
                                                     const float* __restrict__ bias, int T, int H, int E,
                                                     float* __restrict__ logits) {
  const int e = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (e >= E) return;
  const uint4* wrow = reinterpret_cast<const uint4*>(wr + size_t(e) * H);
  const int nchunk = H / 8;
  const float b = bias ? bias[e] : 0.0f;
  for (int t = 0; t < T; ++t) {
    const uint4* xrow = reinterpret_cast<const uint4*>(x + size_t(t) * H);
    float acc = 0.0f;
    for (int c = lane; c < nchunk; c += 32) {
      uint4 wv = __ldg(wrow + c);
      uint4 xv = __ldg(xrow + c);
      const uint32_t* wp = reinterpret_cast<const uint32_t*>(&wv);
      const uint32_t* xp = reinterpret_cast<const uint32_t*>(&xv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 a = Pack2<T16>::unpack(wp[i]);
        float2 bb = Pack2<T16>::unpack(xp[i]);
        acc = fmaf(a.x, bb.x, acc);
        acc = fmaf(a.y, bb.y, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) logits[size_t(t) * E + e] = acc + b;
  }
}

// One warp per token.  NV = values per lane (E <= 32 * NV).
template <int NV>
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ logits, int T, int E, int k, int ks,
                                              int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                              float* __restrict__ topk_logit) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const float* row = logits + size_t(t) * E;
  float v[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    float x = e < E ? row[e] : -FLT_MAX;
    v[i] = (x != x) ? -FLT_MAX : x;  // NaN never wins
  }
  uint32_t removed = 0;  // bit i: value i of this lane already selected (or absent)
#pragma unroll
  for (int i = 0; i < NV; ++i)
    if (lane + 32 * i >= E) removed |= 1u << i;
  float sel_v[16];
  int sel_i[16];
#pragma unroll 1
  for (int r = 0; r < ks; ++r) {
    float bv = -FLT_MAX;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      if (!(removed >> i & 1u) && (v[i] > bv || (v[i] == bv && e < bi))) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) removed |= 1u << (bi >> 5);
    sel_v[r] = bv;
    sel_i[r] = bi;
  }
  // renormalised softmax weights over the k selected experts
  const float m = sel_v[0];
  float z = 0.0f;
  float p[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    p[r] = r < k ? __expf(sel_v[r] - m) : 0.0f;
    z += p[r];
  }
  const float inv = 1.0f / z;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    if (r < ks && lane == r) {
      topk_idx[size_t(t) * ks + r] = sel_i[r];
      if (topk_logit) topk_logit[size_t(t) * ks + r] = sel_v[r];
      if (r < k) topk_w[size_t(t) * k + r] = p[r] * inv;
    }
  }
}

size_t route_ws_bytes(int T, int E) {
  WsCounter c;
  c.take<float>(size_t(T) * E);
  return c.used;
}

int route_topk(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
               int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, void* ws, size_t ws_bytes,
               cudaStream_t stream) {
  WsCarver carve(ws, ws_bytes);
  float* logits = carve.take<float>(size_t(T) * E);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_route_topk: workspace of %zu bytes is too small (need %zu)", ws_bytes,
              route_ws_bytes(T, E));
  const int ks = k + extra;
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
    int rc = launch_grouped_gemm(x, T, w_router, E, a, EPI_STORE, bn, stream);
    if (rc) return rc;
  } else {
    const int blocks = (E * 32 + 255) / 256;
    if (dtype == MOE_DTYPE_BF16)
      k_router_gemv<__nv_bfloat16><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x),
                                                                static_cast<const __nv_bfloat16*>(w_router), bias,
                                                                T, H, E, logits);
    else
      k_router_gemv<__half><<<blocks, 256, 0, stream>>>(static_cast<const __half*>(x),
                                                         static_cast<const __half*>(w_router), bias, T, H, E, logits);
    MOE_CHECK_CUDA(cudaGetLastError());
  }
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

}  // namespace moe
