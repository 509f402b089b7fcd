// Routing and permutation of a small batch (T <= 128 tokens, decode) in one
// cooperative kernel, instead of the router, top-k and four permutation
// launches that a large batch takes.  Three phases separated by grid-wide
// barriers:
//   1. logits: every block computes kRouterEB experts' logits for all tokens
//      (router rows read from HBM once);
//   2. top-k and renormalised weights: one warp per token (all in block 0
//      when T <= 8, which then needs no second grid barrier);
//   3. permutation, by block 0 alone: each expert's tokens as a bitmask in
//      shared memory (T <= 128: at most four words per expert), counts by
//      popcount, exclusive scan into expert_offsets, and every assignment's
//      row = offset + popcount of the expert's bits below its token.  Same
//      order as the standalone permutation: experts ascending, tokens
//      ascending inside an expert.
// With a pre-MoE RMSNorm (norm_w not null) a phase 0 comes first: block b
// normalises tokens b, b + grid, ... into x_norm (16-bit, the block's input
// activation: x / sqrt(mean x^2 + eps) * (1 + w)) and, with a gate vector,
// forms the shared-expert gate sigmoid(x_norm . w_gate) from the values it
// wrote; a grid barrier follows and the logits read x_norm.
// Values written by other blocks of this launch are read with ld.global.cg
// (through L2) after the grid barrier.
#include <cooperative_groups.h>

#include "common.cuh"
#include "route.cuh"

namespace cg = cooperative_groups;

namespace moe {

size_t route_ws_bytes(int T, int E);
size_t permute_ws_bytes(int T, int E);
int route_topk(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
               int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, void* ws, size_t ws_bytes,
               cudaStream_t stream);
int route_topk_bits(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
                    int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, void* ws, size_t ws_bytes,
                    uint32_t* mask, cudaStream_t stream);
int permute_from_mask(const int32_t* topk_idx, int T, int ks, int E, const uint32_t* mask, int32_t* wordpre,
                      int32_t* count, int32_t* offsets, int32_t* row_token, int32_t* slot_row, cudaStream_t stream);
int permute(const int32_t* topk_idx, int T, int ks, int E, int32_t* offsets, int32_t* row_token, int32_t* slot_row,
            void* ws, size_t ws_bytes, cudaStream_t stream);

constexpr int kRouteSmallMaxT = 128;

namespace {

constexpr int kThreads = 256;

struct RouteSmallArgs {
  const void* x;
  const void* wr;
  const float* bias;
  int T, H, E, k, ks;
  float* logits;  // [T, E] scratch
  int32_t* topk_idx;
  float* topk_w;
  float* topk_logit;
  int32_t* offsets;
  int32_t* row_token;
  int32_t* slot_row;
  int* status;
  // optional pre-MoE RMSNorm (phase 0) and shared-expert gate
  const void* norm_w;
  float eps;
  const void* gate_w;
  void* x_norm;
  float* gate;
};

// Phase 0 for token t, by the whole block: the sum of squares in FP32 (each
// thread over 16-byte pieces, a shuffle tree per warp, then the warps' sums
// in order), y = x * r * (1 + w) rounded to 16 bits, and the gate from the
// rounded y.
template <typename T16>
__device__ void norm_token(const T16* __restrict__ x, const T16* __restrict__ w, const T16* __restrict__ wg, int t,
                           int H, float eps, T16* __restrict__ y, float* __restrict__ gate, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const uint4* xr = reinterpret_cast<const uint4*>(x + size_t(t) * H);
  const int nv = H / 8;
  float ss = 0.f;
  for (int c = threadIdx.x; c < nv; c += blockDim.x) {
    const uint4 v = __ldg(xr + c);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = Pack2<T16>::unpack(u[j]);
      ss = fmaf(f.x, f.x, ss);
      ss = fmaf(f.y, f.y, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < nw; ++i) tot += red[i];
  const float r = 1.0f / sqrtf(tot / float(H) + eps);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  const uint4* gr = reinterpret_cast<const uint4*>(wg);
  uint4* yr = reinterpret_cast<uint4*>(y + size_t(t) * H);
  float gacc = 0.f;
  for (int c = threadIdx.x; c < nv; c += blockDim.x) {
    const uint4 v = __ldg(xr + c), g = __ldg(wr + c);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w}, gw[4] = {g.x, g.y, g.z, g.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = Pack2<T16>::unpack(u[j]), gg = Pack2<T16>::unpack(gw[j]);
      o[j] = Pack2<T16>::pack(f.x * r * (1.0f + gg.x), f.y * r * (1.0f + gg.y));
    }
    yr[c] = make_uint4(o[0], o[1], o[2], o[3]);
    if (gate) {
      const uint4 q = __ldg(gr + c);
      const uint32_t qv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 a = Pack2<T16>::unpack(o[j]), b = Pack2<T16>::unpack(qv[j]);
        gacc = fmaf(a.x, b.x, gacc);
        gacc = fmaf(a.y, b.y, gacc);
      }
    }
  }
  if (gate) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gacc += __shfl_xor_sync(0xffffffffu, gacc, o);
    __syncthreads();  // every warp has read red[] above
    if (lane == 0) red[warp] = gacc;
    __syncthreads();
    if (threadIdx.x == 0) {
      float g = 0.f;
      for (int i = 0; i < nw; ++i) g += red[i];
      gate[t] = 1.0f / (1.0f + expf(-g));
    }
  }
  __syncthreads();  // red[] is reused by the block's next token
}

template <typename T16, int NV>
__global__ void __launch_bounds__(kThreads, 1) k_route_permute_small(const RouteSmallArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  cg::grid_group grid = cg::this_grid();
  // launched after its inputs are complete: a programmatic dependent may start its prologue now
  griddep_launch_dependents();
  const int E = a.E, T = a.T, ks = a.ks;
  // 0. pre-MoE RMSNorm (and the shared-expert gate) into x_norm
  if (a.norm_w) {
    __shared__ float red[kThreads / 32];
    for (int t = blockIdx.x; t < T; t += gridDim.x)
      norm_token<T16>(static_cast<const T16*>(a.x), static_cast<const T16*>(a.norm_w),
                      static_cast<const T16*>(a.gate_w), t, a.H, a.eps, static_cast<T16*>(a.x_norm), a.gate, red);
    grid.sync();
  }
  // 1. logits (of x_norm when phase 0 ran: rows other blocks wrote, read through L2)
  for (int eb = blockIdx.x; eb * kRouterEB < E; eb += gridDim.x) {
    if (a.norm_w)
      router_block_logits<T16, true>(static_cast<const T16*>(a.x_norm), static_cast<const T16*>(a.wr), a.bias, T, a.H,
                                     E, eb * kRouterEB, reinterpret_cast<uint4*>(smem), a.logits);
    else
      router_block_logits<T16>(static_cast<const T16*>(a.x), static_cast<const T16*>(a.wr), a.bias, T, a.H, E,
                               eb * kRouterEB, reinterpret_cast<uint4*>(smem), a.logits);
  }
  grid.sync();
  // 2. top-k: by block 0 alone when every token has a warp of its own there
  // (then the permutation follows after a block barrier), else by all blocks
  // with a second grid barrier
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool solo = T <= kThreads / 32;
  if (solo && blockIdx.x != 0) return;
  const int t_first = solo ? warp : blockIdx.x * (kThreads / 32) + warp;
  const int t_step = solo ? kThreads / 32 : gridDim.x * (kThreads / 32);
  for (int t = t_first; t < T; t += t_step)
    topk_token<NV>(a.logits + size_t(t) * E, E, a.k, ks, lane, a.topk_idx + size_t(t) * ks,
                   a.topk_w + size_t(t) * a.k, a.topk_logit ? a.topk_logit + size_t(t) * ks : nullptr);
  if (solo) {
    __syncthreads();
  } else {
    grid.sync();
    if (blockIdx.x != 0) return;
  }
  // 3. permutation (block 0)
  const int W = (T + 31) / 32;
  uint32_t* mask = reinterpret_cast<uint32_t*>(smem);  // [E, W]
  int* off = reinterpret_cast<int*>(mask + E * W);     // [E + 1]
  __shared__ int warp_tot[kThreads / 32];
  for (int i = threadIdx.x; i < E * W; i += kThreads) mask[i] = 0;
  __syncthreads();
  const int n = T * ks;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const int e = __ldcg(a.topk_idx + i);
    const int t = i / ks;
    if (e < 0 || e >= E) {
      report(a.status, MOE_ERR_INVALID_ARG);
      continue;
    }
    atomicOr(mask + e * W + (t >> 5), 1u << (t & 31));
  }
  __syncthreads();
  // exclusive scan of the counts; thread i owns experts 4i .. 4i+3 (E <= 1024)
  int cnt[4], local = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = threadIdx.x * 4 + j;
    cnt[j] = 0;
    if (e < E)
      for (int w = 0; w < W; ++w) cnt[j] += __popc(mask[e * W + w]);
    local += cnt[j];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int run = incl - local;
  for (int w = 0; w < warp; ++w) run += warp_tot[w];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = threadIdx.x * 4 + j;
    if (e < E) {
      off[e] = run;
      a.offsets[e] = run;
    }
    run += cnt[j];
  }
  if (threadIdx.x == kThreads - 1) {
    off[E] = run;
    a.offsets[E] = run;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const int e = __ldcg(a.topk_idx + i);
    const int t = i / ks;
    if (e < 0 || e >= E) {
      a.slot_row[i] = -1;
      continue;
    }
    const uint32_t* m = mask + e * W;
    int rank = __popc(m[t >> 5] & ((1u << (t & 31)) - 1u));
    for (int w = 0; w < (t >> 5); ++w) rank += __popc(m[w]);
    const int pos = off[e] + rank;
    a.row_token[pos] = t;
    a.slot_row[i] = pos;
  }
}

template <typename T16, int NV>
int launch_small(const RouteSmallArgs& a, size_t smem, cudaStream_t stream) {
  auto kern = k_route_permute_small<T16, NV>;
  constexpr int kMaxDev = 64;
  static int co_resident[kMaxDev] = {0};
  static size_t smem_set[kMaxDev] = {0};
  int dev = 0;
  MOE_CHECK_CUDA(cudaGetDevice(&dev));
  MOE_REQUIRE(dev < kMaxDev, MOE_ERR_UNSUPPORTED, "moe_route_permute: device %d >= %d", dev, kMaxDev);
  if (smem > smem_set[dev] || co_resident[dev] == 0) {
    if (smem > 48 * 1024)
      MOE_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    int per_sm = 0;
    MOE_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem));
    MOE_REQUIRE(per_sm > 0, MOE_ERR_UNSUPPORTED, "moe_route_permute: kernel does not fit on an SM");
    co_resident[dev] = per_sm * num_sms();
    smem_set[dev] = smem;
  }
  const int want = (a.E + kRouterEB - 1) / kRouterEB;
  const int grid = want < co_resident[dev] ? want : co_resident[dev];
  void* params[] = {const_cast<RouteSmallArgs*>(&a)};
  MOE_CHECK_CUDA(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(kThreads), params,
                                             smem, stream));
  return MOE_OK;
}

template <typename T16>
int dispatch_small(const RouteSmallArgs& a, size_t smem, cudaStream_t stream) {
  const int nv = (a.E + 31) / 32;
  if (nv <= 4) return launch_small<T16, 4>(a, smem, stream);
  if (nv <= 8) return launch_small<T16, 8>(a, smem, stream);
  if (nv <= 16) return launch_small<T16, 16>(a, smem, stream);
  return launch_small<T16, 32>(a, smem, stream);
}

}  // namespace

size_t route_permute_ws_bytes(int T, int E) {
  if (T <= kRouteSmallMaxT) return route_ws_bytes(T, E);
  WsCounter c;
  c.take<uint8_t>(route_ws_bytes(T, E));
  c.take<uint8_t>(permute_ws_bytes(T, E));
  return c.used;
}

int rmsnorm(const void* x, int T, int H, const void* w, float eps, int dtype, void* y, cudaStream_t stream,
            const void* w_gate, float* gate);

// norm (optional): the pre-MoE RMSNorm of x into norm->x_norm (and the gate)
// before the routing, which then reads x_norm.
int route_permute(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
                  int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, int32_t* offsets,
                  int32_t* row_token, int32_t* slot_row, void* ws, size_t ws_bytes, cudaStream_t stream,
                  const RouteNorm* norm) {
  const int ks = k + extra;
  if (norm && T > kRouteSmallMaxT) {
    // the norm kernel (one read of x; the gate from its output), then the
    // large-batch routing of x_norm
    const int rc = rmsnorm(x, T, H, norm->w, norm->eps, dtype, norm->x_norm, stream, norm->gate_w, norm->gate);
    if (rc) return rc;
    x = norm->x_norm;
  }
  if (T > kRouteSmallMaxT) {
    WsCarver carve(ws, ws_bytes);
    void* ws_r = carve.take<uint8_t>(route_ws_bytes(T, E));
    void* ws_p = carve.take<uint8_t>(permute_ws_bytes(T, E));
    MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_route_permute: workspace of %zu bytes is too small", ws_bytes);
    // router GEMM, top-k setting the expert bitmask as it selects, then the
    // per-expert scan, offsets and scatter as programmatic dependents
    WsCarver pc(ws_p, permute_ws_bytes(T, E));
    const int W = (T + 31) / 32;
    uint32_t* mask = pc.take<uint32_t>(size_t(E) * W);
    int32_t* wordpre = pc.take<int32_t>(size_t(E) * W);
    int32_t* count = pc.take<int32_t>(size_t(E));
    int rc = route_topk_bits(x, T, H, w_router, bias, E, k, extra, dtype, topk_idx, topk_w, topk_logit, ws_r,
                             route_ws_bytes(T, E), mask, stream);
    if (rc) return rc;
    return permute_from_mask(topk_idx, T, ks, E, mask, wordpre, count, offsets, row_token, slot_row, stream);
  }
  WsCarver carve(ws, ws_bytes);
  float* logits = carve.take<float>(size_t(T) * E);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_route_permute: workspace of %zu bytes is too small", ws_bytes);
  RouteSmallArgs a{};
  a.x = x;
  a.wr = w_router;
  a.bias = bias;
  a.T = T;
  a.H = H;
  a.E = E;
  a.k = k;
  a.ks = ks;
  a.logits = logits;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.topk_logit = topk_logit;
  a.offsets = offsets;
  a.row_token = row_token;
  a.slot_row = slot_row;
  a.status = device_status_ptr();
  if (norm) {
    a.norm_w = norm->w;
    a.eps = norm->eps;
    a.gate_w = norm->gate_w;
    a.x_norm = norm->x_norm;
    a.gate = norm->gate;
  }
  const size_t w_bytes = size_t(kRouterEB) * H * 2;
  const size_t p_bytes = (size_t(E) * ((T + 31) / 32) + E + 1) * 4;
  const size_t smem = w_bytes > p_bytes ? w_bytes : p_bytes;
  MOE_REQUIRE(smem <= 200 * 1024, MOE_ERR_UNSUPPORTED, "moe_route_permute: H=%d too large for the small-batch path",
              H);
  return dtype == MOE_DTYPE_BF16 ? dispatch_small<__nv_bfloat16>(a, smem, stream)
                                 : dispatch_small<__half>(a, smem, stream);
}

}  // namespace moe
