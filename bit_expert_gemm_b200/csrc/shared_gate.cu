// Shared-expert gate: gate[t] = sigmoid(x[t, :] . w_gate), one FP32 scalar
// per token, which moe_combine multiplies into the shared expert's output.
//
// Qwen3.8-Flash-Next-AWQ-g32 card, "Checkpoint": the shared-expert gate is
// one of the non-routed tensors stored next to the router and the shared
// expert.  The card gives no formula; this is the plainest reading (a
// row vector over the hidden size and a logistic gate per token).
//
// One warp per token: 16-byte loads of x and of the gate vector (8 16-bit
// values each, lane-strided), FP32 products summed per lane, then a shuffle
// tree; the logistic function uses the accurate expf and an IEEE division.
// The kernel reads x once: HBM-bound at T*H*2 bytes.
#include "common.cuh"

namespace moe {

namespace {

template <typename T16>
__device__ __forceinline__ float2 to_f2(uint32_t v);
template <>
__device__ __forceinline__ float2 to_f2<__nv_bfloat16>(uint32_t v) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v));
}
template <>
__device__ __forceinline__ float2 to_f2<__half>(uint32_t v) {
  return __half22float2(*reinterpret_cast<__half2*>(&v));
}

template <typename T16>
__global__ void __launch_bounds__(256) k_shared_gate(const T16* __restrict__ x, const T16* __restrict__ wg, int T,
                                                     int H, float* __restrict__ gate) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + size_t(t) * H);
  const uint4* gr = reinterpret_cast<const uint4*>(wg);
  float acc = 0.f;
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 a = __ldg(xr + c), b = __ldg(gr + c);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 p = to_f2<T16>(av[i]), q = to_f2<T16>(bv[i]);
      acc = fmaf(p.x, q.x, acc);
      acc = fmaf(p.y, q.y, acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) gate[t] = 1.0f / (1.0f + expf(-acc));
}

}  // namespace

int shared_gate(const void* x, int T, int H, const void* w_gate, int dtype, float* gate, cudaStream_t stream) {
  if (T == 0) return MOE_OK;
  const dim3 grid((T + 7) / 8);
  if (dtype == MOE_DTYPE_BF16)
    k_shared_gate<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x),
                                                           static_cast<const __nv_bfloat16*>(w_gate), T, H, gate);
  else
    k_shared_gate<__half><<<grid, 256, 0, stream>>>(static_cast<const __half*>(x), static_cast<const __half*>(w_gate),
                                                    T, H, gate);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Pre-MoE RMSNorm with a (1 + w) gain (architecture fact sheet,
// normalisation entries: RMSNorm whose gain is 1 + w, before the block,
// epsilon 1e-6):
//   y[t, h] = x[t, h] / sqrt(mean_h x[t, :]^2 + eps) * (1 + w[h])
// One warp per token: the sum of squares in FP32 over 16-byte pieces
// (lane-strided, then a shuffle tree), the scale with an IEEE square root and
// division, then a second pass over the row (from L1/L2) that scales and
// writes it in 16 bits; every lane rewrites only the pieces it reads, after
// the sum is complete, so y may be x.  With a gate vector (w_gate, not
// null) the second pass also forms the shared-expert gate of the token from
// the 16-bit normalised values it writes: gate[t] = sigmoid(y[t] . w_gate),
// so that the block's input is normalised, and its gate computed, in one
// read of x.
// ---------------------------------------------------------------------------
namespace moe {
namespace {

template <typename T16>
__global__ void __launch_bounds__(256) k_rmsnorm(const T16* x, const T16* __restrict__ w, int T, int H, float eps,
                                                 T16* y, const T16* __restrict__ w_gate, float* __restrict__ gate) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + size_t(t) * H);
  const int nv = H / 8;
  float ss = 0.f;
  for (int c = lane; c < nv; c += 32) {
    const uint4 v = xr[c];
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
  const float r = 1.0f / sqrtf(ss / float(H) + eps);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  const uint4* gr = reinterpret_cast<const uint4*>(w_gate);
  uint4* yr = reinterpret_cast<uint4*>(y + size_t(t) * H);
  float gacc = 0.f;
  for (int c = lane; c < nv; c += 32) {
    const uint4 v = xr[c], g = __ldg(wr + c);
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
    if (lane == 0) gate[t] = 1.0f / (1.0f + expf(-gacc));
  }
}

}  // namespace

int rmsnorm(const void* x, int T, int H, const void* w, float eps, int dtype, void* y, cudaStream_t stream,
            const void* w_gate, float* gate) {
  if (T == 0) return MOE_OK;
  const dim3 grid((T + 7) / 8);
  if (dtype == MOE_DTYPE_BF16)
    k_rmsnorm<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w), T, H, eps,
        static_cast<__nv_bfloat16*>(y), static_cast<const __nv_bfloat16*>(w_gate), gate);
  else
    k_rmsnorm<__half><<<grid, 256, 0, stream>>>(static_cast<const __half*>(x), static_cast<const __half*>(w), T, H,
                                                eps, static_cast<__half*>(y), static_cast<const __half*>(w_gate), gate);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // namespace moe
