// One dense SwiGLU expert on a decode batch (T <= 16 tokens): the always-on
// shared expert when it runs on its own (beside the NVFP4 routed experts).
//
// Qwen3.8-Flash-Next architecture fact sheet: one always-on expert of width
// 640 per MoE layer, SwiGLU, no bias.  f = (silu(x Wg^T) * (x Wu^T)) Wd^T
// with FP32 sums and h rounded to the 16-bit activation type, the same
// function as the grouped GEMMs compute for one group.
//
// A lone expert gives a tile-per-block GEMM only a few blocks, so here the
// weights stream through two GEMV launches spread over the SMs:
//   k_dense_gemv1  grid (I/16 feature slices, 4 K quarters): 32 rows per
//                  block (16 gate + 16 up rows), eight lanes per row with
//                  16-byte chunks, every chunk of the lane's quarter row in
//                  flight at once; FP32 partial dot products to
//                  P[quarter][t][row];
//   k_dense_gemv2  grid H/32: each block first forms h[t][f] =
//                  silu(sum of the gate quarters) * (sum of the up quarters)
//                  in a fixed order, rounded to 16 bits, then streams 32 down
//                  rows against it.
// The expert's rows are offsets[0] .. offsets[1] (at most T), read on the
// device; the fixed-order quarter sums keep results deterministic.
#include "common.cuh"

namespace moe {

constexpr int kDenseGemvMaxT = 16;

namespace {

template <typename T16>
__device__ __forceinline__ T16 from_f32(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

template <typename T16>
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 p = Pack2<T16>::unpack(w[i]);
    f[2 * i] = p.x;
    f[2 * i + 1] = p.y;
  }
}

// gate/up partial sums over K quarter blockIdx.y for the 16 features of slice
// blockIdx.x; xs: the expert's n tokens' quarter rows in shared memory
template <typename T16, int NT>
__global__ void __launch_bounds__(256) k_dense_gemv1(const T16* __restrict__ x, const int32_t* __restrict__ offsets,
                                                     int T, const T16* __restrict__ w_gu, int H, int I,
                                                     float* __restrict__ P) {
  extern __shared__ __align__(16) uint8_t smem[];
  griddep_wait();
  griddep_launch_dependents();
  T16* xs = reinterpret_cast<T16*>(smem);  // [NT][H/4]
  // the expert's rows, clamped to the batch
  const int r0 = max(0, offsets[0]);
  const int n = max(0, min(min(offsets[1] - r0, NT), T - r0));
  const int KQ = H / 4, k_base = blockIdx.y * KQ;
  // stage the tokens' quarter rows (16-byte copies)
  for (int i = threadIdx.x; i < n * (KQ / 8); i += blockDim.x) {
    const int t = i / (KQ / 8), c = i - t * (KQ / 8);
    reinterpret_cast<uint4*>(xs + t * KQ)[c] =
        __ldg(reinterpret_cast<const uint4*>(x + size_t(r0 + t) * H + k_base) + c);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c8 = lane & 7;
  const int r = warp * 4 + (lane >> 3);  // 0..31: gate rows then up rows of the slice
  const int f = blockIdx.x * 16 + (r & 15);
  const int row = r < 16 ? f : I + f;
  const uint4* wr = reinterpret_cast<const uint4*>(w_gu + size_t(row) * H + k_base);
  const int nch = KQ / 64;  // chunks of this lane (8 lanes x 8 elements per step)
  float acc[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t] = 0.f;
  for (int u0 = 0; u0 < nch; u0 += 8) {
    uint4 cw[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) cw[u] = u0 + u < nch ? __ldg(wr + (u0 + u) * 8 + c8) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (u0 + u >= nch) continue;
      float wf[8];
      unpack8<T16>(cw[u], wf);
      const int k = ((u0 + u) * 8 + c8) * 8;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (t < n) {
          float xf[8];
          unpack8<T16>(*reinterpret_cast<const uint4*>(xs + t * KQ + k), xf);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[t] = fmaf(wf[j], xf[j], acc[t]);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float v = acc[t];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    if (c8 == 0 && t < n) P[(size_t(blockIdx.y) * NT + t) * (2 * I) + row] = v;
  }
}

// h from the quarter sums, then 32 down rows (blockIdx.x) against it
template <typename T16, int NT>
__global__ void __launch_bounds__(256) k_dense_gemv2(const float* __restrict__ P, const int32_t* __restrict__ offsets,
                                                     int T, const T16* __restrict__ w_d, int H, int I, int out_fp32,
                                                     void* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem[];
  griddep_wait();
  griddep_launch_dependents();
  T16* hs = reinterpret_cast<T16*>(smem);  // [NT][I]
  // the expert's rows, clamped to the batch
  const int r0 = max(0, offsets[0]);
  const int n = max(0, min(min(offsets[1] - r0, NT), T - r0));
  for (int i = threadIdx.x; i < n * I; i += blockDim.x) {
    const int t = i / I, f = i - t * I;
    float g = 0.f, u = 0.f;
#pragma unroll
    for (int p = 0; p < 4; ++p) {  // quarters in ascending order
      g += P[(size_t(p) * NT + t) * (2 * I) + f];
      u += P[(size_t(p) * NT + t) * (2 * I) + I + f];
    }
    hs[t * I + f] = from_f32<T16>(silu_f(g) * u);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c8 = lane & 7;
  const int o = blockIdx.x * 32 + warp * 4 + (lane >> 3);  // output feature
  const uint4* wr = reinterpret_cast<const uint4*>(w_d + size_t(o) * I);
  const int nch = I / 64;
  float acc[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t] = 0.f;
  for (int u0 = 0; u0 < nch; u0 += 8) {
    uint4 cw[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) cw[u] = u0 + u < nch ? __ldg(wr + (u0 + u) * 8 + c8) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (u0 + u >= nch) continue;
      float wf[8];
      unpack8<T16>(cw[u], wf);
      const int k = ((u0 + u) * 8 + c8) * 8;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (t < n) {
          float hf[8];
          unpack8<T16>(*reinterpret_cast<const uint4*>(hs + t * I + k), hf);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[t] = fmaf(wf[j], hf[j], acc[t]);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float v = acc[t];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    if (c8 == 0 && t < n) {
      const size_t idx = size_t(r0 + t) * H + o;
      if (out_fp32)
        static_cast<float*>(out)[idx] = v;
      else
        static_cast<T16*>(out)[idx] = from_f32<T16>(v);
    }
  }
}

template <typename T16, int NT>
int launch_dense(const void* x, const int32_t* offsets, int T, int H, int I, const void* w_gu, const void* w_d, int out_fp32,
                 void* out, float* P, cudaStream_t stream) {
  const size_t s1 = size_t(NT) * (H / 4) * sizeof(T16), s2 = size_t(NT) * I * sizeof(T16);
  if (s1 > 48 * 1024)
    MOE_CHECK_CUDA(cudaFuncSetAttribute(k_dense_gemv1<T16, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(s1)));
  if (s2 > 48 * 1024)
    MOE_CHECK_CUDA(cudaFuncSetAttribute(k_dense_gemv2<T16, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(s2)));
  // programmatic dependents: launch and block scheduling overlap the kernel before
  MOE_CHECK_CUDA(launch_pdl(k_dense_gemv1<T16, NT>, dim3(I / 16, 4), dim3(256), s1, stream, static_cast<const T16*>(x),
                            offsets, T, static_cast<const T16*>(w_gu), H, I, P));
  MOE_CHECK_CUDA(launch_pdl(k_dense_gemv2<T16, NT>, dim3(H / 32), dim3(256), s2, stream, static_cast<const float*>(P),
                            offsets, T, static_cast<const T16*>(w_d), H, I, out_fp32, out));
  return MOE_OK;
}

template <typename T16>
int dense_dispatch(int T, const void* x, const int32_t* offsets, int H, int I, const void* w_gu, const void* w_d,
                   int out_fp32, void* out, float* P, cudaStream_t stream) {
  if (T <= 1) return launch_dense<T16, 1>(x, offsets, T, H, I, w_gu, w_d, out_fp32, out, P, stream);
  if (T <= 2) return launch_dense<T16, 2>(x, offsets, T, H, I, w_gu, w_d, out_fp32, out, P, stream);
  if (T <= 4) return launch_dense<T16, 4>(x, offsets, T, H, I, w_gu, w_d, out_fp32, out, P, stream);
  if (T <= 8) return launch_dense<T16, 8>(x, offsets, T, H, I, w_gu, w_d, out_fp32, out, P, stream);
  return launch_dense<T16, 16>(x, offsets, T, H, I, w_gu, w_d, out_fp32, out, P, stream);
}

}  // namespace

// Workspace of the small-batch dense path: the FP32 quarter partials
// P [4][NT][2I] (NT = T rounded up to a power of two).
size_t dense_gemv_ws_bytes(int T, int I) {
  int nt = 1;
  while (nt < T) nt <<= 1;
  return size_t(4) * nt * 2 * I * sizeof(float);
}

bool dense_gemv_fits(int T, int H, int I) {
  return T >= 1 && T <= kDenseGemvMaxT && H % 256 == 0 && I % 64 == 0 && H % 32 == 0;
}

int dense_swiglu_gemv(const void* x, const int32_t* offsets, int T, int H, int I, const void* w_gu, const void* w_d,
                      int dtype, int out_fp32, void* out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  MOE_REQUIRE(dense_gemv_fits(T, H, I), MOE_ERR_UNSUPPORTED, "dense small-batch expert: T=%d H=%d I=%d", T, H, I);
  MOE_REQUIRE(ws_bytes >= dense_gemv_ws_bytes(T, I), MOE_ERR_WORKSPACE,
              "dense small-batch expert: workspace of %zu bytes is too small (need %zu)", ws_bytes,
              dense_gemv_ws_bytes(T, I));
  float* P = static_cast<float*>(ws);
  if (dtype == MOE_DTYPE_BF16)
    return dense_dispatch<__nv_bfloat16>(T, x, offsets, H, I, w_gu, w_d, out_fp32, out, P, stream);
  return dense_dispatch<__half>(T, x, offsets, H, I, w_gu, w_d, out_fp32, out, P, stream);
}

}  // namespace moe
