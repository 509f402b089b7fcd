// Device pieces of routing shared by the standalone router / top-k kernels
// and the fused small-batch route + permute kernel.
//
//   l[t, e] = x[t] . w_router[e] + bias[e]   (FP32 accumulate)
//   S_t     = the k (+ extra) largest l[t, :], ties to the lower expert index
//   w[t, j] = exp(l_j - l_max) / sum_{i in S_t, i < k} exp(l_i - l_max)
//
// softmax is monotone and the selected probabilities are renormalised over
// the selection, so the renormalised softmax weights need only the selected
// logits (the softmax denominator over all E experts cancels).
#pragma once
#include <float.h>

#include "common.cuh"

namespace moe {

constexpr int kRouterEB = 4;  // experts per block of the small-batch logits kernel

// Logits of experts [e0, e0 + kRouterEB) for every token.  The block's weight
// rows are staged in shared memory with cp.async (w_sh: kRouterEB * H 16-bit
// values); warp w then takes tokens w, w + nwarps, ...: its lanes stride over
// H in 8-value chunks, with up to 8 chunks of the token row in flight at
// once, keeping one partial sum per expert, reduced across the warp at the
// end.  Every thread of the block must call this.  X_CG: x was written
// earlier in the same launch by other blocks (read through L2, not the
// read-only path).
template <typename T16, bool X_CG = false>
__device__ void router_block_logits(const T16* __restrict__ x, const T16* __restrict__ wr,
                                    const float* __restrict__ bias, int T, int H, int E, int e0, uint4* w_sh,
                                    float* __restrict__ logits) {
  const int nchunk = H / 8;
  const int ne = min(kRouterEB, E - e0);
  const uint4* src = reinterpret_cast<const uint4*>(wr + size_t(e0) * H);
  for (int i = threadIdx.x; i < ne * nchunk; i += blockDim.x)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(w_sh + i)), "l"(src + i) : "memory");
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  constexpr int U = 8;  // chunks of the token row per lane in flight
  for (int t = warp; t < T; t += nw) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + size_t(t) * H);
    float acc[kRouterEB];
#pragma unroll
    for (int e = 0; e < kRouterEB; ++e) acc[e] = 0.0f;
    for (int c0 = lane; c0 < nchunk; c0 += 32 * U) {
      uint4 xv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        xv[u] = c < nchunk ? (X_CG ? __ldcg(xr + c) : __ldg(xr + c)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        if (c < nchunk) {
          const uint32_t* xp = reinterpret_cast<const uint32_t*>(&xv[u]);
          float2 xf[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) xf[i] = Pack2<T16>::unpack(xp[i]);
#pragma unroll
          for (int e = 0; e < kRouterEB; ++e) {
            if (e < ne) {
              const uint4 wv = w_sh[e * nchunk + c];
              const uint32_t* wp = reinterpret_cast<const uint32_t*>(&wv);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 wf = Pack2<T16>::unpack(wp[i]);
                acc[e] = fmaf(wf.x, xf[i].x, acc[e]);
                acc[e] = fmaf(wf.y, xf[i].y, acc[e]);
              }
            }
          }
        }
      }
    }
    float mine = 0.0f;
#pragma unroll
    for (int e = 0; e < kRouterEB; ++e) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
      if (lane == e) mine = acc[e];
    }
    if (lane < ne) logits[size_t(t) * E + e0 + lane] = mine + (bias ? bias[e0 + lane] : 0.0f);
  }
  __syncthreads();  // w_sh is refilled by the caller's next block
}

// Order-preserving map of a float to an unsigned key (a < b <=> key(a) <
// key(b) for non-NaN values; -0 is made +0 first so that it ties with +0).
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Top-(k + extra) of one token's logits by one warp: each lane holds E/32
// values (NV per lane, E <= 32 * NV) as order keys; each of the ks rounds
// takes the lane's best remaining key, then a warp max of the keys and a warp
// min of the indices holding that max (ties to the lower expert index), two
// redux.sync instructions.  NaN counts as -FLT_MAX; absent and selected
// values have key 0, below every real value.  Lane r keeps the r-th
// selection and writes idx_out[r], logit_out[r] (if not null) and, for r < k,
// the renormalised weight w_out[r].  `row` is read through L2 (it may have
// been written by other blocks of the same kernel).
template <int NV>
__device__ __forceinline__ void topk_token(const float* row, int E, int k, int ks, int lane, int32_t* idx_out,
                                           float* w_out, float* logit_out) {
  uint32_t key[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    float x = e < E ? __ldcg(row + e) : -FLT_MAX;
    x = (x != x) ? -FLT_MAX : x;
    key[i] = e < E ? order_key(x) : 0u;
  }
  uint32_t my_key = 0, top_key = 0;
  int my_i = 0;
#pragma unroll 1
  for (int r = 0; r < ks; ++r) {
    uint32_t bk = 0;
    uint32_t bi = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < NV; ++i)
      if (key[i] > bk) {
        bk = key[i];
        bi = uint32_t(lane + 32 * i);
      }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t win = __reduce_min_sync(0xffffffffu, bk == m ? bi : 0xffffffffu);
#pragma unroll
    for (int i = 0; i < NV; ++i)
      if (uint32_t(lane + 32 * i) == win) key[i] = 0;
    if (lane == r) {
      my_key = m;
      my_i = int(win);
    }
    if (r == 0) top_key = m;
  }
  const float my_v = key_value(my_key), top = key_value(top_key);
  // renormalised softmax over the k selected experts (max-shifted)
  const float p = lane < k ? __expf(my_v - top) : 0.0f;
  float z = p;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (lane < ks) {
    idx_out[lane] = my_i;
    if (logit_out) logit_out[lane] = my_v;
    if (lane < k) w_out[lane] = p * (1.0f / z);
  }
}

}  // namespace moe
