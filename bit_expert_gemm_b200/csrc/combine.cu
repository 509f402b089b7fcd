// Weighted combine, Refill-RMS accumulation (fused with the combine of the
// (k+1)-slot pass) and Refill-RMS expert selection.  These are HBM-bound
// streaming kernels: every byte of f is read once with 16-byte vector loads.
#include <float.h>

#include <algorithm>

#include "common.cuh"

namespace moe {

// Loads 4 consecutive values of row `r` starting at column c as FP32.
template <typename T16, bool F32>
__device__ __forceinline__ void load4(const void* f, size_t r, int H, int c, float (&v)[4]) {
  if (F32) {
    float4 q = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(f) + r * H + c));
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  } else {
    uint2 q = __ldg(reinterpret_cast<const uint2*>(static_cast<const T16*>(f) + r * H + c));
    float2 a = Pack2<T16>::unpack(q.x), b = Pack2<T16>::unpack(q.y);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
}

// Loads 8 consecutive values of row `r` starting at column c as FP32 (one or
// two 16-byte loads).
template <typename T16, bool F32>
__device__ __forceinline__ void load8(const void* f, size_t r, int H, int c, float (&v)[8]) {
  if (F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(f) + r * H + c);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(static_cast<const T16*>(f) + r * H + c));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 u = Pack2<T16>::unpack(w[i]);
      v[2 * i] = u.x;
      v[2 * i + 1] = u.y;
    }
  }
}

template <typename T16>
__device__ __forceinline__ void store4(T16* y, size_t r, int H, int c, const float (&v)[4]) {
  uint2 q;
  q.x = Pack2<T16>::pack(v[0], v[1]);
  q.y = Pack2<T16>::pack(v[2], v[3]);
  *reinterpret_cast<uint2*>(y + r * H + c) = q;
}

// y[t] = sum_j w[t,j] f[slot_row[t,j]] (+ gate[t] * shared[t]).  Each thread
// owns 8 consecutive columns (16-byte loads of 16-bit f); a block of 256
// threads covers 2048 columns of a row and walks tokens t = blockIdx.x,
// blockIdx.x + gridDim.x, ... (grid (min(T, 8 x SMs), ceil(H/2048))).  The
// KM (>= k) row loads of a token are all issued before the first is used, so
// that they are in flight together; the sum then runs in slot order.
template <typename T16, bool F32, int KM>
__global__ void __launch_bounds__(256) k_combine(const void* __restrict__ f, const int32_t* __restrict__ slot_row,
                                                 int ks, const float* __restrict__ w, const T16* __restrict__ shared,
                                                 const float* __restrict__ gate, int k, int H, int T,
                                                 T16* __restrict__ y) {
  constexpr int NV = F32 ? 2 : 1;  // 16-byte vectors per row and thread
  griddep_wait();  // f comes from the kernel just before (programmatic dependent launch)
  griddep_launch_dependents();
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (c >= H) return;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    int r[KM];
    float wj[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      r[j] = j < k ? __ldg(slot_row + size_t(t) * ks + j) : -1;
      wj[j] = j < k ? __ldg(w + size_t(t) * k + j) : 0.0f;
    }
    uint4 raw[KM][NV];
#pragma unroll
    for (int j = 0; j < KM; ++j) {  // -1: past k, or an assignment the permutation rejected
      const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(f) +
                                                      (size_t(r[j] < 0 ? 0 : r[j]) * H + c) * (F32 ? 4 : 2));
#pragma unroll
      for (int v = 0; v < NV; ++v) raw[j][v] = r[j] >= 0 ? __ldg(p + v) : make_uint4(0u, 0u, 0u, 0u);
    }
    uint4 sraw = make_uint4(0u, 0u, 0u, 0u);
    if (shared) sraw = __ldg(reinterpret_cast<const uint4*>(shared + size_t(t) * H + c));
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if (r[j] >= 0) {
        float v[8];
        if (F32) {
#pragma unroll
          for (int q = 0; q < NV; ++q) {
            v[4 * q] = __uint_as_float(raw[j][q].x);
            v[4 * q + 1] = __uint_as_float(raw[j][q].y);
            v[4 * q + 2] = __uint_as_float(raw[j][q].z);
            v[4 * q + 3] = __uint_as_float(raw[j][q].w);
          }
        } else {
          const uint32_t u[4] = {raw[j][0].x, raw[j][0].y, raw[j][0].z, raw[j][0].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 h = Pack2<T16>::unpack(u[i]);
            v[2 * i] = h.x;
            v[2 * i + 1] = h.y;
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj[j], v[i], acc[i]);
      }
    }
    if (shared) {
      const float g = gate ? gate[t] : 1.0f;
      const uint32_t u[4] = {sraw.x, sraw.y, sraw.z, sraw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 h = Pack2<T16>::unpack(u[i]);
        acc[2 * i] = fmaf(g, h.x, acc[2 * i]);
        acc[2 * i + 1] = fmaf(g, h.y, acc[2 * i + 1]);
      }
    }
    uint4 q;
    q.x = Pack2<T16>::pack(acc[0], acc[1]);
    q.y = Pack2<T16>::pack(acc[2], acc[3]);
    q.z = Pack2<T16>::pack(acc[4], acc[5]);
    q.w = Pack2<T16>::pack(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(y + size_t(t) * H + c) = q;
  }
}

template <typename T16, bool F32>
static cudaError_t launch_combine(dim3 grid, cudaStream_t stream, const void* f, const int32_t* slot_row, int ks,
                                  const float* w, const void* shared, const float* gate, int k, int H, int T,
                                  void* y) {
  const T16* sh = static_cast<const T16*>(shared);
  T16* yy = static_cast<T16*>(y);
  if (k <= 8) return launch_pdl(k_combine<T16, F32, 8>, grid, dim3(256), 0, stream, f, slot_row, ks, w, sh, gate, k, H, T, yy);
  if (k <= 12) return launch_pdl(k_combine<T16, F32, 12>, grid, dim3(256), 0, stream, f, slot_row, ks, w, sh, gate, k, H, T, yy);
  return launch_pdl(k_combine<T16, F32, 16>, grid, dim3(256), 0, stream, f, slot_row, ks, w, sh, gate, k, H, T, yy);
}

int combine(const void* f, int f_fp32, const int32_t* slot_row, int ks, const float* w, const void* shared,
            const float* gate, int T, int k, int H, int dtype, void* y, cudaStream_t stream) {
  if (T == 0) return MOE_OK;
  dim3 grid(std::min(T, 8 * num_sms()), (H / 8 + 255) / 256);
  if (dtype == MOE_DTYPE_BF16) {
    if (f_fp32)
      MOE_CHECK_CUDA((launch_combine<__nv_bfloat16, true>(grid, stream, f, slot_row, ks, w, shared, gate, k, H, T, y)));
    else
      MOE_CHECK_CUDA((launch_combine<__nv_bfloat16, false>(grid, stream, f, slot_row, ks, w, shared, gate, k, H, T, y)));
  } else {
    if (f_fp32)
      MOE_CHECK_CUDA((launch_combine<__half, true>(grid, stream, f, slot_row, ks, w, shared, gate, k, H, T, y)));
    else
      MOE_CHECK_CUDA((launch_combine<__half, false>(grid, stream, f, slot_row, ks, w, shared, gate, k, H, T, y)));
  }
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Refill-RMS: one block per token.  With p_j = exp(l_j - l_0):
//   Z = sum_{j<k} p_j, U = sum_{j<k} p_j f_j, y = U / Z,
//   delta_j = (U - p_j f_j + p_r f_r) / (Z - p_j + p_r) - y.
// ||delta_j||^2 is written to d2[slot_row[t, j]] (the permuted row of the
// assignment), the promoted slot's row gets -1; a second kernel sums each
// expert's rows in a fixed order.  A slot whose row is -1 (the permutation
// skipped an out-of-range expert id and recorded it in the status word)
// contributes zeros and writes nothing.
// ---------------------------------------------------------------------------
constexpr int kRefillMaxSlots = 16;

template <typename T16, bool F32>
__global__ void __launch_bounds__(256) k_refill(const void* __restrict__ f, const int32_t* __restrict__ slot_row,
                                                const float* __restrict__ topk_logit, int k, int H,
                                                const T16* __restrict__ shared, T16* __restrict__ y_out,
                                                double* __restrict__ d2) {
  const int t = blockIdx.x;
  const int ks = k + 1;
  __shared__ float p_sh[kRefillMaxSlots];
  __shared__ int row_sh[kRefillMaxSlots];
  __shared__ double red[8][kRefillMaxSlots];
  if (threadIdx.x < ks) {
    const float l0 = topk_logit[size_t(t) * ks];
    p_sh[threadIdx.x] = __expf(topk_logit[size_t(t) * ks + threadIdx.x] - l0);
    row_sh[threadIdx.x] = slot_row[size_t(t) * ks + threadIdx.x];
  }
  __syncthreads();
  float Z = 0.f;
  for (int j = 0; j < k; ++j) Z += p_sh[j];
  const float pr = p_sh[k];
  const float invZ = 1.0f / Z;
  float part[kRefillMaxSlots - 1];
#pragma unroll
  for (int j = 0; j < kRefillMaxSlots - 1; ++j) part[j] = 0.f;

  for (int c = threadIdx.x * 4; c < H; c += blockDim.x * 4) {
    float fv[kRefillMaxSlots][4];
    // every row load of the token is issued before the first use; a slot
    // without a row (-1: an out-of-range expert id, recorded by the
    // permutation) loads row 0 and contributes zeros
#pragma unroll
    for (int j = 0; j < kRefillMaxSlots; ++j)
      if (j < ks) load4<T16, F32>(f, size_t(max(row_sh[j], 0)), H, c, fv[j]);
#pragma unroll
    for (int j = 0; j < kRefillMaxSlots; ++j)
      if (j < ks && row_sh[j] < 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) fv[j][i] = 0.f;
      }
    float U[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kRefillMaxSlots - 1; ++j)
      if (j < k) {
#pragma unroll
        for (int i = 0; i < 4; ++i) U[i] = fmaf(p_sh[j], fv[j][i], U[i]);
      }
    float yv[4], fr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) yv[i] = U[i] * invZ;
#pragma unroll
    for (int j = 0; j < kRefillMaxSlots; ++j)
      if (j == k) {
#pragma unroll
        for (int i = 0; i < 4; ++i) fr[i] = fv[j][i];
      }
#pragma unroll
    for (int j = 0; j < kRefillMaxSlots - 1; ++j)
      if (j < k) {
        const float inv = 1.0f / (Z - p_sh[j] + pr);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float num = fmaf(pr, fr[i], fmaf(-p_sh[j], fv[j][i], U[i]));
          const float d = fmaf(num, inv, -yv[i]);
          part[j] = fmaf(d, d, part[j]);
        }
      }
    if (y_out) {
      if (shared) {
        float s[4];
        load4<T16, false>(shared, size_t(t), H, c, s);
#pragma unroll
        for (int i = 0; i < 4; ++i) yv[i] += s[i];
      }
      store4<T16>(y_out, size_t(t), H, c, yv);
    }
  }
  // block reduction of part[j] in FP64, fixed order
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int j = 0; j < kRefillMaxSlots - 1; ++j) {
    if (j < k) {
      double v = part[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp][j] = v;
    }
  }
  __syncthreads();
  if (threadIdx.x < ks && row_sh[threadIdx.x] >= 0) {
    const int j = threadIdx.x;
    if (j < k) {
      double s = 0.0;
      for (int w = 0; w < int(blockDim.x >> 5); ++w) s += red[w][j];
      d2[row_sh[j]] = s;
    } else {
      d2[row_sh[j]] = -1.0;  // the promoted expert earns nothing
    }
  }
}

// One block per expert: sum of its rows' ||delta||^2 (skipping -1 markers)
// in a fixed order; sum_sq[e] += total, count[e] += selected rows.
__global__ void __launch_bounds__(256) k_refill_reduce(const double* __restrict__ d2, const int32_t* __restrict__ offsets,
                                                       double* __restrict__ sum_sq, int64_t* __restrict__ count) {
  const int e = blockIdx.x;
  const int a = offsets[e], b = offsets[e + 1];
  double s = 0.0;
  long long n = 0;
  for (int r = a + threadIdx.x; r < b; r += blockDim.x) {
    const double v = d2[r];
    if (v >= 0.0) {
      s += v;
      ++n;
    }
  }
  __shared__ double rs[256];
  __shared__ long long rn[256];
  rs[threadIdx.x] = s;
  rn[threadIdx.x] = n;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      rs[threadIdx.x] += rs[threadIdx.x + o];
      rn[threadIdx.x] += rn[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0 && b > a) {
    sum_sq[e] += rs[0];
    count[e] += rn[0];
  }
}

size_t refill_ws_bytes(int T, int k) {
  WsCounter c;
  c.take<double>(size_t(T) * (k + 1));
  return c.used;
}

int refill(const void* f, int f_fp32, const int32_t* slot_row, const float* topk_logit, const int32_t* offsets, int T,
           int k, int H, int E, double* sum_sq, int64_t* count, const void* shared, void* y_out, int dtype, void* ws,
           size_t ws_bytes, cudaStream_t stream) {
  WsCarver carve(ws, ws_bytes);
  double* d2 = carve.take<double>(size_t(T) * (k + 1));
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "razor_refill_rms_accumulate: workspace of %zu bytes is too small", ws_bytes);
  if (T > 0) {
    if (dtype == MOE_DTYPE_BF16) {
      using T16 = __nv_bfloat16;
      if (f_fp32)
        k_refill<T16, true><<<T, 256, 0, stream>>>(f, slot_row, topk_logit, k, H, static_cast<const T16*>(shared),
                                                   static_cast<T16*>(y_out), d2);
      else
        k_refill<T16, false><<<T, 256, 0, stream>>>(f, slot_row, topk_logit, k, H, static_cast<const T16*>(shared),
                                                    static_cast<T16*>(y_out), d2);
    } else {
      using T16 = __half;
      if (f_fp32)
        k_refill<T16, true><<<T, 256, 0, stream>>>(f, slot_row, topk_logit, k, H, static_cast<const T16*>(shared),
                                                   static_cast<T16*>(y_out), d2);
      else
        k_refill<T16, false><<<T, 256, 0, stream>>>(f, slot_row, topk_logit, k, H, static_cast<const T16*>(shared),
                                                    static_cast<T16*>(y_out), d2);
    }
    MOE_CHECK_CUDA(cudaGetLastError());
  }
  k_refill_reduce<<<E, 256, 0, stream>>>(d2, offsets, sum_sq, count);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Selection: one block of 1024 threads, bitonic sort of (score desc, index
// asc) over the next power of two >= E, then the kept set in ascending index
// order by a block prefix sum over "rank < keep" flags.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_select(const double* __restrict__ sum_sq, const int64_t* __restrict__ count,
                                                 int E, int keep, int32_t* __restrict__ kept,
                                                 int32_t* __restrict__ ranking, double* __restrict__ score) {
  __shared__ double key[1024];
  __shared__ int id[1024];
  __shared__ int flag[1024];
  __shared__ int warp_tot[32];
  const int i = threadIdx.x;
  double s = -1.0;  // below every real score
  if (i < E) {
    const long long c = count[i];
    s = c > 0 ? sqrt(sum_sq[i] / double(c)) : 0.0;
    if (score) score[i] = s;
  }
  key[i] = s;
  id[i] = i;
  __syncthreads();
  // bitonic sort: "a before b" iff key_a > key_b or (key_a == key_b and id_a < id_b)
  for (int size = 2; size <= 1024; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int j = i ^ stride;
      if (j > i) {
        const bool up = (i & size) == 0;
        const bool i_first = key[i] > key[j] || (key[i] == key[j] && id[i] < id[j]);
        if (i_first != up) {
          double tk = key[i]; key[i] = key[j]; key[j] = tk;
          int ti = id[i]; id[i] = id[j]; id[j] = ti;
        }
      }
      __syncthreads();
    }
  }
  if (ranking && i < E) ranking[i] = id[i];
  flag[i] = 0;
  __syncthreads();
  if (i < keep) flag[id[i]] = 1;
  __syncthreads();
  const int v = flag[i];
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
  if (v && i < E) kept[base + incl - 1] = i;
}

int select_experts(const double* sum_sq, const int64_t* count, int E, int keep, int32_t* kept, int32_t* ranking,
                   double* score, cudaStream_t stream) {
  k_select<<<1, 1024, 0, stream>>>(sum_sq, count, E, keep, kept, ranking, score);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // namespace moe
