// RAZOR slicing and the router-norm keep policy.
//
// Qwen3.8-Flash-Next-RAZOR-65B-A6B-E256of512 card, opening paragraphs: a
// pruned layer keeps the selected experts' weights and router rows, cut from
// the original checkpoint in one and the same order, and its manifest lists
// the original expert indices in the pruned layer's order.  Same card, "Selection and
// calibration", MTP item: the MTP layer, which the text calibration never
// runs, keeps the experts whose original router rows have the largest L2
// norm (policy router_norm).
//
// k_router_norm  one warp per router row: the squares of the 16-bit weights,
//                exact in FP64, summed in a fixed order (lane-strided, then
//                a shuffle tree), written as Refill-style statistics
//                (sum_sq = ||row||^2, count = 1) so that razor_select ranks
//                them by sqrt(sum_sq / count) = ||row||.
// k_slice        dst[j] = src[kept[j]] for whole per-expert blocks of bytes:
//                one grid row per kept expert, 16-byte vectors when the block
//                size and both pointers allow, else 4-byte words, else bytes.
//                An index outside [0, E) is skipped and recorded in the
//                device status word.
#include "common.cuh"

namespace moe {

namespace {

template <typename T>
__device__ __forceinline__ double to_f64(T v);
template <>
__device__ __forceinline__ double to_f64<__nv_bfloat16>(__nv_bfloat16 v) { return double(__bfloat162float(v)); }
template <>
__device__ __forceinline__ double to_f64<__half>(__half v) { return double(__half2float(v)); }

template <typename T>
__global__ void __launch_bounds__(256) k_router_norm(const T* __restrict__ w, int E, int H, double* __restrict__ sum_sq,
                                                     int64_t* __restrict__ count) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (e >= E) return;
  const T* row = w + size_t(e) * H;
  double acc = 0.0;
  if ((H & 7) == 0 && (reinterpret_cast<uintptr_t>(w) & 15) == 0) {
    // 8 weights per 16-byte load; lane l takes chunks l, l + 32, ...
    const uint4* r4 = reinterpret_cast<const uint4*>(row);
    for (int c = lane; c < H / 8; c += 32) {
      const uint4 v = __ldg(r4 + c);
      const T* t = reinterpret_cast<const T*>(&v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const double d = to_f64(t[i]);
        acc = fma(d, d, acc);
      }
    }
  } else {
    for (int h = lane; h < H; h += 32) {
      const double d = to_f64(row[h]);
      acc = fma(d, d, acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    sum_sq[e] = acc;
    if (count) count[e] = 1;
  }
}

// Copies one kept expert's block per grid row (blockIdx.y = output slot j);
// the blocks of a row split the expert's units (V-byte vectors) between them.
template <typename V>
__global__ void __launch_bounds__(256) k_slice(const unsigned char* __restrict__ src, int E, size_t units_per_expert,
                                               const int32_t* __restrict__ kept, unsigned char* __restrict__ dst,
                                               int* status) {
  const int j = blockIdx.y;
  const int e = __ldg(kept + j);
  if (e < 0 || e >= E) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, MOE_ERR_INVALID_ARG);
    return;
  }
  const V* s = reinterpret_cast<const V*>(src) + size_t(e) * units_per_expert;
  V* d = reinterpret_cast<V*>(dst) + size_t(j) * units_per_expert;
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  size_t u = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  // four loads in flight per thread before their stores
  for (; u + 3 * stride < units_per_expert; u += 4 * stride) {
    const V a = s[u], b = s[u + stride], c = s[u + 2 * stride], q = s[u + 3 * stride];
    d[u] = a;
    d[u + stride] = b;
    d[u + 2 * stride] = c;
    d[u + 3 * stride] = q;
  }
  for (; u < units_per_expert; u += stride) d[u] = s[u];
}

template <typename V>
int launch_slice(const void* src, int E, size_t bytes_per_expert, const int32_t* kept, int keep, void* dst,
                 cudaStream_t stream) {
  const size_t units = bytes_per_expert / sizeof(V);
  // about four blocks of 256 threads per SM over the whole copy, at least one
  // per kept expert, and no more per expert than it has units for
  const size_t want = (size_t(num_sms()) * 4 + keep - 1) / keep;
  const size_t cap = (units + 255) / 256;
  size_t bx = want < cap ? want : cap;
  if (bx == 0) bx = 1;
  k_slice<V><<<dim3(unsigned(bx), keep), 256, 0, stream>>>(static_cast<const unsigned char*>(src), E, units, kept,
                                                  static_cast<unsigned char*>(dst), device_status_ptr());
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // namespace

int router_norm(const void* w_router, int E, int H, int dtype, double* sum_sq, int64_t* count, cudaStream_t stream) {
  const int rows_per_block = 8;
  const dim3 grid((E + rows_per_block - 1) / rows_per_block);
  if (dtype == MOE_DTYPE_BF16)
    k_router_norm<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(w_router), E, H, sum_sq,
                                                           count);
  else
    k_router_norm<__half><<<grid, 256, 0, stream>>>(static_cast<const __half*>(w_router), E, H, sum_sq, count);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

int slice_experts(const void* src, int E, size_t bytes_per_expert, const int32_t* kept, int keep, void* dst,
                  cudaStream_t stream) {
  if (keep == 0 || bytes_per_expert == 0) return MOE_OK;
  const uintptr_t a = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) | uintptr_t(bytes_per_expert);
  if ((a & 15) == 0) return launch_slice<uint4>(src, E, bytes_per_expert, kept, keep, dst, stream);
  if ((a & 3) == 0) return launch_slice<uint32_t>(src, E, bytes_per_expert, kept, keep, dst, stream);
  return launch_slice<unsigned char>(src, E, bytes_per_expert, kept, keep, dst, stream);
}

}  // namespace moe
