// AWQ W4A16 asymmetric group-32 experts: grouped SwiGLU on the tcgen05 GEMM
// with in-kernel dequantisation, and a standalone dequantisation kernel that
// uses the same device function (exposes the GEMM's FP16 weights for tests).
#include "common.cuh"
#include "gemm_sm100.cuh"

namespace moe {

int gather_rows(const void* x, const int32_t* row_token, int rows, int H, void* out, cudaStream_t stream);

size_t awq_ws_bytes(int rows, int H, int I, int E) {
  WsCounter c;
  c.take<uint16_t>(size_t(rows) * H);
  c.take<uint16_t>(size_t(rows) * I);
  (void)E;
  return c.used;
}

int grouped_swiglu_awq(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                       int E, const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu, const int32_t* qw_d,
                       const int32_t* qz_d, const void* sc_d, int out_fp32, void* f, void* ws, size_t ws_bytes,
                       cudaStream_t stream) {
  (void)T;
  WsCarver carve(ws, ws_bytes);
  void* xp = row_token ? carve.take<uint16_t>(size_t(rows) * H) : nullptr;
  uint16_t* h = carve.take<uint16_t>(size_t(rows) * I);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_grouped_swiglu_awq_g32: workspace of %zu bytes is too small",
              ws_bytes);
  if (rows == 0) return MOE_OK;
  const void* a = x;
  if (row_token) {
    int rc = gather_rows(x, row_token, rows, H, xp, stream);
    if (rc) return rc;
    a = xp;
  }
  GemmArgs g1{};
  g1.group_offsets = offsets;
  g1.G = E;
  g1.rows = rows;
  g1.K = H;
  g1.n_out = I;
  g1.b_rows_per_group = 0;
  g1.up_offset = I;
  g1.out = h;
  g1.ldo = I;
  g1.out_fp32 = 0;
  g1.bias = nullptr;
  g1.bf16 = 0;
  g1.status = device_status_ptr();
  g1.limit_ns = wait_limit_ns();
  int rc = launch_grouped_gemm_awq(a, rows, qw_gu, qz_gu, sc_gu, 2 * I, g1, EPI_SWIGLU, pick_bn(rows, E, I, true),
                                   stream);
  if (rc) return rc;
  GemmArgs g2 = g1;
  g2.K = I;
  g2.n_out = H;
  g2.up_offset = 0;
  g2.out = f;
  g2.ldo = H;
  g2.out_fp32 = out_fp32;
  return launch_grouped_gemm_awq(h, rows, qw_d, qz_d, sc_d, H, g2, EPI_STORE, pick_bn(rows, E, H, false), stream);
}

// out[b, k, 8w .. 8w+7] = dequantised word (b, k, w); one thread per word.
__global__ void __launch_bounds__(256) k_awq_dequant(const uint32_t* __restrict__ qw, const uint32_t* __restrict__ qz,
                                                     const uint4* __restrict__ sc, int K, int W, long total,
                                                     uint4* __restrict__ out) {
  const long i = long(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const long bk = i / W;  // b * K + k
  const int w = int(i - bk * W);
  const long b = bk / K;
  const int k = int(bk - b * K);
  const long grow = b * (K / 32) + k / 32;
  out[i] = awq_dequant8(qw[i], qz[grow * W + w], sc[grow * W + w]);
}

int awq_dequant(const int32_t* qweight, const int32_t* qzeros, const void* scales, int batch, int K, int N, void* out,
                cudaStream_t stream) {
  const long total = long(batch) * K * (N / 8);
  if (total == 0) return MOE_OK;
  k_awq_dequant<<<int((total + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const uint32_t*>(qweight), reinterpret_cast<const uint32_t*>(qzeros),
      static_cast<const uint4*>(scales), K, N / 8, total, static_cast<uint4*>(out));
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // namespace moe
