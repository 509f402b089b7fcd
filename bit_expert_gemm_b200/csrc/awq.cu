// AWQ W4A16 asymmetric group-32 experts: grouped SwiGLU on the tcgen05 GEMM
// with in-kernel dequantisation, and a standalone dequantisation kernel that
// uses the same device function (exposes the GEMM's 16-bit weights for
// tests).  dtype selects FP16 (the checkpoint's runtime) or the BF16 mode
// (FP16 scales rounded to BF16, BF16 weights and activations).
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
                       const int32_t* qz_d, const void* sc_d, int dtype, int out_fp32, void* f, void* ws,
                       size_t ws_bytes, cudaStream_t stream, const void* awq_packed) {
  WsCarver carve(ws, ws_bytes);
  void* xp = row_token ? carve.take<uint16_t>(size_t(rows) * H) : nullptr;
  uint16_t* h = carve.take<uint16_t>(size_t(rows) * I);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_grouped_swiglu_awq_g32: workspace of %zu bytes is too small",
              ws_bytes);
  if (rows == 0) return MOE_OK;
  // with the packed copy GEMM1 gathers its A rows (x[row_token[r]]) itself;
  // otherwise they are gathered into xp first
  const void* a = x;
  const bool gather_in_gemm = row_token && awq_packed;
  if (row_token && !gather_in_gemm) {
    int rc = gather_rows(x, row_token, rows, H, xp, stream);
    if (rc) return rc;
    a = xp;
  }
  GemmArgs g1{};
  if (gather_in_gemm) {
    g1.row_token = row_token;
    g1.a_src = x;
    g1.a_src_rows = T;
  }
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
  g1.bf16 = dtype == MOE_DTYPE_BF16;
  g1.status = device_status_ptr();
  g1.limit_ns = wait_limit_ns();
  int rc = launch_grouped_gemm_awq(a, rows, qw_gu, qz_gu, sc_gu, 2 * I, g1, EPI_SWIGLU, pick_bn(rows, E, I, true),
                                   stream, awq_packed);
  if (rc) return rc;
  GemmArgs g2 = g1;
  g2.row_token = nullptr;  // GEMM2 reads h in the permuted order
  g2.a_src = nullptr;
  g2.a_src_rows = 0;
  g2.K = I;
  g2.n_out = H;
  g2.up_offset = 0;
  g2.out = f;
  g2.ldo = H;
  g2.out_fp32 = out_fp32;
  return launch_grouped_gemm_awq(h, rows, qw_d, qz_d, sc_d, H, g2, EPI_STORE, pick_bn(rows, E, H, false), stream,
                                 awq_packed);
}

// out[b, k, 8w .. 8w+7] = dequantised word (b, k, w); one thread per word.
template <bool BF>
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
  out[i] = awq_dequant8<BF>(qw[i], qz[grow * W + w], sc[grow * W + w]);
}

int awq_dequant(const int32_t* qweight, const int32_t* qzeros, const void* scales, int batch, int K, int N, int dtype,
                void* out, cudaStream_t stream) {
  const long total = long(batch) * K * (N / 8);
  if (total == 0) return MOE_OK;
  auto kern = dtype == MOE_DTYPE_BF16 ? k_awq_dequant<true> : k_awq_dequant<false>;
  kern<<<int((total + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const uint32_t*>(qweight), reinterpret_cast<const uint32_t*>(qzeros),
      static_cast<const uint4*>(scales), K, N / 8, total, static_cast<uint4*>(out));
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Tile-packed AWQ weights for the fused decode kernel.  Per expert, first the
// gate/up units (j, kt) for j < I/64, kt < H/64, then the down units (j, m)
// for j < I/64, m < H/128; each unit is kAwqUnitBytes = 4736 bytes laid out
// exactly as the kernel stages one 64-row K sub-tile in shared memory, so a
// single bulk copy brings it:
//   codes  [r0 16][wc 16][i 4] words: K row r0 + 16 i, code word wc of the
//          unit's 128 output columns (4096 bytes);
//   scales [2 groups][128 columns] FP16 (512 bytes);
//   zeros  [2 groups][16 words] (128 bytes).
// Gate/up unit (j, kt): K rows 64 kt.., output words 8j..8j+7 of the gate
// half (wc < 8) and I/8 + 8j.. of the up half (wc >= 8); down unit (j, m):
// K rows 64 j.. (the down projection's input features), output words
// 16 m..16 m + 15.  Codes and zero points are stored in pair order: the
// value of a word's output column 2m goes to nibble m, that of column 2m + 1
// to nibble m + 4 (the checkpoint has column c in nibble c), so that the
// dequantisation forms consecutive column pairs; scales are copied as they
// are.
// ---------------------------------------------------------------------------
constexpr int kAwqUnitBytes = 4736;

size_t awq_packed_bytes(int E, int H, int I) {
  return size_t(E) * size_t(I / 64) * size_t(H / 64 + H / 128) * kAwqUnitBytes;
}

// Column c of a checkpoint word (nibble c) to pair order: columns 2m, 2m + 1
// in nibbles m, m + 4.
__device__ __forceinline__ uint32_t awq_pair_order(uint32_t w) {
  uint32_t o = 0;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    o |= ((w >> (8 * m)) & 0xFu) << (4 * m);           // column 2m
    o |= ((w >> (8 * m + 4)) & 0xFu) << (4 * m + 16);  // column 2m + 1
  }
  return o;
}

// grid (units per expert, E), 256 threads
__global__ void __launch_bounds__(256) k_awq_pack(const uint32_t* __restrict__ qw_gu, const uint32_t* __restrict__ qz_gu,
                                                  const uint16_t* __restrict__ sc_gu, const uint32_t* __restrict__ qw_d,
                                                  const uint32_t* __restrict__ qz_d, const uint16_t* __restrict__ sc_d,
                                                  int H, int I, uint8_t* __restrict__ out) {
  const int u = blockIdx.x, e = blockIdx.y, t = threadIdx.x;
  const int nka = H / 64, nkb = H / 128, J = I / 64;
  const int NA = J * nka;
  uint8_t* dst = out + (size_t(e) * (NA + J * nkb) + u) * kAwqUnitBytes;
  const bool gu = u < NA;
  int j, m = 0, k0, W;
  const uint32_t *qw, *qz;
  const uint16_t* sc;
  if (gu) {
    j = u / nka;
    k0 = 64 * (u - j * nka);
    W = 2 * I / 8;
    qw = qw_gu + size_t(e) * H * W;
    qz = qz_gu + size_t(e) * (H / 32) * W;
    sc = sc_gu + size_t(e) * (H / 32) * (2 * I);
  } else {
    const int v = u - NA;
    j = v / nkb;
    m = v - j * nkb;
    k0 = 64 * j;
    W = H / 8;
    qw = qw_d + size_t(e) * I * W;
    qz = qz_d + size_t(e) * (I / 32) * W;
    sc = sc_d + size_t(e) * (I / 32) * H;
  }
  auto word = [&](int wc) { return gu ? (wc < 8 ? 8 * j + wc : I / 8 + 8 * j + wc - 8) : 16 * m + wc; };
  const int g0 = k0 / 32;
  {  // codes: thread t = (r0, wc) copies rows r0, r0 + 16, r0 + 32, r0 + 48 of word wc
    const int r0 = t >> 4, wc = t & 15;
    uint4 c;
    c.x = awq_pair_order(qw[size_t(k0 + r0) * W + word(wc)]);
    c.y = awq_pair_order(qw[size_t(k0 + r0 + 16) * W + word(wc)]);
    c.z = awq_pair_order(qw[size_t(k0 + r0 + 32) * W + word(wc)]);
    c.w = awq_pair_order(qw[size_t(k0 + r0 + 48) * W + word(wc)]);
    reinterpret_cast<uint4*>(dst)[t] = c;
  }
  {  // scales: thread t = (group, column)
    const int gi = t >> 7, c = t & 127;
    reinterpret_cast<uint16_t*>(dst + 4096)[t] = sc[size_t(g0 + gi) * (W * 8) + word(c >> 3) * 8 + (c & 7)];
  }
  if (t < 32) {  // zero points
    const int gi = t >> 4, wc = t & 15;
    reinterpret_cast<uint32_t*>(dst + 4608)[t] = awq_pair_order(qz[size_t(g0 + gi) * W + word(wc)]);
  }
}

int awq_prepack(const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu, const int32_t* qw_d,
                const int32_t* qz_d, const void* sc_d, int E, int H, int I, void* out, cudaStream_t stream) {
  const int units = (I / 64) * (H / 64 + H / 128);
  k_awq_pack<<<dim3(units, E), 256, 0, stream>>>(
      reinterpret_cast<const uint32_t*>(qw_gu), reinterpret_cast<const uint32_t*>(qz_gu),
      static_cast<const uint16_t*>(sc_gu), reinterpret_cast<const uint32_t*>(qw_d),
      reinterpret_cast<const uint32_t*>(qz_d), static_cast<const uint16_t*>(sc_d), H, I, static_cast<uint8_t*>(out));
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // namespace moe
