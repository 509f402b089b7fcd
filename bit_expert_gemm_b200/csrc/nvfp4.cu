// NVFP4 W4A4: per-tensor amax, group-16 quantisation (E2M1 codes, E4M3 block
// scales, FP32 global scale), and the grouped SwiGLU built on the
// block-scaled tcgen05 GEMM (gemm_nvfp4.cu).
#include <cstdlib>

#include "common.cuh"
#include "nvfp4.cuh"

namespace moe {

int gather_rows(const void* x, const int32_t* row_token, int rows, int H, void* out, cudaStream_t stream);
// decode batches (decode_fp4.cu)
int nvfp4_decode(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                 int E, const uint8_t* w_gu, const uint8_t* w1sf, const float* gs_gu, const uint8_t* w_d,
                 const uint8_t* w2sf, const float* gs_d, const float* act_gs_in, int out_fp32, void* f, uint8_t* xq,
                 uint8_t* xsf, uint16_t* h, unsigned* amax, float* gs, int32_t* active, cudaStream_t stream);

// BIT_EXPERT_GEMM_FP4_DECODE=0 sends decode batches through the grouped FP4 GEMMs too.
static bool fp4_decode_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* s = getenv("BIT_EXPERT_GEMM_FP4_DECODE");
    on = (s && s[0] == '0') ? 0 : 1;
  }
  return on != 0;
}

struct Nvfp4GemmArgs;  // gemm_nvfp4.cu
int launch_grouped_gemm_nvfp4(const uint8_t* A, const uint8_t* sfa, int a_rows, const uint8_t* B, const uint8_t* sfb,
                              int b_rows_total, const int* group_offsets, int G, int rows, int K, int n_out,
                              int b_rows_per_group, int up_offset, int swiglu, const float* gs_act,
                              const float* gs_w, int gs_w_stride, void* out, int ldo, int out_fp32, float* amax_out,
                              cudaStream_t stream, const int32_t* row_token);

// amax[b] = max |v| over tensor b of `batch` tensors of `n` 16-bit values
// (stored as float bits: non-negative floats order like integers).
template <typename T16>
__global__ void __launch_bounds__(256) k_amax(const T16* __restrict__ v, long n, int batch, unsigned* __restrict__ amax) {
  const int b = blockIdx.y;
  const uint4* p = reinterpret_cast<const uint4*>(v + b * n);
  const long nv = n / 8;
  float m = 0.0f;
  const long step = long(gridDim.x) * blockDim.x;
  // four independent 16-byte loads in flight per thread
  for (long i0 = long(blockIdx.x) * blockDim.x + threadIdx.x; i0 < nv; i0 += 4 * step) {
    uint4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) q[u] = i0 + u * step < nv ? __ldg(p + i0 + u * step) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f = Pack2<T16>::unpack(w[j]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax + b, __float_as_uint(m));
}

// One thread per block of 16 values of row r of tensor b.  Source row of
// output row r: row_token[r] when given (a gather), else r.  s_g = gs_in[b]
// when given, else amax[b] / 2688; thread 0 of each tensor writes gs_out[b].
template <typename T16>
__global__ void __launch_bounds__(256) k_nvfp4_quant(const T16* __restrict__ v, const int32_t* __restrict__ row_token,
                                                     int rows, int K, long src_tensor_stride,
                                                     const float* __restrict__ gs_in,
                                                     const unsigned* __restrict__ amax, uint8_t* __restrict__ codes,
                                                     uint8_t* __restrict__ sf, float* __restrict__ gs_out) {
  const int b = blockIdx.y;
  const int nb = K / 16;
  const long i = long(blockIdx.x) * blockDim.x + threadIdx.x;
  const float s_g = gs_in ? gs_in[b] : nvfp4_global_scale(__uint_as_float(amax[b]));
  if (i == 0 && gs_out) gs_out[b] = s_g;
  if (i >= long(rows) * nb) return;
  const int r = int(i / nb);
  const int blk = int(i - long(r) * nb);
  const long src_row = row_token ? row_token[r] : r;
  const uint4* src = reinterpret_cast<const uint4*>(v + b * src_tensor_stride + src_row * K + blk * 16);
  float x[16];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint4 q = __ldg(src + h);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = Pack2<T16>::unpack(w[j]);
      x[8 * h + 2 * j] = f.x;
      x[8 * h + 2 * j + 1] = f.y;
    }
  }
  uint32_t c[2];
  const uint32_t s = nvfp4_quant_block(x, s_g, c);
  const long out_row = long(b) * rows + r;
  *reinterpret_cast<uint2*>(codes + out_row * (K / 2) + blk * 8) = make_uint2(c[0], c[1]);
  sf[out_row * nb + blk] = uint8_t(s);
}

// ---------------------------------------------------------------------------
// Scale factors in the block-scaled GEMM's operand-tile order.  For operand
// tile t (128 rows) and K step kt (256 elements = 16 scales per row): four
// 512-byte atoms, one per MMA of K = 64; in atom j, 16-byte row i holds the
// scales 16kt + 4j .. 16kt + 4j + 3 of tile rows i, i + 32, i + 64, i + 96
// (one 32-bit word each), the layout tcgen05.cp copies into TMEM.  Rows
// outside the operand and scales past K are zero.  The GEMM then fetches a
// stage's scales with one 2 KB bulk copy per operand.
// ---------------------------------------------------------------------------
constexpr int kSfTileBytes = 2048;

__device__ __forceinline__ void pack_sf_row(const uint8_t* sf, int nsf, bool valid, size_t row, int kt, int i,
                                            uint8_t* tile) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = 16 * kt + 4 * j;
    const uint32_t w = (valid && c < nsf) ? __ldg(reinterpret_cast<const uint32_t*>(sf + row * nsf + c)) : 0u;
    *reinterpret_cast<uint32_t*>(tile + j * 512 + (i & 31) * 16 + (i >> 5) * 4) = w;
  }
}

// tile_start[g] = 128-row tiles of groups 0..g-1 (groups from offsets [G+1]); one block
__global__ void __launch_bounds__(1024) k_tile_starts(const int32_t* __restrict__ offsets, int G,
                                                      int32_t* __restrict__ tile_start) {
  __shared__ int warp_tot[32];
  const int per = (G + 1023) / 1024;
  const int g0 = threadIdx.x * per;
  int local = 0;
  for (int g = g0; g < g0 + per && g < G; ++g) local += (offsets[g + 1] - offsets[g] + 127) / 128;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
  for (int g = g0; g < g0 + per && g < G; ++g) {
    tile_start[g] = run;
    run += (offsets[g + 1] - offsets[g] + 127) / 128;
  }
  if (threadIdx.x == 1023) tile_start[G] = run;
}

// A operand (activations in permuted row order): tile t is rows
// offsets[g] + 128 m .. of group g, t = tile_start[g] + m; with row_token the
// scales of permuted row r are those of source row row_token[r].  Grid (max
// tiles, KT), 128 threads (one per tile row).
__global__ void __launch_bounds__(128) k_pack_sf_a(const uint8_t* __restrict__ sf, int K,
                                                   const int32_t* __restrict__ offsets, int G,
                                                   const int32_t* __restrict__ tile_start,
                                                   const int32_t* __restrict__ row_token, int src_rows,
                                                   uint8_t* __restrict__ out) {
  const int t = blockIdx.x, kt = blockIdx.y, i = threadIdx.x;
  if (t >= tile_start[G]) return;
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int m = t - tile_start[lo];
  const long row = long(offsets[lo]) + long(m) * 128 + i;
  bool valid = row < offsets[lo + 1];
  long src = row;
  if (valid && row_token) {
    src = row_token[row];
    valid = src >= 0 && src < src_rows;
  }
  pack_sf_row(sf, K / 16, valid, size_t(valid ? src : 0), kt, i, out + (size_t(t) * gridDim.y + kt) * kSfTileBytes);
}

// B operand (weights): tile (g, n) is, for SwiGLU, the 64 gate rows n*64.. and
// the 64 up rows up_offset + n*64.. of group g, else the 128 rows n*128...
// Grid (G * nt, KT), 128 threads.
__global__ void __launch_bounds__(128) k_pack_sf_b(const uint8_t* __restrict__ sf, int K, int nt, int rows_per_group,
                                                   int swiglu, int up_offset, uint8_t* __restrict__ out) {
  const int tile = blockIdx.x, kt = blockIdx.y, i = threadIdx.x;
  const int g = tile / nt, n = tile - g * nt;
  const int r = swiglu ? (i < 64 ? n * 64 + i : up_offset + n * 64 + i - 64) : n * 128 + i;
  pack_sf_row(sf, K / 16, r < rows_per_group, size_t(g) * rows_per_group + r, kt, i,
              out + (size_t(tile) * gridDim.y + kt) * kSfTileBytes);
}

// amax_n > 0: reduce amax over the first amax_n values of each tensor
// first; amax_n == 0: amax already holds it (or gs_in is given).
template <typename T16>
static int quant_impl(const void* v, const int32_t* row_token, int batch, int rows, int K, long src_tensor_stride,
                      long amax_n, const float* gs_in, unsigned* amax, uint8_t* codes, uint8_t* sf, float* gs_out,
                      cudaStream_t stream) {
  const T16* src = static_cast<const T16*>(v);
  if (!gs_in && amax_n > 0) {
    MOE_CHECK_CUDA(cudaMemsetAsync(amax, 0, sizeof(unsigned) * batch, stream));
    const long nv = amax_n / 8;
    const int gx = int(std::min<long>((nv + 255) / 256, long(num_sms()) * 8));
    k_amax<T16><<<dim3(gx > 0 ? gx : 1, batch), 256, 0, stream>>>(src, amax_n, batch, amax);
    MOE_CHECK_CUDA(cudaGetLastError());
  }
  const long n = long(rows) * (K / 16);
  if (n == 0) return MOE_OK;
  k_nvfp4_quant<T16><<<dim3(int((n + 255) / 256), batch), 256, 0, stream>>>(src, row_token, rows, K,
                                                                               src_tensor_stride, gs_in, amax, codes,
                                                                               sf, gs_out);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

static int quantize_rows(const void* v, int dtype, const int32_t* row_token, int batch, int rows, int K,
                         long src_tensor_stride, long amax_n, const float* gs_in, unsigned* amax, uint8_t* codes,
                         uint8_t* sf, float* gs_out, cudaStream_t stream) {
  if (dtype == MOE_DTYPE_BF16)
    return quant_impl<__nv_bfloat16>(v, row_token, batch, rows, K, src_tensor_stride, amax_n, gs_in, amax, codes, sf,
                                     gs_out, stream);
  return quant_impl<__half>(v, row_token, batch, rows, K, src_tensor_stride, amax_n, gs_in, amax, codes, sf, gs_out,
                            stream);
}

size_t nvfp4_quant_ws_bytes(int batch, int rows, int K) {
  (void)rows;
  (void)K;
  WsCounter c;
  c.take<unsigned>(size_t(batch > 0 ? batch : 1));
  return c.used;
}

int nvfp4_quantize(const void* v, int batch, int rows, int K, int dtype, const float* gs_in, uint8_t* codes,
                   uint8_t* sf, float* gs_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  WsCarver carve(ws, ws_bytes);
  unsigned* amax = carve.take<unsigned>(size_t(batch));
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_nvfp4_quantize: workspace of %zu bytes is too small", ws_bytes);
  const long n = long(rows) * K;
  return quantize_rows(v, dtype, nullptr, batch, rows, K, n, n, gs_in, amax, codes, sf, gs_out, stream);
}

// ---------------------------------------------------------------------------
// Grouped SwiGLU with NVFP4 weights and on-the-fly NVFP4 activations:
//   amax(x) -> quantise each token -> scales of the permuted rows in tile
//   order -> GEMM1 (gathering the FP4 rows of the permuted order itself;
//   +SwiGLU, h in BF16, amax(h)) -> quantise h -> scales in tile order ->
//   GEMM2.
// ---------------------------------------------------------------------------
struct Nvfp4Ws {
  uint8_t *xq, *xsf, *xq_tok, *xsf_tok, *hq, *hsf;
  int32_t* tile_start;                 // [E+1] 128-row tiles before each group
  uint8_t *xsf_p, *hsf_p, *w1sf_p, *w2sf_p;  // scales in GEMM tile order
  uint16_t* h;
  unsigned* amax;  // [2]: x, h
  float* gs;       // [2]: x, h
};

template <typename C>
static void carve_nvfp4(C& c, int rows, int H, int I) {
  c.template take<uint8_t>(size_t(rows) * H / 2);
  c.template take<uint8_t>(size_t(rows) * H / 16);
  // per-token codes and scales of x: T <= rows tokens
  c.template take<uint8_t>(size_t(rows) * H / 2);
  c.template take<uint8_t>(size_t(rows) * H / 16);
  c.template take<uint8_t>(size_t(rows) * I / 2);
  c.template take<uint8_t>(size_t(rows) * I / 16);
  c.template take<uint16_t>(size_t(rows) * I);
  c.template take<unsigned>(2);
  c.template take<float>(2);
}

// Tile-ordered scale factors: A tiles of the permuted rows (at most
// ceil(rows/128) + E), B tiles of every expert's weights.
template <typename C>
static void carve_nvfp4_packed(C& c, int rows, int H, int I, int E) {
  const size_t tiles = size_t(rows + 127) / 128 + E;
  const size_t kt1 = (H + 255) / 256, kt2 = (I + 255) / 256;
  c.template take<int32_t>(size_t(E) + 1);
  c.template take<uint8_t>(tiles * kt1 * kSfTileBytes);
  c.template take<uint8_t>(tiles * kt2 * kSfTileBytes);
  c.template take<uint8_t>(size_t(E) * (I / 64) * kt1 * kSfTileBytes);
  c.template take<uint8_t>(size_t(E) * (H / 128) * kt2 * kSfTileBytes);
}

size_t nvfp4_ws_bytes(int rows, int H, int I, int E) {
  WsCounter c;
  carve_nvfp4(c, rows, H, I);
  carve_nvfp4_packed(c, rows, H, I, E);
  return c.used;
}

int grouped_swiglu_nvfp4(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H,
                         int I, int E, const uint8_t* w_gu, const uint8_t* sf_gu, const float* gs_gu,
                         const uint8_t* w_d, const uint8_t* sf_d, const float* gs_d, const float* act_gs_in,
                         float* act_gs_out, int out_fp32, void* f, void* ws, size_t ws_bytes, cudaStream_t stream,
                         const uint8_t* w1sf_packed, const uint8_t* w2sf_packed) {
  WsCarver carve(ws, ws_bytes);
  Nvfp4Ws w;
  w.xq = carve.take<uint8_t>(size_t(rows) * H / 2);
  w.xsf = carve.take<uint8_t>(size_t(rows) * H / 16);
  w.xq_tok = carve.take<uint8_t>(size_t(T) * H / 2);
  w.xsf_tok = carve.take<uint8_t>(size_t(T) * H / 16);
  w.hq = carve.take<uint8_t>(size_t(rows) * I / 2);
  w.hsf = carve.take<uint8_t>(size_t(rows) * I / 16);
  w.h = carve.take<uint16_t>(size_t(rows) * I);
  w.amax = carve.take<unsigned>(2);
  w.gs = carve.take<float>(2);
  {
    const size_t tiles = size_t(rows + 127) / 128 + E;
    const size_t kt1 = (H + 255) / 256, kt2 = (I + 255) / 256;
    w.tile_start = carve.take<int32_t>(size_t(E) + 1);
    w.xsf_p = carve.take<uint8_t>(tiles * kt1 * kSfTileBytes);
    w.hsf_p = carve.take<uint8_t>(tiles * kt2 * kSfTileBytes);
    w.w1sf_p = carve.take<uint8_t>(size_t(E) * (I / 64) * kt1 * kSfTileBytes);
    w.w2sf_p = carve.take<uint8_t>(size_t(E) * (H / 128) * kt2 * kSfTileBytes);
  }
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_grouped_swiglu_nvfp4: workspace of %zu bytes is too small", ws_bytes);
  if (rows == 0) return MOE_OK;
  if (T <= kFp4DecodeMaxT && E <= 1024 && fp4_decode_enabled()) {
    // decode batch: CUDA-core GEMVs over the touched experts (decode_fp4.cu),
    // reading the weight scales in tile order
    const uint8_t* w1sf = w1sf_packed;
    const uint8_t* w2sf = w2sf_packed;
    const int kt1 = (H + 255) / 256, kt2 = (I + 255) / 256;
    if (!w1sf) {
      k_pack_sf_b<<<dim3(E * (I / 64), kt1), 128, 0, stream>>>(sf_gu, H, I / 64, 2 * I, 1, I, w.w1sf_p);
      w1sf = w.w1sf_p;
    }
    if (!w2sf) {
      k_pack_sf_b<<<dim3(E * (H / 128), kt2), 128, 0, stream>>>(sf_d, I, H / 128, H, 0, 0, w.w2sf_p);
      w2sf = w.w2sf_p;
    }
    MOE_CHECK_CUDA(cudaGetLastError());
    int rc = nvfp4_decode(x, row_token, offsets, T, rows, H, I, E, w_gu, w1sf, gs_gu, w_d, w2sf, gs_d, act_gs_in,
                          out_fp32, f, w.xq_tok, w.xsf_tok, w.h, w.amax, w.gs, w.tile_start, stream);
    if (rc) return rc;
    if (act_gs_out)
      MOE_CHECK_CUDA(cudaMemcpyAsync(act_gs_out, w.gs, 2 * sizeof(float), cudaMemcpyDeviceToDevice, stream));
    return MOE_OK;
  }
  // x: amax over the whole [T, H] input, each token quantised once; GEMM1
  // reads the FP4 rows of the permuted order through row_token (identical to
  // quantising the gathered rows: the quantisation is per row with the one
  // global scale of x), and the scale packing reads the per-token scales the
  // same way (identity rows, row_token == NULL: quantised in place)
  int rc = quantize_rows(x, MOE_DTYPE_BF16, nullptr, 1, T, H, 0, long(T) * H, act_gs_in, w.amax,
                         row_token ? w.xq_tok : w.xq, row_token ? w.xsf_tok : w.xsf, w.gs, stream);
  if (rc) return rc;
  // scale factors in GEMM tile order: A tiles of the permuted rows, B tiles of the weights
  const int tiles = (rows + 127) / 128 + E;
  const int kt1 = (H + 255) / 256, kt2 = (I + 255) / 256;
  k_tile_starts<<<1, 1024, 0, stream>>>(offsets, E, w.tile_start);
  k_pack_sf_a<<<dim3(tiles, kt1), 128, 0, stream>>>(row_token ? w.xsf_tok : w.xsf, H, offsets, E, w.tile_start,
                                                    row_token, T, w.xsf_p);
  const uint8_t* w1sf = w1sf_packed;
  if (!w1sf) {  // weight scales not packed by the caller: pack them for this call
    k_pack_sf_b<<<dim3(E * (I / 64), kt1), 128, 0, stream>>>(sf_gu, H, I / 64, 2 * I, 1, I, w.w1sf_p);
    w1sf = w.w1sf_p;
  }
  MOE_CHECK_CUDA(cudaGetLastError());
  MOE_CHECK_CUDA(cudaMemsetAsync(w.amax + 1, 0, sizeof(unsigned), stream));
  // A: the per-token FP4 rows gathered in the GEMM (row_token), or the rows in order
  rc = launch_grouped_gemm_nvfp4(row_token ? w.xq_tok : w.xq, w.xsf_p, row_token ? T : rows, w_gu, w1sf, E * 2 * I,
                                 offsets, E, rows, H, I, 2 * I, I, 1, w.gs, gs_gu, 2, w.h, I, 0,
                                 reinterpret_cast<float*>(w.amax + 1), stream, row_token);
  if (rc) return rc;
  rc = quantize_rows(w.h, MOE_DTYPE_BF16, nullptr, 1, rows, I, 0, 0, act_gs_in ? act_gs_in + 1 : nullptr, w.amax + 1,
                     w.hq, w.hsf, w.gs + 1, stream);
  if (rc) return rc;
  k_pack_sf_a<<<dim3(tiles, kt2), 128, 0, stream>>>(w.hsf, I, offsets, E, w.tile_start, nullptr, rows, w.hsf_p);
  const uint8_t* w2sf = w2sf_packed;
  if (!w2sf) {
    k_pack_sf_b<<<dim3(E * (H / 128), kt2), 128, 0, stream>>>(sf_d, I, H / 128, H, 0, 0, w.w2sf_p);
    w2sf = w.w2sf_p;
  }
  MOE_CHECK_CUDA(cudaGetLastError());
  rc = launch_grouped_gemm_nvfp4(w.hq, w.hsf_p, rows, w_d, w2sf, E * H, offsets, E, rows, I, H, H, 0, 0, w.gs + 1,
                                 gs_d, 1, f, H, out_fp32, nullptr, stream, nullptr);
  if (rc) return rc;
  if (act_gs_out) MOE_CHECK_CUDA(cudaMemcpyAsync(act_gs_out, w.gs, 2 * sizeof(float), cudaMemcpyDeviceToDevice, stream));
  return MOE_OK;
}

// Weight scales [E, rows_per_expert, K/16] in the FP4 GEMM's B-tile order:
// SwiGLU (gate/up) projections pair 64 gate rows n*64.. with the 64 up rows
// up_offset + n*64..; other projections take 128 rows per tile.
size_t nvfp4_packed_sf_bytes(int E, int rows_per_expert, int K, int swiglu) {
  (void)swiglu;  // both orders put 128 rows in a tile
  const size_t nt = size_t(rows_per_expert) / 128;
  return size_t(E) * nt * ((K + 255) / 256) * kSfTileBytes;
}

int nvfp4_prepack_sf(const uint8_t* sf, int E, int rows_per_expert, int K, int swiglu, uint8_t* out,
                     cudaStream_t stream) {
  const int kt = (K + 255) / 256;
  const int nt = rows_per_expert / 128;  // SwiGLU: I/64 tiles of 64 gate + 64 up rows (rows_per_expert = 2I)
  k_pack_sf_b<<<dim3(E * nt, kt), 128, 0, stream>>>(sf, K, nt, rows_per_expert, swiglu, rows_per_expert / 2, out);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // namespace moe
