// NVFP4 W4A4 routed experts for decode batches (T <= 16): weight-streaming
// GEMVs on the CUDA cores with exact integer block products.
//
// Qwen3.8-Flash-Next-RAZOR-96B-A6B-NVFP4 card, component table: routed
// experts NVFP4 W4A4 -- E2M1 values in groups of 16 with an FP8 E4M3 scale
// per group and an FP32 scale per tensor -- for weights and activations.
//
// Inside one 16-element group both operands are E2M1 codes, and 2*e2m1 is an
// integer in {0, +-1, +-2, +-3, +-4, +-6, +-8, +-12}.  So the group's dot
// product sum (2w)(2x) is an exact integer (|.| <= 2304), computed with four
// dp4a; it is scaled by s_bw * s_bx (exact in FP32: two 4-bit significands)
// and accumulated in FP32 over the groups, and the sum is multiplied by
// s_gw * s_gx / 4.  That is the arithmetic of the block-scaled tensor-core
// MMA (exact products, FP32 sums), so this path and the grouped FP4 GEMMs
// compute the same function; a decode batch streams each touched expert's
// 2.2 MB once, which is HBM-bound work with no use for a 128-row MMA tile.
//
// Three launches, each a programmatic dependent of the one before (its
// launch and block scheduling overlap the previous kernel's tail):
//   k_fp4_prep    one block: amax of x, each token quantised once (the
//                 library's group-16 recipe), the list of experts with
//                 routed rows, and the h amax word cleared;
//   k_fp4_gemv<1> gate/up rows of every active expert against its tokens,
//                 SwiGLU, h in BF16 and its amax;
//   k_fp4_gemv<0> h quantised with its global scale (from the amax, or
//                 static), down rows against it, f.
// A work item is 32 weight rows of one expert, a quarter of a 128-row tile
// of the packed scale layout: gate/up tile n pairs gate rows 64n.. with up
// rows I + 64n.., and quarter q takes gate rows 64n + 16q.. with their 16 up
// rows; down quarter q of tile n is rows 128n + 32q...  Eight lanes share a
// row (16 bytes of codes = 32 elements each per 256-element K step,
// coalesced), each of the block's eight warps holds four rows, and the
// eight partial sums of a row are added with three shuffles.  The item's
// activations (the expert's n_e <= 16 tokens) are staged in shared memory as
// signed 2*e2m1 bytes plus FP32 group scales once per expert.
#include <algorithm>

#include "common.cuh"
#include "nvfp4.cuh"

namespace moe {

constexpr int kSfTileBytesDec = 2048;  // packed scales per 128-row tile and 256-element K step

namespace {

// 2*|e2m1| of codes 0..7 as bytes: 0, 1, 2, 3, 4, 6, 8, 12
constexpr uint32_t kMagLo = 0x03020100u, kMagHi = 0x0C080604u;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Four E2M1 codes (the low four nibbles of q, nibble i -> byte i) -> signed
// bytes 2*e2m1.  prmt selects the magnitude byte by the code's low three
// bits; a selector nibble with its top bit set (a negative code) replicates
// the selected byte's sign bit instead, which is 0 for every magnitude, so
// `pos` keeps the positive codes and `neg` (codes with the sign flipped) the
// negative ones.  (0x80 - m) ^ 0x80 is -m as a byte for 0 <= m <= 12, with
// no borrow between bytes.
__device__ __forceinline__ uint32_t e2m1x4_to_s8x4(uint32_t q) {
  const uint32_t pos = prmt(kMagLo, kMagHi, q);
  const uint32_t neg = prmt(kMagLo, kMagHi, q ^ 0x8888u);
  return pos | ((0x80808080u - neg) ^ 0x80808080u);
}

__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t pair16) {
  uint32_t h2;
  const uint16_t c = uint16_t(pair16 & 0xFFFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

struct Fp4DecArgs {
  const int32_t* offsets;   // [E+1]
  const int32_t* row_token; // [rows] token of each permuted row
  const int32_t* active;    // [1 + E]: count, then the experts with rows
  int E, T, H, I;
  // activations
  const uint8_t* xq;        // [T, H/2] codes of x (GEMM1)
  const uint8_t* xsf;       // [T, H/16] E4M3 scales of x
  float* gs;                // [2] global scales of x and h (written)
  unsigned* amax;           // [2] amax words of x and h
  const float* gs_in;       // [2] static scales or null
  __nv_bfloat16* h;         // [rows, I]
  // weights (codes [E, rows_pe, K/2], tile-ordered scales, global scales)
  const uint8_t* w;
  const uint8_t* wsf;
  const float* gsw;         // [E, 2] gate/up or [E] down
  void* f;                  // [rows, H] GEMM2 output
  int f_fp32;
};

// ---------------------------------------------------------------------------
// prep: x amax and quantisation, active experts, h amax cleared
// ---------------------------------------------------------------------------
template <typename T16>
__global__ void __launch_bounds__(1024) k_fp4_prep(const T16* __restrict__ x, Fp4DecArgs a, uint8_t* xq, uint8_t* xsf,
                                                   int32_t* active) {
  // launched as a programmatic dependent: inputs from the kernels before
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float red[32];
  __shared__ int scan[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = a.H, T = a.T;
  float s_g;
  if (a.gs_in) {
    s_g = a.gs_in[0];
  } else {
    float m = 0.f;
    const uint4* p = reinterpret_cast<const uint4*>(x);
    for (int i = tid; i < T * H / 8; i += blockDim.x) {
      const uint4 q = __ldg(p + i);
      const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = Pack2<T16>::unpack(wv[j]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
      m = lane < int(blockDim.x >> 5) ? red[lane] : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) red[0] = m;
    }
    __syncthreads();
    s_g = nvfp4_global_scale(red[0]);
  }
  if (tid == 0) {
    a.gs[0] = s_g;
    a.amax[1] = 0u;
  }
  // one 16-value group per thread and step, as the library's quantiser
  const int nb = H / 16;
  for (int i = tid; i < T * nb; i += blockDim.x) {
    const int t = i / nb, b = i - t * nb;
    const uint4* src = reinterpret_cast<const uint4*>(x + size_t(t) * H + b * 16);
    float v[16];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint4 q = __ldg(src + hh);
      const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = Pack2<T16>::unpack(wv[j]);
        v[8 * hh + 2 * j] = f.x;
        v[8 * hh + 2 * j + 1] = f.y;
      }
    }
    uint32_t c[2];
    const uint32_t s = nvfp4_quant_block(v, s_g, c);
    *reinterpret_cast<uint2*>(xq + size_t(t) * (H / 2) + b * 8) = make_uint2(c[0], c[1]);
    xsf[size_t(t) * nb + b] = uint8_t(s);
  }
  // experts with routed rows, in ascending order (E <= 1024 = blockDim)
  const int e = tid;
  const int has = e < a.E && a.offsets[e + 1] > a.offsets[e];
  const unsigned bal = __ballot_sync(0xffffffffu, has);
  if (lane == 0) scan[warp] = __popc(bal);
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += scan[w];
  if (has) active[1 + base + __popc(bal & ((1u << lane) - 1u))] = e;
  if (tid == blockDim.x - 1) active[0] = base + __popc(bal);
}

// ---------------------------------------------------------------------------
// GEMV over 32-row slices of one expert's 128-row tiles
// ---------------------------------------------------------------------------
// shared memory for T tokens: act [T][K] signed bytes, sx [T][K/16] FP32,
// res [T][32] FP32
__host__ __device__ constexpr size_t fp4_dec_smem(int K, int T) {
  return size_t(T) * K + size_t(T) * (K / 16) * 4 + size_t(T) * 32 * 4;
}

// Dot products of the slice's 32 weight rows with the n_e staged tokens:
// res[t][r] for slice row r.  Each warp takes four rows, eight lanes per
// row; all code and scale loads of the row (up to 8 K steps = 128 bytes per
// lane) are issued before the arithmetic, and the tokens are taken NT at a
// time with the codes kept in registers.
template <int NT>
__device__ __forceinline__ void fp4_rows(int K, int n_e, const uint8_t* wbase, const uint8_t* sf_tile, int I,
                                         int swiglu, int n, int q, const int8_t* act, const float* sx, float* res) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c8 = lane & 7;         // chunk of the row within a K step
  const int KT = (K + 255) / 256;  // K steps of 256 elements
  const int nchunk = K / 32;       // 32-element (16-byte) chunks of a row
  const int nb = K / 16;
  const int r = warp * 4 + (lane >> 3);  // slice row (8 warps x 4 rows)
  // tile row: gate/up slices pair gate rows 16q.. with up rows 64 + 16q..
  const int i = swiglu ? (r < 16 ? 16 * q + r : 64 + 16 * q + (r - 16)) : 32 * q + r;
  const int row = swiglu ? (i < 64 ? 64 * n + i : I + 64 * n + (i - 64)) : 128 * n + i;
  const uint8_t* wr = wbase + size_t(row) * (K / 2);
  const uint8_t* sfr = sf_tile + (c8 >> 1) * 512 + (i & 31) * 16 + (i >> 5) * 4;
  for (int kt0 = 0; kt0 < KT; kt0 += 8) {
    uint4 cw[8];
    uint32_t sw[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = (kt0 + u) * 8 + c8;
      const bool ok = kt0 + u < KT && c < nchunk;
      cw[u] = ok ? __ldg(reinterpret_cast<const uint4*>(wr) + c) : make_uint4(0, 0, 0, 0);
      sw[u] = ok ? __ldg(reinterpret_cast<const uint32_t*>(sfr + size_t(kt0 + u) * kSfTileBytesDec)) : 0u;
    }
    for (int t0 = 0; t0 < n_e; t0 += NT) {
      float acc[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t] = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = (kt0 + u) * 8 + c8;
        if (kt0 + u >= KT || c >= nchunk) continue;
        // the chunk's weights as signed bytes: group g0 (elements 0..15), g1 (16..31)
        const uint32_t w0 = e2m1x4_to_s8x4(cw[u].x), w1 = e2m1x4_to_s8x4(cw[u].x >> 16);
        const uint32_t w2 = e2m1x4_to_s8x4(cw[u].y), w3 = e2m1x4_to_s8x4(cw[u].y >> 16);
        const uint32_t w4 = e2m1x4_to_s8x4(cw[u].z), w5 = e2m1x4_to_s8x4(cw[u].z >> 16);
        const uint32_t w6 = e2m1x4_to_s8x4(cw[u].w), w7 = e2m1x4_to_s8x4(cw[u].w >> 16);
        // group scales: bytes 2 (c8 & 1) and 2 (c8 & 1) + 1 of the tile word
        const float2 swf = e4m3x2_to_f2(sw[u] >> (16 * (c8 & 1)));
        const int k0 = c * 32;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (t0 + t < n_e) {
            const int tt = t0 + t;
            const uint4 xa = *reinterpret_cast<const uint4*>(act + tt * K + k0);
            const uint4 xb = *reinterpret_cast<const uint4*>(act + tt * K + k0 + 16);
            const float2 sxf = *reinterpret_cast<const float2*>(sx + tt * nb + k0 / 16);
            int s0 = __dp4a(int(w0), int(xa.x), 0);
            s0 = __dp4a(int(w1), int(xa.y), s0);
            s0 = __dp4a(int(w2), int(xa.z), s0);
            s0 = __dp4a(int(w3), int(xa.w), s0);
            int s1 = __dp4a(int(w4), int(xb.x), 0);
            s1 = __dp4a(int(w5), int(xb.y), s1);
            s1 = __dp4a(int(w6), int(xb.z), s1);
            s1 = __dp4a(int(w7), int(xb.w), s1);
            acc[t] = fmaf(float(s0), swf.x * sxf.x, acc[t]);
            acc[t] = fmaf(float(s1), swf.y * sxf.y, acc[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float v = acc[t];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        // K steps beyond the first eight add to the partial result
        if (c8 == 0 && t0 + t < n_e) res[(t0 + t) * 32 + r] = (kt0 ? res[(t0 + t) * 32 + r] : 0.f) + v;
      }
    }
  }
}

// One launch of either GEMM.  Work item = (active expert, 128-row tile n,
// quarter q): 32 weight rows.  Each block takes a contiguous range of items
// and restages the activations only when the expert changes.
template <int SWIGLU>
__global__ void __launch_bounds__(256, 3) k_fp4_gemv(Fp4DecArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  griddep_wait();
  griddep_launch_dependents();
  const int K = SWIGLU ? a.H : a.I;
  const int nb = K / 16;
  int8_t* act = reinterpret_cast<int8_t*>(smem);
  float* sx = reinterpret_cast<float*>(smem + size_t(a.T) * K);
  float* res = sx + size_t(a.T) * nb;
  const int tiles = SWIGLU ? a.I / 64 : a.H / 128;  // 128-row tiles per expert
  const int rows_pe = SWIGLU ? 2 * a.I : a.H;
  const int KT = (K + 255) / 256;
  const int per_expert = 4 * tiles;
  const int n_items = a.active[0] * per_expert;
  const int per = (n_items + gridDim.x - 1) / gridDim.x;
  const int it0 = blockIdx.x * per, it1 = min(n_items, it0 + per);
  // global scale of the activations: x (written by k_fp4_prep), or h (from
  // the amax the gate/up launch left, or static)
  float s_ga;
  if (SWIGLU) {
    s_ga = a.gs[0];
  } else {
    s_ga = a.gs_in ? a.gs_in[1] : nvfp4_global_scale(__uint_as_float(a.amax[1]));
    if (blockIdx.x == 0 && threadIdx.x == 0) a.gs[1] = s_ga;
  }
  int staged = -1;
  for (int it = it0; it < it1; ++it) {
    const int e = a.active[1 + it / per_expert];
    const int rem = it - (it / per_expert) * per_expert;
    const int n = rem >> 2, q = rem & 3;
    const int r0 = a.offsets[e];
    const int n_e = min(a.offsets[e + 1] - r0, a.T);
    if (e != staged) {
      for (int qq = threadIdx.x; qq < n_e * nb; qq += blockDim.x) {
        const int t = qq / nb, b = qq - t * nb;
        uint32_t c[2];
        uint32_t s;
        if (SWIGLU) {
          const int tok = a.row_token ? a.row_token[r0 + t] : r0 + t;
          const uint2 cc = *reinterpret_cast<const uint2*>(a.xq + size_t(tok) * (K / 2) + b * 8);
          c[0] = cc.x;
          c[1] = cc.y;
          s = a.xsf[size_t(tok) * nb + b];
        } else {
          // group b of h row r0 + t, quantised as the library's quantiser does
          const uint4* src = reinterpret_cast<const uint4*>(a.h + size_t(r0 + t) * K + b * 16);
          float v[16];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint4 qv = src[hh];
            const uint32_t wv[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 f = Pack2<__nv_bfloat16>::unpack(wv[j]);
              v[8 * hh + 2 * j] = f.x;
              v[8 * hh + 2 * j + 1] = f.y;
            }
          }
          s = nvfp4_quant_block(v, s_ga, c);
        }
        uint4 o;
        o.x = e2m1x4_to_s8x4(c[0]);
        o.y = e2m1x4_to_s8x4(c[0] >> 16);
        o.z = e2m1x4_to_s8x4(c[1]);
        o.w = e2m1x4_to_s8x4(c[1] >> 16);
        *reinterpret_cast<uint4*>(act + t * K + b * 16) = o;
        sx[t * nb + b] = e4m3_to_f32(s);
      }
      __syncthreads();
      staged = e;
    }
    const uint8_t* wbase = a.w + size_t(e) * rows_pe * (K / 2);
    const uint8_t* sf_tile = a.wsf + (size_t(e) * tiles + n) * KT * kSfTileBytesDec;
    if (n_e <= 1)
      fp4_rows<1>(K, n_e, wbase, sf_tile, a.I, SWIGLU, n, q, act, sx, res);
    else if (n_e <= 2)
      fp4_rows<2>(K, n_e, wbase, sf_tile, a.I, SWIGLU, n, q, act, sx, res);
    else if (n_e <= 4)
      fp4_rows<4>(K, n_e, wbase, sf_tile, a.I, SWIGLU, n, q, act, sx, res);
    else
      fp4_rows<8>(K, n_e, wbase, sf_tile, a.I, SWIGLU, n, q, act, sx, res);
    __syncthreads();
    const int r = threadIdx.x;
    if (SWIGLU) {
      // h = silu(g) * u of feature 64n + 16q + r, rounded to BF16; its amax
      float m = 0.f;
      if (r < 16) {
        const float sg = a.gsw[2 * e] * s_ga * 0.25f, su = a.gsw[2 * e + 1] * s_ga * 0.25f;
        for (int t = 0; t < n_e; ++t) {
          const float g = res[t * 32 + r] * sg, u = res[t * 32 + 16 + r] * su;
          const __nv_bfloat16 hv = __float2bfloat16_rn(silu_f(g) * u);
          a.h[size_t(r0 + t) * a.I + 64 * n + 16 * q + r] = hv;
          m = fmaxf(m, fabsf(__bfloat162float(hv)));
        }
      }
      if (r < 32) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (r == 0) atomicMax(a.amax + 1, __float_as_uint(m));
      }
    } else if (r < 32) {
      const float sc = a.gsw[e] * s_ga * 0.25f;
      for (int t = 0; t < n_e; ++t) {
        const float v = res[t * 32 + r] * sc;
        const size_t o = size_t(r0 + t) * a.H + 128 * n + 32 * q + r;
        if (a.f_fp32)
          static_cast<float*>(a.f)[o] = v;
        else
          static_cast<__nv_bfloat16*>(a.f)[o] = __float2bfloat16_rn(v);
      }
    }
    __syncthreads();  // res and the staged activations are free again
  }
}

}  // namespace


// Routed NVFP4 experts of a decode batch.  xq/xsf: [T, H/2] / [T, H/16]
// scratch for the quantised tokens; h [rows, I] BF16 scratch; amax, gs [2];
// active [E + 1] scratch; w1sf / w2sf the weights' scales in tile order
// (moe_nvfp4_prepack_sf).
int nvfp4_decode(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                 int E, const uint8_t* w_gu, const uint8_t* w1sf, const float* gs_gu, const uint8_t* w_d,
                 const uint8_t* w2sf, const float* gs_d, const float* act_gs_in, int out_fp32, void* f, uint8_t* xq,
                 uint8_t* xsf, uint16_t* h, unsigned* amax, float* gs, int32_t* active, cudaStream_t stream) {
  MOE_REQUIRE(T >= 1 && T <= kFp4DecodeMaxT, MOE_ERR_UNSUPPORTED, "NVFP4 decode path: T=%d", T);
  MOE_REQUIRE(E <= 1024, MOE_ERR_UNSUPPORTED, "NVFP4 decode path: E=%d > 1024", E);
  Fp4DecArgs a{};
  a.offsets = offsets;
  a.row_token = row_token;
  a.active = active;
  a.E = E;
  a.T = T;
  a.H = H;
  a.I = I;
  a.xq = xq;
  a.xsf = xsf;
  a.gs = gs;
  a.amax = amax;
  a.gs_in = act_gs_in;
  a.h = reinterpret_cast<__nv_bfloat16*>(h);
  MOE_CHECK_CUDA(launch_pdl(k_fp4_prep<__nv_bfloat16>, dim3(1), dim3(1024), 0, stream,
                            static_cast<const __nv_bfloat16*>(x), a, xq, xsf, active));
  // work items: at most min(E, rows) experts x tiles x 4 slices; up to 8
  // blocks of 8 warps per SM
  const int max_active = std::min(E, rows);
  const size_t smem1 = fp4_dec_smem(H, T), smem2 = fp4_dec_smem(I, T);
  MOE_REQUIRE(smem1 <= 200 * 1024 && smem2 <= 200 * 1024, MOE_ERR_UNSUPPORTED, "NVFP4 decode path: H=%d too large",
              H);
  if (smem1 > 48 * 1024)
    MOE_CHECK_CUDA(cudaFuncSetAttribute(k_fp4_gemv<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem1)));
  if (smem2 > 48 * 1024)
    MOE_CHECK_CUDA(cudaFuncSetAttribute(k_fp4_gemv<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem2)));
  const int cap = num_sms() * 8;
  a.w = w_gu;
  a.wsf = w1sf;
  a.gsw = gs_gu;
  const int g1 = std::max(1, std::min(cap, max_active * (I / 64) * 4));
  MOE_CHECK_CUDA(launch_pdl(k_fp4_gemv<1>, dim3(g1), dim3(256), smem1, stream, a));
  a.w = w_d;
  a.wsf = w2sf;
  a.gsw = gs_d;
  a.f = f;
  a.f_fp32 = out_fp32;
  const int g2 = std::max(1, std::min(cap, max_active * (H / 128) * 4));
  MOE_CHECK_CUDA(launch_pdl(k_fp4_gemv<0>, dim3(g2), dim3(256), smem2, stream, a));
  return MOE_OK;
}

}  // namespace moe
