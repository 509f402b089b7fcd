// Persistent grouped GEMM on FP4 E2M1 operands with E4M3 block scales
// (tcgen05.mma kind::mxf4nvf4, one scale per 16 elements along K), fed by
// TMA, used by the NVFP4 W4A4 experts.
//
//   D[r, n] = sum_k e2m1(A[r,k]) sfa[r, k/16] * e2m1(B[n,k]) sfb[n, k/16]
//
// then scaled by the FP32 global scales of the activation and of the weight
// tensor in the epilogue.  Tiles: 128 rows of A x 128 rows of B, K stepped by
// 256 elements (one 128-byte swizzle row of packed FP4), four MMAs of K = 64
// per step.  The block scales arrive already in operand-tile order (nvfp4.cu
// k_pack_sf_a / k_pack_sf_b): per 128-row tile and K step, four 512-byte
// atoms in the 32x128-bit layout the tensor cores read (rows r, r+32, r+64,
// r+96 interleaved per 16-byte row), fetched with one 2 KB bulk copy per
// operand on the stage's barrier.  Two copy warps move them into a TMEM slot
// of their own per pipeline stage (tcgen05.cp, one for A and one for B, each
// committing to the stage's scales-ready barrier), so that the copies neither
// queue behind the MMA issue nor overwrite columns an MMA in flight still
// reads: copies issued by the MMA thread itself into one shared slot held
// the MMA pipe to about a third of its rate.
//
// With row_token, A rows are gathered in the kernel: four gather warps copy
// the 128-byte row segments of each K step from the per-token source with
// cp.async straight into the 128-byte-swizzled A tile (the layout the TMA
// would write), arriving on the stage barrier; rows past the group read zero.
//
// Warp roles: 0 and 8 TMA producers (A with its scales, B with its scales:
// one thread issuing every copy of a stage held the loads to about 86 GB/s
// per SM, since copy instructions block while the TMA unit is busy),
// 1 UMMA issuer (TMEM owner), 2..5 epilogue, 6 and 7 scale-factor copies
// (A and B), 9..12 A-row gather (with row_token).
#include <cstring>

#include "common.cuh"
#include "gemm_sm100.cuh"

namespace moe {

int make_tmap_2d_u8_sw128(CUtensorMap* map, const void* base, int rows, int cols_bytes, int box_rows);

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BKE = 256;                 // K elements per pipeline step
constexpr int BKB = BKE / 2;             // bytes per row per step
constexpr int A_BYTES = BM * BKB;        // 16 KB
constexpr int B_BYTES = BN * BKB;        // 16 KB
constexpr int SF_ATOM = 512;             // 128 rows x 4 scales
constexpr int SFA_OFF = A_BYTES + B_BYTES;
constexpr int SFB_OFF = SFA_OFF + 4 * SF_ATOM;
constexpr int STAGE_BYTES = SFB_OFF + 4 * SF_ATOM;  // 36 KB
#ifndef NVFP4_STAGES
#define NVFP4_STAGES 5
#endif
constexpr int STAGES = NVFP4_STAGES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
constexpr int kThreads = 416;
constexpr int kGatherWarp0 = 9;
constexpr int SF_TILE = 4 * SF_ATOM;     // scales of one operand tile for one K step
constexpr uint32_t TMEM_COLS = 512;      // 2 x 128 accumulator + a scale slot per stage
constexpr uint32_t SF_COL = 2 * BN;      // slot s at SF_COL + 32 s: A (4 MMAs x 4 columns), then B
constexpr uint32_t SF_SLOT = 32;
static_assert(SF_COL + STAGES * SF_SLOT <= TMEM_COLS, "scale slots must fit in TMEM");
static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte alignment");

struct Args {
  const int* group_offsets;
  int G, rows, K, n_out, b_rows_per_group, up_offset, swiglu;
  const uint8_t* sfa;  // A tiles (tile_start[g] + m) x K steps x SF_TILE
  const uint8_t* sfb;  // B tiles (g * n_tiles + n) x K steps x SF_TILE
  int a_rows, b_rows_total;
  const float* gs_act;  // device scalar
  const float* gs_w;    // [G * gs_w_stride]
  int gs_w_stride;
  void* out;
  int ldo, out_fp32;
  float* amax_out;  // SwiGLU: atomic max of |h| (float bits), may be null
  const int32_t* row_token;  // gathered A: A row r = source row row_token[r], or null (A rows in order)
  const uint8_t* a_src;      // gathered A: [a_src_rows, K/2] codes
  int a_src_rows;
  int* status;
  unsigned long long limit_ns;
};

__device__ __forceinline__ void umma_mxf4nvf4(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t sfa,
                                              uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}

// shared -> TMEM copy of one 32-row x 16-byte atom, replicated to the four
// 32-lane quadrants
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// descriptor of a contiguous 32 x 16-byte source (no swizzle; 8-row core
// matrices 128 bytes apart)
__device__ __forceinline__ uint64_t sdesc_sf_atom(uint32_t addr) {
  uint64_t d = 0;
  d |= uint64_t((addr >> 4) & 0x3FFFu);
  d |= uint64_t(128 >> 4) << 32;
  d |= uint64_t(1) << 46;
  return d;
}

// kind::mxf4nvf4 instruction descriptor: A, B E2M1 (1), K-major, UE4M3
// scales, M = 128, N = 128.
constexpr uint32_t kIdescMxf4 = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

struct TileMap {
  int g, m, n;
};

__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ void build_tile_table(const Args& a, int* goff, int* tile_start, int* warp_sums) {
  const int G = a.G, tid = threadIdx.x;
  for (int i = tid; i <= G; i += blockDim.x) goff[i] = a.group_offsets[i];
  __syncthreads();
  const int per = (G + blockDim.x - 1) / blockDim.x;
  const int g0 = tid * per;
  int local = 0;
  for (int g = g0; g < g0 + per && g < G; ++g) {
    int n = goff[g + 1] - goff[g];
    local += (n > 0 ? (n + BM - 1) / BM : 0);
  }
  const int lane = tid & 31, warp = tid >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_sums[w];
  int run = base + incl - local;
  for (int g = g0; g < g0 + per && g < G; ++g) {
    tile_start[g] = run;
    int n = goff[g + 1] - goff[g];
    run += (n > 0 ? (n + BM - 1) / BM : 0);
  }
  if (tid == blockDim.x - 1) tile_start[G] = run;
  __syncthreads();
}

__device__ __forceinline__ TileMap decode_tile(int L, int nt, const int* tile_start, int G) {
  TileMap t;
  int mt = L / nt;
  t.n = L - mt * nt;
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  t.g = lo;
  t.m = mt - tile_start[lo];
  return t;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm_nvfp4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const Args args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES], sfready_bar[STAGES], tfull_bar[2],
      tempty_bar[2], drain_bar, cdrain_bar[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int goff[kGemmMaxGroups + 1];
  __shared__ int tile_start[kGemmMaxGroups + 1];
  __shared__ int warp_sums[kThreads / 32];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  auto stg = [&](int s) { return smem + s * STAGE_BYTES; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // one expect_tx arrival from each producer (+ one per gather thread)
      mbar_init(&full_bar[s], 2 + (args.row_token ? 128 : 0));
      mbar_init(&empty_bar[s], 1);
      mbar_init(&sfready_bar[s], 2);  // one tcgen05.commit from each copy warp
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 128);
    }
    mbar_init(&drain_bar, 1);
    mbar_init(&cdrain_bar[0], 1);
    mbar_init(&cdrain_bar[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if ((warp == 0 || warp == 8) && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  build_tile_table(args, goff, tile_start, warp_sums);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;

  const int G = args.G;
  const int BNH = args.swiglu ? BN / 2 : BN;
  const int nt = args.n_out / BNH;
  const int total = tile_start[G] * nt;
  const int KT = (args.K + BKE - 1) / BKE;
  int* status = args.status;
  const unsigned long long lim = args.limit_ns;

  if (warp == 0 || warp == 8) {
    if (lane == 0) {
      // ---------------- TMA producers: warp 0 A, warp 8 B (codes + scales) ----------------
      const bool pa = warp == 0;
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        TileMap t = decode_tile(L, nt, tile_start, G);
        const int a_row = goff[t.g] + t.m * BM;
        const int b_row = t.g * args.b_rows_per_group + t.n * BNH;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, lim)) { ok = false; break; }
          if (pa) {
            const bool gathered = args.row_token != nullptr;  // then the gather warps bring A
            mbar_arrive_expect_tx(&full_bar[stage], (gathered ? 0 : A_BYTES) + SF_TILE);
            if (!gathered) tma_load_2d(stg(stage), &tmA, &full_bar[stage], kt * BKB, a_row);
            bulk_load(stg(stage) + SFA_OFF, args.sfa + (size_t(tile_start[t.g] + t.m) * KT + kt) * SF_TILE, SF_TILE,
                      &full_bar[stage]);
          } else {
            mbar_arrive_expect_tx(&full_bar[stage], B_BYTES + SF_TILE);
            bulk_load(stg(stage) + SFB_OFF, args.sfb + (size_t(t.g * nt + t.n) * KT + kt) * SF_TILE, SF_TILE,
                      &full_bar[stage]);
            if (args.swiglu) {
              tma_load_2d(stg(stage) + A_BYTES, &tmB, &full_bar[stage], kt * BKB, b_row);
              tma_load_2d(stg(stage) + A_BYTES + BNH * BKB, &tmB, &full_bar[stage], kt * BKB, b_row + args.up_offset);
            } else {
              tma_load_2d(stg(stage) + A_BYTES, &tmB, &full_bar[stage], kt * BKB, b_row);
            }
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        volatile int never = 0;
        for (long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          mbar_wait(&full_bar[i % STAGES], uint32_t((i / STAGES) & 1), &never, nullptr, lim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, &abort_flag, status, lim)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(acc * BN);
        for (int kt = 0; kt < KT; ++kt) {
          // the stage's scales are in TMEM (the copy warps saw its operands land first)
          if (!mbar_wait(&sfready_bar[stage], phase, &abort_flag, status, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sbase = smem_u32(stg(stage));
          const uint32_t sf = tmem_base + SF_COL + uint32_t(stage) * SF_SLOT;
          const uint64_t ad = sdesc_kmajor_sw128(sbase);
          const uint64_t bd = sdesc_kmajor_sw128(sbase + A_BYTES);
#pragma unroll
          for (int j = 0; j < 4; ++j)  // K = 64 per MMA: 32 bytes along the swizzled row
            umma_mxf4nvf4(d, ad + uint64_t(2 * j), bd + uint64_t(2 * j), kIdescMxf4, sf + 4 * j, sf + 16 + 4 * j,
                          (kt | j) != 0);
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      umma_commit(&drain_bar);
      volatile int never = 0;
      mbar_wait(&drain_bar, 0, &never, nullptr, lim);
    }
  } else if (warp >= kGatherWarp0) {
    if (args.row_token) {
      // ---------------- A row gather: warps 9..12 ----------------
      // Thread gt copies 16-byte chunk (gt % 8) of tile rows gt/8, gt/8 + 16, ...
      const int gt = threadIdx.x - kGatherWarp0 * 32;
      const int chunk = gt & 7, rbase = gt >> 3;
      const size_t pitch = size_t(args.K) / 2;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        TileMap t = decode_tile(L, nt, tile_start, G);
        const int a_row = goff[t.g] + t.m * BM;
        const int g_end = goff[t.g + 1];
        int tok[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = a_row + rbase + 16 * i;
          const int tk = (r < g_end && r < args.rows) ? __ldg(args.row_token + r) : -1;
          tok[i] = (tk >= 0 && tk < args.a_src_rows) ? tk : -1;
        }
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, lim)) { ok = false; break; }
          const uint32_t dst0 = smem_u32(stg(stage));
          const size_t kb = size_t(kt) * BKB + size_t(chunk) * 16;  // byte of the row
          const bool in_k = kb < pitch;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = rbase + 16 * i;
            const uint32_t dst = dst0 + uint32_t(r * 128 + ((chunk ^ (r & 7)) << 4));
            const bool v = tok[i] >= 0 && in_k;
            const uint8_t* g = args.a_src + (v ? size_t(tok[i]) * pitch + kb : 0);
            cp_async_16_zfill(dst, g, v ? 16u : 0u);
          }
          cp_async_arrive_noinc(&full_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      asm volatile("cp.async.wait_all;" ::: "memory");  // every copy has landed before the CTA exits
    }
  } else if (warp == 6 || warp == 7) {
    if (lane == 0) {
      // ---------------- scale-factor copies: warp 6 A, warp 7 B ----------------
      // Slot `stage` is free again once the stage has been refilled: the
      // producer refills only after the MMAs that read the slot completed.
      const int which = warp - 6;
      const uint32_t src_off = which ? SFB_OFF : SFA_OFF;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t src = smem_u32(stg(stage)) + src_off;
          const uint32_t dst = tmem_base + SF_COL + uint32_t(stage) * SF_SLOT + uint32_t(which * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j) tmem_cp_32x128b_x4(dst + 4 * j, sdesc_sf_atom(src + j * SF_ATOM));
          umma_commit(&sfready_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // this warp's copies have landed before TMEM is released
      umma_commit(&cdrain_bar[which]);
      volatile int never = 0;
      mbar_wait(&cdrain_bar[which], 0, &never, nullptr, lim);
    }
  } else {
    // ---------------- epilogue: warps 2..5 ----------------
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    const float gsa = *args.gs_act;
    int acc = 0;
    uint32_t acc_phase = 0;
    float hmax = 0.0f;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      TileMap t = decode_tile(L, nt, tile_start, G);
      const int n_g = goff[t.g + 1] - goff[t.g];
      const size_t out_row = size_t(goff[t.g]) + size_t(t.m) * BM + row_in_tile;
      const bool valid = t.m * BM + row_in_tile < n_g && out_row < size_t(args.rows);
      // the tile's weight global scales, loaded while the MMAs still run
      const float gw0 = __ldg(args.gs_w + t.g * args.gs_w_stride);
      const float gw1 = args.swiglu ? __ldg(args.gs_w + t.g * args.gs_w_stride + 1) : 0.0f;
      if (!mbar_wait(&tfull_bar[acc], acc_phase, &abort_flag, status, lim)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
      if (args.swiglu) {
        const float sg = gsa * gw0;
        const float su = gsa * gw1;
#pragma unroll 1
        for (int c = 0; c < BN / 2 / 32; ++c) {
          float gv[32], uv[32];
          tmem_ld32x2(tb + c * 32, tb + BN / 2 + c * 32, gv, uv);
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              // h is quantised to FP4 next: the fast division is ample here
              const float g0 = gv[2 * i] * sg, g1 = gv[2 * i + 1] * sg;
              const float h0 = __fdividef(g0, 1.0f + __expf(-g0)) * (uv[2 * i] * su);
              const float h1 = __fdividef(g1, 1.0f + __expf(-g1)) * (uv[2 * i + 1] * su);
              pk[i] = Pack2<__nv_bfloat16>::pack(h0, h1);
              // the amax is taken on the stored BF16 values, the ones that get quantised
              const float2 r = Pack2<__nv_bfloat16>::unpack(pk[i]);
              hmax = fmaxf(hmax, fmaxf(fabsf(r.x), fabsf(r.y)));
            }
            uint16_t* dst = reinterpret_cast<uint16_t*>(args.out) + out_row * size_t(args.ldo) + t.n * (BN / 2) + c * 32;
#pragma unroll
            for (int v = 0; v < 4; ++v) st_global_v4(dst + 8 * v, pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      } else {
        const float sw = gsa * gw0;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(tb + c * 32, v);
          if (valid) {
            const int col0 = t.n * BN + c * 32;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= sw;
            if (args.out_fp32) {
              float* dst = reinterpret_cast<float*>(args.out) + out_row * size_t(args.ldo) + col0;
#pragma unroll
              for (int i = 0; i < 8; ++i)
                st_global_v4(dst + 4 * i, __float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]),
                             __float_as_uint(v[4 * i + 2]), __float_as_uint(v[4 * i + 3]));
            } else {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = Pack2<__nv_bfloat16>::pack(v[2 * i], v[2 * i + 1]);
              uint16_t* dst = reinterpret_cast<uint16_t*>(args.out) + out_row * size_t(args.ldo) + col0;
#pragma unroll
              for (int i = 0; i < 4; ++i) st_global_v4(dst + 8 * i, pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    if (args.swiglu && args.amax_out) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
      if (lane == 0) atomicMax(reinterpret_cast<unsigned*>(args.amax_out), __float_as_uint(hmax));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

int launch_grouped_gemm_nvfp4(const uint8_t* A, const uint8_t* sfa, int a_rows, const uint8_t* B, const uint8_t* sfb,
                              int b_rows_total, const int* group_offsets, int G, int rows, int K, int n_out,
                              int b_rows_per_group, int up_offset, int swiglu, const float* gs_act,
                              const float* gs_w, int gs_w_stride, void* out, int ldo, int out_fp32, float* amax_out,
                              cudaStream_t stream, const int32_t* row_token) {
  MOE_REQUIRE(K % 64 == 0 && K > 0, MOE_ERR_UNSUPPORTED, "NVFP4 GEMM K=%d is not a positive multiple of 64", K);
  MOE_REQUIRE(G >= 1 && G <= kGemmMaxGroups, MOE_ERR_UNSUPPORTED, "NVFP4 GEMM group count %d", G);
  const int bnh = swiglu ? BN / 2 : BN;
  MOE_REQUIRE(n_out % bnh == 0, MOE_ERR_UNSUPPORTED, "NVFP4 GEMM output width %d is not a multiple of %d", n_out, bnh);
  if (a_rows == 0) return MOE_OK;
  CUtensorMap ta, tb;
  int rc = make_tmap_2d_u8_sw128(&ta, A, a_rows, K / 2, BM);
  if (rc) return rc;
  rc = make_tmap_2d_u8_sw128(&tb, B, b_rows_total, K / 2, bnh);
  if (rc) return rc;
  Args a{};
  a.group_offsets = group_offsets;
  a.G = G;
  a.rows = rows;
  a.K = K;
  a.n_out = n_out;
  a.b_rows_per_group = b_rows_per_group;
  a.up_offset = up_offset;
  a.swiglu = swiglu;
  a.sfa = sfa;
  a.sfb = sfb;
  a.a_rows = a_rows;
  a.b_rows_total = b_rows_total;
  a.gs_act = gs_act;
  a.gs_w = gs_w;
  a.gs_w_stride = gs_w_stride;
  a.out = out;
  a.ldo = ldo;
  a.out_fp32 = out_fp32;
  a.amax_out = amax_out;
  a.row_token = row_token;  // A = per-source rows [a_rows, K/2], gathered through row_token
  a.a_src = A;
  a.a_src_rows = a_rows;
  a.status = device_status_ptr();
  a.limit_ns = wait_limit_ns();
  static bool attr_set[64] = {false};
  int dev = 0;
  MOE_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev >= 64 || !attr_set[dev]) {
    MOE_CHECK_CUDA(cudaFuncSetAttribute(k_grouped_gemm_nvfp4, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    if (dev < 64) attr_set[dev] = true;
  }
  k_grouped_gemm_nvfp4<<<num_sms(), kThreads, SMEM_BYTES, stream>>>(ta, tb, a);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // namespace moe
