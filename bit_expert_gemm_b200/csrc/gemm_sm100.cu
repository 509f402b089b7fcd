// Persistent grouped tcgen05 GEMM (see gemm_sm100.cuh for the contract).
#include <cstring>

#include "gemm_sm100.cuh"

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_TILE_BYTES = BM * BK * 2;
constexpr int kBaseThreads = 192;    // producer, UMMA issuer, 4 epilogue warps
constexpr int kDequantThreads = 256;  // 8 AWQ dequantisation warps
constexpr int kGatherThreads = 128;   // 4 row-gather warps (A rows loaded through row_token)
constexpr int kStoreStride = 128 + 16;  // epilogue staging: bytes per row of a 32-column chunk, padded
constexpr int kSmemBudget = 196 * 1024;
// one unit of the tile-packed AWQ copy (awq.cu): codes, scales and zero
// points of 64 K rows x 128 output columns
constexpr int kAwqUnit = 4736;

enum { W_DENSE = 0, W_AWQ = 1, W_AWQ_BF16 = 2 };  // AWQ_BF16: the BF16 mode of the AWQ dequantisation

template <int BN, int EPI, int WQ, int AG>
struct GemmCfg {
  static constexpr int B_TILE_BYTES = BN * BK * 2;
  // AWQ staging per stage, one TMA box per output half (gate / up for SwiGLU):
  // codes [64][W2] words, scales [2][8*W2] FP16, zeros [2][W2] words.  Every
  // box starts on a 128-byte boundary (a requirement of tensor copies).
  static constexpr int NBOX = (EPI == EPI_SWIGLU) ? 2 : 1;
  static constexpr int W2 = BN / 8 / NBOX;
  static constexpr int CODE_BOX = WQ ? BK * W2 * 4 : 0;
  static constexpr int SCALE_BOX = WQ ? (2 * W2 * 8 * 2 + 127) / 128 * 128 : 0;
  static constexpr int ZERO_BOX = WQ ? (2 * W2 * 4 + 127) / 128 * 128 : 0;
  static constexpr int CODE_OFF = A_TILE_BYTES + B_TILE_BYTES;
  static constexpr int SCALE_OFF = CODE_OFF + NBOX * CODE_BOX;
  static constexpr int ZERO_OFF = SCALE_OFF + NBOX * SCALE_BOX;
  static constexpr int RAW_BYTES = ZERO_OFF + NBOX * ZERO_BOX;
  static constexpr int STAGE_BYTES = (RAW_BYTES + 1023) / 1024 * 1024;  // keep every tile 1024-byte aligned
  // bytes the TMA brings per stage (a gathered A tile arrives through cp.async instead)
  static constexpr int TX_BYTES =
      (AG ? 0 : A_TILE_BYTES) + (WQ ? NBOX * (BK * W2 * 4 + 2 * W2 * 8 * 2 + 2 * W2 * 4) : B_TILE_BYTES);
  static constexpr int STAGES = kSmemBudget / STAGE_BYTES > 8 ? 8 : kSmemBudget / STAGE_BYTES;
  static constexpr int STORE_BYTES = 4 * 32 * kStoreStride;   // epilogue staging, 32 rows per epilogue warp
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + STORE_BYTES;  // +1024: alignment slack
  static constexpr uint32_t TMEM_COLS = 2 * BN;                    // two accumulators
  static constexpr int GATHER_WARP0 = (kBaseThreads + (WQ ? kDequantThreads : 0)) / 32;
  static constexpr int THREADS = kBaseThreads + (WQ ? kDequantThreads : 0) + (AG ? kGatherThreads : 0);
  static constexpr uint32_t FULL_ARRIVALS = 1 + (AG ? kGatherThreads : 0);
  // MN-major B tile (AWQ): 64-element atoms along N are LBO apart, 8-row K groups SBO apart
  static constexpr uint32_t B_SBO = 1024;
  static constexpr uint32_t B_LBO = (BK / 8) * 1024;
  static_assert(STAGE_BYTES % 1024 == 0 && A_TILE_BYTES % 1024 == 0 && B_TILE_BYTES % 1024 == 0,
                "swizzled tiles must stay 1024-byte aligned");
  static_assert(CODE_BOX % 128 == 0 && SCALE_BOX % 128 == 0 && ZERO_BOX % 128 == 0 && CODE_OFF % 128 == 0 &&
                    SCALE_OFF % 128 == 0 && ZERO_OFF % 128 == 0,
                "every TMA destination must be 128-byte aligned");
  static_assert(W2 * 4 >= 16, "TMA boxes need at least 16 bytes per row");
  // the tile-packed AWQ path brings BN / 128 units of 4736 bytes into the same staging area
  static_assert(!WQ || BN < 128 || (TX_BYTES - (AG ? 0 : A_TILE_BYTES) == BN / 128 * 4736 &&
                                    RAW_BYTES - CODE_OFF >= BN / 128 * 4736),
                "packed AWQ units must match the staging area");
};

struct TileMap {
  int g, m, n;
};

// Exclusive scan of per-group m-tile counts into tile_start[0..G]; also
// stores group row offsets in goff[0..G].  All threads participate.
__device__ void build_tile_table(const GemmArgs& a, int* goff, int* tile_start, int* warp_sums) {
  const int G = a.G;
  const int tid = threadIdx.x;
  for (int i = tid; i <= G; i += blockDim.x) goff[i] = a.group_offsets ? a.group_offsets[i] : (i == 0 ? 0 : a.rows);
  __syncthreads();
  const int per = (G + blockDim.x - 1) / blockDim.x;  // each thread owns a contiguous chunk of groups
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
  int warp_base = 0;
  for (int w = 0; w < warp; ++w) warp_base += warp_sums[w];
  int run = warp_base + incl - local;
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
  // last g with tile_start[g] <= mt (empty groups share their start with the next one)
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  t.g = lo;
  t.m = mt - tile_start[lo];
  return t;
}

// Epilogue store of a 32-row x RB-byte chunk held one row per lane: the rows
// go through the warp's staging area so that every store instruction writes
// whole contiguous row segments (RB/16 lanes per row) instead of 16 bytes of
// 32 different rows.  Rows r >= nvalid are not written.
template <int RB>
__device__ __forceinline__ void warp_store_rows(uint8_t* stg, const uint32_t* vals, int nvalid, uint8_t* gbase,
                                                size_t pitch, int lane) {
  uint4* mine = reinterpret_cast<uint4*>(stg + lane * kStoreStride);
#pragma unroll
  for (int i = 0; i < RB / 16; ++i) mine[i] = make_uint4(vals[4 * i], vals[4 * i + 1], vals[4 * i + 2], vals[4 * i + 3]);
  __syncwarp();
  constexpr int LPR = RB / 16, RPP = 32 / LPR;
  const int seg = lane % LPR;
#pragma unroll
  for (int p = 0; p < LPR; ++p) {
    const int r = p * RPP + lane / LPR;
    const uint4 v = *reinterpret_cast<const uint4*>(stg + r * kStoreStride + seg * 16);
    if (r < nvalid) st_global_v4(gbase + size_t(r) * pitch + seg * 16, v.x, v.y, v.z, v.w);
  }
  __syncwarp();
}

__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Tensor maps of the B source.  Dense: b = the weight matrix.  AWQ: codes,
// scales, zeros (b unused).
struct BMaps {
  CUtensorMap b, codes, scales, zeros;
};

template <int BN, int EPI, int WQ, int AG>
__global__ void __launch_bounds__(GemmCfg<BN, EPI, WQ, AG>::THREADS, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BMaps bm, const GemmArgs args) {
  using Cfg = GemmCfg<BN, EPI, WQ, AG>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int BNH = (EPI == EPI_SWIGLU) ? BN / 2 : BN;  // output columns per tile
  constexpr int WC = BN / 8;                               // AWQ code words per K row of the tile
  constexpr int W2 = Cfg::W2;                              // words per TMA box (gate / up halves)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES], bready_bar[STAGES], tfull_bar[2],
      tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int goff[kGemmMaxGroups + 1];
  __shared__ int tile_start[kGemmMaxGroups + 1];
  __shared__ int warp_sums[Cfg::THREADS / 32];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  auto smA = [&](int s) { return smem + s * Cfg::STAGE_BYTES; };
  auto smB = [&](int s) { return smem + s * Cfg::STAGE_BYTES + A_TILE_BYTES; };
  // AWQ staging box `half` (0: gate / all, 1: up) of stage s
  auto smCodes = [&](int s, int half) {
    return reinterpret_cast<uint32_t*>(smA(s) + Cfg::CODE_OFF + half * Cfg::CODE_BOX);
  };
  auto smScales = [&](int s, int half) {
    return reinterpret_cast<uint16_t*>(smA(s) + Cfg::SCALE_OFF + half * Cfg::SCALE_BOX);
  };
  auto smZeros = [&](int s, int half) {
    return reinterpret_cast<uint32_t*>(smA(s) + Cfg::ZERO_OFF + half * Cfg::ZERO_BOX);
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], Cfg::FULL_ARRIVALS);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&bready_bar[s], kDequantThreads / 32);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 128);
    }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    if (WQ) {
      tma_prefetch_desc(&bm.codes);
      tma_prefetch_desc(&bm.scales);
      tma_prefetch_desc(&bm.zeros);
    } else {
      tma_prefetch_desc(&bm.b);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  build_tile_table(args, goff, tile_start, warp_sums);  // contains __syncthreads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;

  const int G = args.G;
  const int nt = args.n_out / BNH;
  const int total = tile_start[G] * nt;
  const int KB = args.K / BK;
  int* status = args.status;
  const unsigned long long lim = args.limit_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        TileMap t = decode_tile(L, nt, tile_start, G);
        const int a_row = goff[t.g] + t.m * BM;
        const int b_row = t.g * args.b_rows_per_group + t.n * BNH;
        const int col0 = t.n * BNH;  // AWQ: first output column of the tile (gate half)
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::TX_BYTES);
          if (!AG) tma_load_2d(smA(stage), &tmA, &full_bar[stage], kb * BK, a_row);
          if (WQ && args.awq_packed) {
            // the stage's BN / 128 packed units, contiguous in the staging
            // area: gate/up unit (j, kb) of column block j, or down unit
            // (kb, m) of column block m (per expert: J = I/64 column blocks
            // of H/64 gate/up units, then J K-blocks of H/128 down units)
            const int Hd = EPI == EPI_SWIGLU ? args.K : args.n_out;
            const int Iw = EPI == EPI_SWIGLU ? args.n_out : args.K;
            const int nka = Hd / 64, nkb = Hd / 128, J = Iw / 64;
            const size_t base = size_t(t.g) * J * (nka + nkb);
            constexpr int NU = BN / 128;
#pragma unroll
            for (int u = 0; u < NU; ++u) {
              const int c = t.n * NU + u;
              const size_t unit = base + (EPI == EPI_SWIGLU ? size_t(c) * nka + kb
                                                            : size_t(J) * nka + size_t(kb) * nkb + c);
              bulk_load(reinterpret_cast<uint8_t*>(smCodes(stage, 0)) + u * kAwqUnit,
                        args.awq_packed + unit * kAwqUnit, uint32_t(kAwqUnit), &full_bar[stage]);
            }
          } else if (WQ) {
            const int crow = t.g * args.K + kb * BK;          // code rows (input dim)
            const int grow = t.g * (args.K / 32) + kb * (BK / 32);  // scale / zero rows (groups)
            tma_load_2d(smCodes(stage, 0), &bm.codes, &full_bar[stage], col0 / 8, crow);
            tma_load_2d(smScales(stage, 0), &bm.scales, &full_bar[stage], col0, grow);
            tma_load_2d(smZeros(stage, 0), &bm.zeros, &full_bar[stage], col0 / 8, grow);
            if (EPI == EPI_SWIGLU) {
              const int c1 = args.up_offset + col0;
              tma_load_2d(smCodes(stage, 1), &bm.codes, &full_bar[stage], c1 / 8, crow);
              tma_load_2d(smScales(stage, 1), &bm.scales, &full_bar[stage], c1, grow);
              tma_load_2d(smZeros(stage, 1), &bm.zeros, &full_bar[stage], c1 / 8, grow);
            }
          } else if (EPI == EPI_SWIGLU) {
            tma_load_2d(smB(stage), &bm.b, &full_bar[stage], kb * BK, b_row);
            tma_load_2d(smB(stage) + BNH * BK * 2, &bm.b, &full_bar[stage], kb * BK, b_row + args.up_offset);
          } else {
            tma_load_2d(smB(stage), &bm.b, &full_bar[stage], kb * BK, b_row);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // let the copies already in flight land before the CTA exits
        volatile int never = 0;
        for (long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          mbar_wait(&full_bar[i % STAGES], uint32_t((i / STAGES) & 1), &never, nullptr, lim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer ----------------
      const uint32_t idesc = idesc_f16(args.bf16, BM, BN) | (WQ ? (1u << 16) : 0u);  // AWQ: B is MN-major
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, &abort_flag, status, lim)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(acc * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status, lim)) { ok = false; break; }
          if (WQ && !mbar_wait(&bready_bar[stage], phase, &abort_flag, status, lim)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = sdesc_kmajor_sw128(smem_u32(smA(stage)));
          if (WQ) {
            const uint64_t bd = sdesc_mnmajor_sw128(smem_u32(smB(stage)), Cfg::B_LBO, Cfg::B_SBO);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)  // 16 K = two 8-row groups = 2 * SBO bytes
              umma_f16(d, ad + uint64_t(kk * 2), bd + uint64_t(kk * (2 * Cfg::B_SBO >> 4)), idesc, (kb | kk) != 0);
          } else {
            const uint64_t bd = sdesc_kmajor_sw128(smem_u32(smB(stage)));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_f16(d, ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc, (kb | kk) != 0);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // every issued UMMA must be complete before TMEM is released
      umma_commit(&drain_bar);
      volatile int never = 0;
      mbar_wait(&drain_bar, 0, &never, nullptr, lim);
    }
  } else if (warp < 6) {
    // ---------------- epilogue: warps 2..5 ----------------
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    uint8_t* stg = smem + STAGES * Cfg::STAGE_BYTES + (warp - 2) * 32 * kStoreStride;
    const size_t esize = args.out_fp32 ? 4 : 2;
    const size_t pitch = size_t(args.ldo) * esize;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      TileMap t = decode_tile(L, nt, tile_start, G);
      const int n_g = goff[t.g + 1] - goff[t.g];
      const size_t row0 = size_t(goff[t.g]) + size_t(t.m) * BM + q * 32;  // this warp's first output row
      // rows past the group, or (with inconsistent offsets) past the output, are not written
      int nvalid = n_g - (t.m * BM + q * 32);
      nvalid = nvalid < 0 ? 0 : (nvalid > 32 ? 32 : nvalid);
      if (row0 + nvalid > size_t(args.rows)) nvalid = row0 < size_t(args.rows) ? int(size_t(args.rows) - row0) : 0;
      uint8_t* gtile = reinterpret_cast<uint8_t*>(args.out) + row0 * pitch;
      if (!mbar_wait(&tfull_bar[acc], acc_phase, &abort_flag, status, lim)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
      if (EPI == EPI_SWIGLU) {
#pragma unroll 1
        for (int c = 0; c < BNH / 32; ++c) {
          float gv[32], uv[32];
          tmem_ld32x2(tb + c * 32, tb + BNH + c * 32, gv, uv);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float h0 = silu_f(gv[2 * i]) * uv[2 * i];
            float h1 = silu_f(gv[2 * i + 1]) * uv[2 * i + 1];
            pk[i] = args.bf16 ? Pack2<__nv_bfloat16>::pack(h0, h1) : Pack2<__half>::pack(h0, h1);
          }
          warp_store_rows<64>(stg, pk, nvalid, gtile + size_t(t.n * BNH + c * 32) * 2, pitch, lane);
        }
      } else if (!args.out_fp32 && !args.bias) {
        // 16-bit output: 64 columns per TMEM load wait, stored as whole
        // 128-byte segments of each row
        static_assert(BN % 64 == 0, "tile widths are 64, 128 or 256");
#pragma unroll 1
        for (int c = 0; c < BN / 32; c += 2) {
          float v0[32], v1[32];
          tmem_ld32x2(tb + c * 32, tb + (c + 1) * 32, v0, v1);
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            pk[i] = args.bf16 ? Pack2<__nv_bfloat16>::pack(v0[2 * i], v0[2 * i + 1])
                              : Pack2<__half>::pack(v0[2 * i], v0[2 * i + 1]);
            pk[16 + i] = args.bf16 ? Pack2<__nv_bfloat16>::pack(v1[2 * i], v1[2 * i + 1])
                                   : Pack2<__half>::pack(v1[2 * i], v1[2 * i + 1]);
          }
          warp_store_rows<128>(stg, pk, nvalid, gtile + size_t(t.n * BN + c * 32) * 2, pitch, lane);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(tb + c * 32, v);
          const int col0 = t.n * BN + c * 32;
          if (args.bias) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += __ldg(args.bias + col0 + i);
          }
          if (args.out_fp32) {
            warp_store_rows<128>(stg, reinterpret_cast<const uint32_t*>(v), nvalid, gtile + size_t(col0) * 4, pitch,
                                 lane);
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = args.bf16 ? Pack2<__nv_bfloat16>::pack(v[2 * i], v[2 * i + 1])
                                : Pack2<__half>::pack(v[2 * i], v[2 * i + 1]);
            warp_store_rows<64>(stg, pk, nvalid, gtile + size_t(col0) * 2, pitch, lane);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  } else if (AG && warp >= Cfg::GATHER_WARP0) {
    // ---------------- A row gather: 4 warps ----------------
    // Thread gt copies 16-byte chunk (gt % 8) of tile rows gt/8, gt/8 + 16, ...
    // of A = a_src[row_token[row]] into the 128-byte-swizzled K-major layout
    // (chunk index XOR row mod 8) that the TMA would write; rows past the
    // problem are zero-filled.  Each thread then arrives on the stage's full
    // barrier once its copies have landed.
    const int gt = threadIdx.x - Cfg::GATHER_WARP0 * 32;
    const int chunk = gt & 7;
    const int rbase = gt >> 3;
    const uint8_t* src = static_cast<const uint8_t*>(args.a_src);
    const size_t src_pitch = size_t(args.K) * 2;
    int stage = 0;
    uint32_t phase = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      TileMap t = decode_tile(L, nt, tile_start, G);
      const int a_row = goff[t.g] + t.m * BM;
      int tok[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = a_row + rbase + 16 * i;
        int tk = r < args.rows ? __ldg(args.row_token + r) : -1;
        tok[i] = (tk >= 0 && tk < args.a_src_rows) ? tk : -1;
      }
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, lim)) { ok = false; break; }
        const uint32_t dst0 = smem_u32(smA(stage));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = rbase + 16 * i;
          const uint32_t dst = dst0 + uint32_t(r * 128 + ((chunk ^ (r & 7)) << 4));
          const uint8_t* g = src + (tok[i] >= 0 ? size_t(tok[i]) * src_pitch + size_t(kb) * 128 + chunk * 16 : 0);
          cp_async_16_zfill(dst, g, tok[i] >= 0 ? 16u : 0u);
        }
        cp_async_arrive_noinc(&full_bar[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // every copy has landed before the CTA exits
  } else if (WQ && warp < Cfg::GATHER_WARP0) {
    // ---------------- AWQ dequantisation: warps 6..13 ----------------
    // Thread (wc, r0) turns code word column wc (output columns 8wc..8wc+7)
    // of K rows r0, r0 + RP, ... into one 16-byte chunk of the MN-major B tile
    // per row.
    const int dt = threadIdx.x - kBaseThreads;
    const int wc = dt % WC;
    const int r0 = dt / WC;
    constexpr int RP = kDequantThreads / WC;  // rows per pass
    const int half = (EPI == EPI_SWIGLU && wc >= W2) ? 1 : 0;
    const int wl = wc - half * W2;
    const uint32_t chunk = uint32_t(wc & 7);
    const uint32_t atom_off = uint32_t(wc >> 3) * Cfg::B_LBO;
    // packed copy: the unit and its word holding the thread's word column
    // (a gate/up unit holds 8 gate then 8 up words of one 64-column block)
    const bool packed = args.awq_packed != nullptr;
    const int pu = EPI == EPI_SWIGLU ? wl >> 3 : wc >> 4;
    const int pw = EPI == EPI_SWIGLU ? (wl & 7) + 8 * half : wc & 15;
    int stage = 0;
    uint32_t phase = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status, lim)) { L = total; break; }
        constexpr int NR = BK / RP;
        if constexpr (BN >= 128) {  // the packed copy serves 128- and 256-column tiles
        if (packed) {
          // unit layout: codes [r % 16][word][r / 16], scales [group][128], zeros [group][16 words]
          const uint8_t* ub = reinterpret_cast<const uint8_t*>(smCodes(stage, 0)) + pu * kAwqUnit;
          const uint4 s0 = *reinterpret_cast<const uint4*>(ub + 4096 + (8 * pw) * 2);
          const uint4 s1 = *reinterpret_cast<const uint4*>(ub + 4096 + (128 + 8 * pw) * 2);
          const uint32_t z0 = *reinterpret_cast<const uint32_t*>(ub + 4608 + pw * 4);
          const uint32_t z1 = *reinterpret_cast<const uint32_t*>(ub + 4608 + (16 + pw) * 4);
          uint8_t* btile = smB(stage) + atom_off;
          // rows r0 + 16 i' of the word are one 16-byte piece of the unit:
          // RP = 16 -> one piece (rows r0 + 16 i), RP = 8 -> two (rows r0 and
          // r0 + 8 onwards, interleaved); a warp's pieces are consecutive
          static_assert(RP == 8 || RP == 16, "packed rows per pass: 256- or 128-column tiles");
          uint32_t cw[NR];
          {
            const uint4 a = *reinterpret_cast<const uint4*>(ub + (r0 * 16 + pw) * 16);
            if constexpr (RP == 16) {
              cw[0] = a.x;
              cw[1] = a.y;
              cw[2] = a.z;
              cw[3] = a.w;
            } else {
              const uint4 b = *reinterpret_cast<const uint4*>(ub + ((r0 + 8) * 16 + pw) * 16);
              cw[0] = a.x;
              cw[1] = b.x;
              cw[2] = a.y;
              cw[3] = b.y;
              cw[4] = a.z;
              cw[5] = b.z;
              cw[6] = a.w;
              cw[7] = b.w;
            }
          }
          const AwqGroup g0 = awq_group_paired<WQ == W_AWQ_BF16>(z0, s0),
                         g1 = awq_group_paired<WQ == W_AWQ_BF16>(z1, s1);
#pragma unroll
          for (int i = 0; i < NR; ++i) {
            const int r = r0 + i * RP;
            const uint4 v = awq_dequant8_paired<WQ == W_AWQ_BF16>(cw[i], r < 32 ? g0 : g1);
            const uint32_t off =
                uint32_t(r >> 3) * Cfg::B_SBO + uint32_t(r & 7) * 128 + ((chunk ^ uint32_t(r & 7)) << 4);
            *reinterpret_cast<uint4*>(btile + off) = v;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bready_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
          continue;
        }
        }
        const uint32_t* codes = smCodes(stage, half) + wl;
        const uint16_t* sc = smScales(stage, half) + wl * 8;
        const uint32_t* zr = smZeros(stage, half) + wl;
        const uint4 s0 = *reinterpret_cast<const uint4*>(sc);
        const uint4 s1 = *reinterpret_cast<const uint4*>(sc + W2 * 8);
        const uint32_t z0 = zr[0], z1 = zr[W2];
        uint8_t* btile = smB(stage) + atom_off;
        // the thread's code words first (loads before any store, so that the
        // rows' conversions overlap), then convert and store
        uint32_t cw[NR];
#pragma unroll
        for (int i = 0; i < NR; ++i) cw[i] = codes[(r0 + i * RP) * W2];
        const AwqGroup g0 = awq_group<WQ == W_AWQ_BF16>(z0, s0), g1 = awq_group<WQ == W_AWQ_BF16>(z1, s1);
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const int r = r0 + i * RP;
          const uint4 v = awq_dequant8<WQ == W_AWQ_BF16>(cw[i], r < 32 ? g0 : g1);
          const uint32_t off = uint32_t(r >> 3) * Cfg::B_SBO + uint32_t(r & 7) * 128 + ((chunk ^ uint32_t(r & 7)) << 4);
          *reinterpret_cast<uint4*>(btile + off) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bready_bar[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

// 2-D tensor map of a row-major [rows, cols] matrix of `esize`-byte elements,
// box [box_rows, box_cols].
int make_tmap_2d(CUtensorMap* map, const void* base, int rows, int cols, int esize, int box_rows, int box_cols,
                 CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encode_fn();
  MOE_REQUIRE(enc != nullptr, MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  MOE_REQUIRE((reinterpret_cast<uintptr_t>(base) & 15) == 0, MOE_ERR_INVALID_ARG, "operand is not 16-byte aligned");
  MOE_REQUIRE((size_t(cols) * esize) % 16 == 0, MOE_ERR_UNSUPPORTED, "row pitch of %d bytes is not a multiple of 16",
              cols * esize);
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols) * esize};
  cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMapDataType dt = esize == 4 ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                      : (esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8);
  CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  MOE_REQUIRE(r == CUDA_SUCCESS, MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for a [%d, %d] operand, box [%d, %d]",
              int(r), rows, cols, box_rows, box_cols);
  return MOE_OK;
}


// 2-D tensor map of a row-major [rows, cols] 16-bit matrix, box [box_rows, 64]
// with the 128-byte swizzle (the K-major UMMA operand layout).
int make_tmap_16bit_sw128(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  return make_tmap_2d(map, base, rows, cols, 2, box_rows, 64, CU_TENSOR_MAP_SWIZZLE_128B);
}

// 2-D tensor map of a row-major [rows, cols_bytes] byte matrix (packed FP4),
// box [box_rows, 128 bytes] with the 128-byte swizzle.
int make_tmap_2d_u8_sw128(CUtensorMap* map, const void* base, int rows, int cols_bytes, int box_rows) {
  return make_tmap_2d(map, base, rows, cols_bytes, 1, box_rows, 128, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int BN, int EPI, int WQ, int AG>
static int launch_bn(const CUtensorMap& ta, const BMaps& bmaps, const GemmArgs& args, cudaStream_t stream) {
  using Cfg = GemmCfg<BN, EPI, WQ, AG>;
  static bool attr_set[64] = {false};  // per device
  auto kern = k_grouped_gemm<BN, EPI, WQ, AG>;
  int dev = 0;
  MOE_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev >= 64 || !attr_set[dev]) {
    MOE_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
    if (dev < 64) attr_set[dev] = true;
  }
  kern<<<num_sms(), Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(ta, bmaps, args);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}

template <int WQ, int AG>
static int dispatch(const CUtensorMap& ta, const BMaps& bm, const GemmArgs& args, int epi, int bn,
                    cudaStream_t stream) {
  if (epi == EPI_SWIGLU) {
    if (bn == 256) return launch_bn<256, EPI_SWIGLU, WQ, AG>(ta, bm, args, stream);
    if (bn == 128) return launch_bn<128, EPI_SWIGLU, WQ, AG>(ta, bm, args, stream);
    return launch_bn<64, EPI_SWIGLU, WQ, AG>(ta, bm, args, stream);
  }
  if (bn == 256) return launch_bn<256, EPI_STORE, WQ, AG>(ta, bm, args, stream);
  if (bn == 128) return launch_bn<128, EPI_STORE, WQ, AG>(ta, bm, args, stream);
  return launch_bn<64, EPI_STORE, WQ, AG>(ta, bm, args, stream);
}

static int check_common(const GemmArgs& args, int epi, int bn) {
  MOE_REQUIRE(args.K % BK == 0 && args.K > 0, MOE_ERR_UNSUPPORTED, "GEMM K=%d is not a positive multiple of 64",
              args.K);
  MOE_REQUIRE(args.G >= 1 && args.G <= kGemmMaxGroups, MOE_ERR_UNSUPPORTED, "GEMM group count %d outside [1, %d]",
              args.G, kGemmMaxGroups);
  MOE_REQUIRE(bn == 64 || bn == 128 || bn == 256, MOE_ERR_INVALID_ARG, "tile width %d", bn);
  const int bnh = epi == EPI_SWIGLU ? bn / 2 : bn;
  MOE_REQUIRE(args.n_out % bnh == 0, MOE_ERR_UNSUPPORTED, "output width %d is not a multiple of the tile (%d)",
              args.n_out, bnh);
  return MOE_OK;
}

int launch_grouped_gemm(const void* A, int a_rows, const void* B, int b_rows_total, const GemmArgs& args, int epi,
                        int bn, cudaStream_t stream) {
  int rc = check_common(args, epi, bn);
  if (rc) return rc;
  if (a_rows == 0) return MOE_OK;
  const int bnh = epi == EPI_SWIGLU ? bn / 2 : bn;
  CUtensorMap ta;
  BMaps bm;
  memset(&bm, 0, sizeof(bm));
  if (args.row_token) {
    // A rows are gathered in the kernel; the map over the source only keeps the parameter valid
    MOE_REQUIRE(args.a_src != nullptr && args.a_src_rows > 0, MOE_ERR_INVALID_ARG, "gathered GEMM without a source");
    MOE_REQUIRE((reinterpret_cast<uintptr_t>(args.a_src) & 15) == 0, MOE_ERR_INVALID_ARG,
                "gathered rows are not 16-byte aligned");
    rc = make_tmap_16bit_sw128(&ta, args.a_src, args.a_src_rows, args.K, BM);
  } else {
    rc = make_tmap_16bit_sw128(&ta, A, a_rows, args.K, BM);
  }
  if (rc) return rc;
  rc = make_tmap_16bit_sw128(&bm.b, B, b_rows_total, args.K, bnh);
  if (rc) return rc;
  if (args.row_token) return dispatch<W_DENSE, 1>(ta, bm, args, epi, bn, stream);
  return dispatch<W_DENSE, 0>(ta, bm, args, epi, bn, stream);
}

int launch_grouped_gemm_awq(const void* A, int a_rows, const int32_t* qweight, const int32_t* qzeros,
                            const void* scales, int n_total, const GemmArgs& args_in, int epi, int bn,
                            cudaStream_t stream, const void* awq_packed) {
  GemmArgs args = args_in;
  // the packed units are 128 columns wide: tile widths 128 and 256 read them
  args.awq_packed = (awq_packed && bn >= 128) ? static_cast<const uint8_t*>(awq_packed) : nullptr;
  int rc = check_common(args, epi, bn);
  if (rc) return rc;
  MOE_REQUIRE(args.K % 32 == 0, MOE_ERR_UNSUPPORTED, "AWQ K=%d is not a multiple of the group size 32", args.K);
  if (a_rows == 0) return MOE_OK;
  const int bnh = epi == EPI_SWIGLU ? bn / 2 : bn;
  MOE_REQUIRE(bnh % 32 == 0, MOE_ERR_UNSUPPORTED, "AWQ tile half-width %d is not a multiple of 32", bnh);
  CUtensorMap ta;
  BMaps bm;
  memset(&bm, 0, sizeof(bm));
  if (args.row_token) {
    // A rows gathered in the kernel (x[row_token[r]]); the map over the source only keeps the parameter valid
    MOE_REQUIRE(args.a_src != nullptr && args.a_src_rows > 0, MOE_ERR_INVALID_ARG, "gathered GEMM without a source");
    MOE_REQUIRE((reinterpret_cast<uintptr_t>(args.a_src) & 15) == 0, MOE_ERR_INVALID_ARG,
                "gathered rows are not 16-byte aligned");
    rc = make_tmap_16bit_sw128(&ta, args.a_src, args.a_src_rows, args.K, BM);
  } else {
    rc = make_tmap_16bit_sw128(&ta, A, a_rows, args.K, BM);
  }
  if (rc) return rc;
  const int G = args.G;
  rc = make_tmap_2d(&bm.codes, qweight, G * args.K, n_total / 8, 4, BK, bnh / 8, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  rc = make_tmap_2d(&bm.scales, scales, G * (args.K / 32), n_total, 2, 2, bnh, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  rc = make_tmap_2d(&bm.zeros, qzeros, G * (args.K / 32), n_total / 8, 4, 2, bnh / 8, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  if (args.row_token) {
    if (args.bf16) return dispatch<W_AWQ_BF16, 1>(ta, bm, args, epi, bn, stream);
    return dispatch<W_AWQ, 1>(ta, bm, args, epi, bn, stream);
  }
  if (args.bf16) return dispatch<W_AWQ_BF16, 0>(ta, bm, args, epi, bn, stream);
  return dispatch<W_AWQ, 0>(ta, bm, args, epi, bn, stream);
}

}  // namespace moe
