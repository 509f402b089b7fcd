// Routed + shared SwiGLU experts for the smallest batches (T <= 16): one
// weight-streaming kernel whose work items do not depend on one another.
//
// A work item is (group g, block j of 64 intermediate features); group E is
// the shared expert (all T tokens), groups 0..E-1 the routed experts.
//   Phase A: the item's 64 gate rows and the matching 64 up rows against the
//     group's tokens (weights are the MMA's M operand, the at most 16 tokens
//     its N operand), SwiGLU in the epilogue, and the 16-bit h[:, 64j..64j+64)
//     of the group's rows written into a shared-memory tile in the operand
//     layout of the next MMA.
//   Phase B: that h slice times the matching 64 columns of the group's down
//     projection (H x 64, as blocks of 128 rows): a split-K slice of the
//     second GEMM, whose FP32 result is the partial P[j][row][0..H).
// Phase B's weights do not depend on h, so they stream right behind phase
// A's and the whole call is one stream of weights through every SM, with no
// wait between GEMM1 and GEMM2.  A second kernel sums the I/64 partials of
// every row in a fixed order (deterministic) into f (routed rows) and
// shared_out (shared rows).
//
// Weight formats (template parameter WQ):
//   WQ = 0: 16-bit routed and shared weights, output-major [N, K]; each
//     64-wide K sub-tile of 128 weight rows arrives by TMA in the K-major
//     128-byte swizzled layout the MMA reads.
//   WQ = 1: routed experts in AWQ W4A16 g32 (input-major codes, zero points
//     and FP16 scales, FP16 activations), the shared expert 16-bit as above.
//     The producer stages each routed sub-tile's codes, scales and zero
//     points (4.6 KB instead of 16 KB of FP16): from the tile-packed copy of
//     the weights (awq.cu) with one bulk copy per sub-tile when the caller
//     provides it, else with six TMA boxes from the checkpoint layout; eight dequantisation warps
//     expand it, exactly (fp16_rn((q - z) * s)), into an MN-major swizzled
//     FP16 tile, and the MMA reads that.
//   WQ = 2: the same in the BF16 mode (BF16 activations and shared expert;
//     the FP16 scales rounded to BF16, bf16_rn((q - z) * s) tiles).
//
// Warp roles: 0 TMA producer, 1 UMMA issuer (TMEM owner), 2..5 epilogue,
// 6..9 token gather (cp.async, arriving on the stage's barrier), 10..17 AWQ
// dequantisation (WQ = 1, 2).  TMEM: two 16-column phase-A accumulators
// (columns 0..31) and one phase-B accumulator of H/128 blocks x 16 columns
// (from column 32).
#include "common.cuh"
#include "gemm_sm100.cuh"

namespace moe {

int make_tmap_16bit_sw128(CUtensorMap* map, const void* base, int rows, int cols, int box_rows);
int make_tmap_2d(CUtensorMap* map, const void* base, int rows, int cols, int esize, int box_rows, int box_cols,
                 CUtensorMapSwizzle swz);

constexpr int kFusedMaxT = 16;

namespace {

constexpr int BM = 128;                    // weight rows per MMA (M)
constexpr int BK = 64;                     // K per sub-tile (one 128-byte swizzle row)
constexpr int NT = 16;                     // token columns (N) of every MMA
constexpr int A_BYTES = BM * BK * 2;       // 16 KB of 16-bit weights per sub-tile
constexpr int B_BYTES = NT * BK * 2;       // 2 KB of tokens per sub-tile
constexpr int KSUB = 2;                    // sub-tiles per pipeline stage
constexpr int H_BYTES = NT * BK * 2;       // one h tile: 16 rows x 64 features
constexpr int XS = NT + 1;                 // floats per row of the accumulator exchange (bank padding)
constexpr int XCHG_BYTES = BM * XS * 4;    // all 128 phase-A rows (64 gate, 64 up)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACCB_COL = 32;
constexpr int FULL_ARRIVALS = 1 + 128;     // producer (with the TMA bytes) + one per gather thread
// AWQ staging inside a sub-tile, after the FP16 weight tile and the token
// tile: codes [64 K rows][16 words] (phase A: gate box [64][8] then up box
// [64][8]; phase B: one box [64][16]), scales [2 groups][128] FP16 (phase A:
// two boxes [2][64]), zero points [2 groups][16 words] (phase A: two boxes
// [2][8], each in a 128-byte slot).  Every box starts on 128 bytes.
constexpr int Q_CODES = A_BYTES + B_BYTES;
constexpr int Q_SCALES = Q_CODES + 64 * 16 * 4;
constexpr int Q_ZEROS = Q_SCALES + 2 * 128 * 2;
constexpr int Q_END = Q_ZEROS + 2 * 128;
constexpr uint32_t Q_TX = 64 * 16 * 4 + 2 * 128 * 2 + 2 * 16 * 4;  // bytes the TMA brings per AWQ sub-tile
constexpr int kAwqUnitBytes = 4736;  // one tile-packed AWQ unit (awq.cu): codes, scales, zeros of a sub-tile
static_assert(Q_TX == kAwqUnitBytes && Q_SCALES == Q_CODES + 4096 && Q_ZEROS == Q_SCALES + 512,
              "a packed AWQ unit is the sub-tile's staging image");
// MN-major FP16 weight tile (AWQ): 64-element atoms along M are LBO apart,
// 8-row K groups SBO apart; one MMA (K = 16) spans two K groups
constexpr uint32_t AQ_LBO = (BK / 8) * 1024;
constexpr uint32_t AQ_SBO = 1024;
constexpr int kDequantThreads = 256;  // two dequantisation warps per SM sub-partition

template <int WQ>
struct FusedCfg {
  static constexpr int SUB_BYTES = WQ ? (Q_END + 1023) / 1024 * 1024 : A_BYTES + B_BYTES;
  static constexpr int STAGE_BYTES = KSUB * SUB_BYTES;
  static constexpr int STAGES = WQ ? 4 : 5;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 2 * H_BYTES + XCHG_BYTES;
  static constexpr int THREADS = 320 + (WQ ? kDequantThreads : 0);
  static_assert(SUB_BYTES % 1024 == 0 && H_BYTES % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(SMEM_BYTES <= 222 * 1024, "shared memory");
};
static_assert(Q_CODES % 1024 == 0 && Q_SCALES % 128 == 0 && Q_ZEROS % 128 == 0, "TMA destinations");

struct Args {
  const int* offsets;   // [E+1] routed expert offsets (device)
  int E, rows, T, H, I;
  const int* row_token; // [rows] token of each routed row
  const void* x;        // [T, H] 16-bit tokens
  float* partial;       // [I/64][rows + T][H] FP32
  const uint8_t* qpack; // AWQ: tile-packed routed weights (awq.cu layout), or null (TMA from qc/qs/qz)
  int bf16;
  int* status;
  unsigned long long limit_ns;
};

// Tensor maps.  16-bit weights: gu (routed gate/up [E*2I, H], box 64 rows),
// d (routed down [E*H, I], box 128 rows), and the shared expert's sgu, sd.
// AWQ (WQ = 1) replaces gu and d by codes / scales / zero points.
struct Maps {
  CUtensorMap gu, d, sgu, sd;
  CUtensorMap qc_gu, qs_gu, qz_gu, qc_d, qs_d, qz_d;
};

__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void epilogue_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// the four epilogue warps agree on one flag (true only if every thread passes true)
__device__ __forceinline__ bool epilogue_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v))
      : "memory");
  return r != 0;
}

template <int WQ>
__global__ void __launch_bounds__(FusedCfg<WQ>::THREADS, 1)
    k_decode_ffn(const __grid_constant__ Maps maps, const Args args) {
  using Cfg = FusedCfg<WQ>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES], aready_bar[STAGES], empty_bar[STAGES], accA_full[2],
      accA_empty[2], h_full[2], h_empty[2], accB_full, accB_empty, drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int goff[kGemmMaxGroups + 2];
  __shared__ int item_start[kGemmMaxGroups + 2];
  __shared__ int warp_sums[Cfg::THREADS / 32];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // sub-tile u of stage s: weights at sub(s, u), tokens at + A_BYTES, AWQ staging at + Q_CODES ...
  auto sub = [&](int s, int u) { return smem + s * Cfg::STAGE_BYTES + u * Cfg::SUB_BYTES; };
  uint8_t* htile = smem + STAGES * Cfg::STAGE_BYTES;  // two h tiles of H_BYTES
  float* xchg = reinterpret_cast<float*>(htile + 2 * H_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E, G = E + 1;
  const int MB1 = args.I / BK;        // items per group
  const int KA = args.H / BK;         // phase-A sub-tiles per item
  const int NSA = KA / KSUB;          // phase-A stages per item (H % 128 == 0)
  const int MB2 = args.H / BM;        // phase-B sub-tiles (blocks of 128 down-projection rows)
  const int NSB = (MB2 + KSUB - 1) / KSUB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], FULL_ARRIVALS);
      mbar_init(&aready_bar[s], kDequantThreads);
      mbar_init(&empty_bar[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accA_full[i], 1);
      mbar_init(&accA_empty[i], 128);
      mbar_init(&h_full[i], 128);
      mbar_init(&h_empty[i], 1);
    }
    mbar_init(&accB_full, 1);
    mbar_init(&accB_empty, 128);
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.sgu);
    tma_prefetch_desc(&maps.sd);
    if (WQ) {
      tma_prefetch_desc(&maps.qc_gu);
      tma_prefetch_desc(&maps.qs_gu);
      tma_prefetch_desc(&maps.qz_gu);
      tma_prefetch_desc(&maps.qc_d);
      tma_prefetch_desc(&maps.qs_d);
      tma_prefetch_desc(&maps.qz_d);
    } else {
      tma_prefetch_desc(&maps.gu);
      tma_prefetch_desc(&maps.d);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  // the h tiles start as zeros (their token columns past a group's rows are
  // never written)
  for (int i = threadIdx.x; i < 2 * H_BYTES / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(htile)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  // launched as a programmatic dependent: the routing comes from the kernel before
  griddep_wait();
  griddep_launch_dependents();
  for (int i = threadIdx.x; i <= E; i += blockDim.x) goff[i] = args.offsets[i];
  __syncthreads();
  auto group_rows = [&](int g, int& r0, int& n) {
    if (g < E) {
      r0 = goff[g];
      n = goff[g + 1] - goff[g];
    } else {
      r0 = args.rows;
      n = args.T;
    }
  };
  {  // item_start[g]: first item of group g (every group with rows has MB1 items)
    const int per = (G + blockDim.x - 1) / blockDim.x;
    const int g0 = threadIdx.x * per;
    int local = 0;
    for (int g = g0; g < g0 + per && g < G; ++g) {
      int r0, n;
      group_rows(g, r0, n);
      local += n > 0 ? MB1 : 0;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int run = incl - local;
    for (int w = 0; w < warp; ++w) run += warp_sums[w];
    for (int g = g0; g < g0 + per && g < G; ++g) {
      item_start[g] = run;
      int r0, n;
      group_rows(g, r0, n);
      run += n > 0 ? MB1 : 0;
    }
    if (threadIdx.x == blockDim.x - 1) item_start[G] = run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  const int total = item_start[G];
  int* status = args.status;
  const unsigned long long lim = args.limit_ns;
  auto group_of = [&](int L) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (item_start[mid] <= L) lo = mid; else hi = mid - 1;
    }
    return lo;
  };

  if (warp == 0) {
    // ---------------- TMA producer: phase-A then phase-B weights of every item ----------------
    // Lane 0 owns the stage barriers; the copies of a stage (up to 12) are
    // issued together, one per lane, in the same instructions: a copy costs
    // its issuing thread on the order of a hundred cycles.
    const uint64_t pol = l2_policy_evict_first();  // read once per call
    const int I = args.I, H = args.H;
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
      const int g = group_of(L);
      const int j = L - item_start[g];
      const bool q = WQ && g < E;  // AWQ routed expert
      for (int st = 0; st < NSA + NSB; ++st) {
        if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, lim);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const bool pa = st < NSA;
        const int m0 = pa ? 0 : (st - NSA) * KSUB;
        const int nsub = pa ? KSUB : min(KSUB, MB2 - m0);
        if (lane == 0)
          mbar_arrive_expect_tx(&full_bar[stage], uint32_t(nsub) * (q ? Q_TX : uint32_t(A_BYTES)));
        __syncwarp();
        // copy `lane` of the stage: per sub-tile 1 (packed AWQ), 6 (AWQ
        // phase A), 3 (AWQ phase B), 2 (16-bit phase A) or 1 (16-bit phase B)
        const int per = q ? (args.qpack ? 1 : (pa ? 6 : 3)) : (pa ? 2 : 1);
        const int u = lane / per, which = lane - u * per;
        if (u < nsub) {
          uint8_t* d = sub(stage, u);
          uint64_t* fb = &full_bar[stage];
          if (q && args.qpack) {
            // the sub-tile's packed unit: gate/up (j, kt) or down (j, m) of expert g
            const int J = I / BK, nka = H / BK, nkb = H / BM;
            const size_t unit = pa ? size_t(j) * nka + size_t(st * KSUB + u)
                                   : size_t(J) * nka + size_t(j) * nkb + size_t(m0 + u);
            bulk_load(d + Q_CODES, args.qpack + (size_t(g) * J * (nka + nkb) + unit) * kAwqUnitBytes, Q_TX, fb);
          } else if (pa) {
            const int kx = (st * KSUB + u) * BK;
            if (q) {
              // gate columns 64j.., up columns I + 64j.. of the input-major codes
              const int crow = g * H + kx, grow = g * (H / 32) + kx / 32;
              const int half = which & 1, kind = which >> 1;  // kind 0 codes, 1 scales, 2 zeros
              const int c8 = half ? I / 8 + j * 8 : j * 8;
              if (kind == 0) tma_load_2d_hint(d + Q_CODES + half * 2048, &maps.qc_gu, fb, c8, crow, pol);
              else if (kind == 1) tma_load_2d_hint(d + Q_SCALES + half * 256, &maps.qs_gu, fb, c8 * 8, grow, pol);
              else tma_load_2d_hint(d + Q_ZEROS + half * 128, &maps.qz_gu, fb, c8, grow, pol);
            } else {
              const CUtensorMap* gu = g < E ? &maps.gu : &maps.sgu;
              const int base = g < E ? g * 2 * I : 0;
              tma_load_2d_hint(d + which * 64 * BK * 2, gu, fb, kx, base + which * I + j * 64, pol);
            }
          } else {
            const int m = m0 + u;
            if (q) {
              const int crow = g * I + j * BK, grow = g * (I / 32) + j * 2;
              if (which == 0) tma_load_2d_hint(d + Q_CODES, &maps.qc_d, fb, m * 16, crow, pol);
              else if (which == 1) tma_load_2d_hint(d + Q_SCALES, &maps.qs_d, fb, m * BM, grow, pol);
              else tma_load_2d_hint(d + Q_ZEROS, &maps.qz_d, fb, m * 16, grow, pol);
            } else {
              const CUtensorMap* dn = g < E ? &maps.d : &maps.sd;
              tma_load_2d_hint(d, dn, fb, j * BK, (g < E ? g * H : 0) + m * BM, pol);
            }
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok && lane == 0) {  // let the loads in flight land before the block exits
      volatile int never = 0;
      for (long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
        mbar_wait(&full_bar[i % STAGES], uint32_t((i / STAGES) & 1), &never, nullptr, lim);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer ----------------
      // 16-bit weights: K-major A; AWQ: the dequantised MN-major A (bit 15)
      const uint32_t idesc_k = idesc_f16(args.bf16, BM, NT);
      const uint32_t idesc_q = idesc_k | (1u << 15);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int n = 0;  // items of this CTA so far
      // the stage's operands are complete: TMA + tokens (full), or after dequantisation (aready)
      auto wait_operands = [&](int s) {
        return mbar_wait(WQ ? &aready_bar[s] : &full_bar[s], phase, &abort_flag, status, lim);
      };
      auto adesc = [&](const uint8_t* tile, bool q, int kk) {
        return q ? sdesc_mnmajor_sw128(smem_u32(tile), AQ_LBO, AQ_SBO) + uint64_t(kk * (2 * AQ_SBO >> 4))
                 : sdesc_kmajor_sw128(smem_u32(tile)) + uint64_t(kk * 2);
      };
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++n) {
        const int g = group_of(L);
        const bool q = WQ && g < E;
        const uint32_t idesc = q ? idesc_q : idesc_k;
        const int a = n & 1;                     // phase-A accumulator and h tile of this item
        const uint32_t pa = uint32_t((n >> 1) & 1);  // their phase parity
        // phase A: D_A[weight row, token] over K = H
        if (!mbar_wait(&accA_empty[a], pa ^ 1, &abort_flag, status, lim)) break;
        tc_fence_after();
        const uint32_t dA = tmem_base + uint32_t(a * NT);
        for (int st = 0; st < NSA; ++st) {
          if (!wait_operands(stage)) { ok = false; break; }
          tc_fence_after();
          for (int u = 0; u < KSUB; ++u) {
            const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sub(stage, u) + A_BYTES));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_f16(dA, adesc(sub(stage, u), q, kk), bd + uint64_t(kk * 2), idesc, (st | u | kk) != 0);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&accA_full[a]);
        // phase B: D_B[down row, token] = W_d[:, 64j..64j+64) h[:, 64j..64j+64)^T, one
        // 16-column accumulator per block of 128 down-projection rows
        if (!mbar_wait(&h_full[a], pa, &abort_flag, status, lim)) break;
        if (!mbar_wait(&accB_empty, uint32_t(n & 1) ^ 1, &abort_flag, status, lim)) break;
        tc_fence_after();
        const uint64_t hd = sdesc_kmajor_sw128(smem_u32(htile + a * H_BYTES));
        for (int st = 0; st < NSB; ++st) {
          const int m0 = st * KSUB;
          const int nsub = min(KSUB, MB2 - m0);
          if (!wait_operands(stage)) { ok = false; break; }
          tc_fence_after();
          for (int u = 0; u < nsub; ++u) {
            const uint32_t dB = tmem_base + ACCB_COL + uint32_t((m0 + u) * NT);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_f16(dB, adesc(sub(stage, u), q, kk), hd + uint64_t(kk * 2), idesc, kk != 0);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&accB_full);
        umma_commit(&h_empty[a]);
      }
      umma_commit(&drain_bar);
      volatile int never = 0;
      mbar_wait(&drain_bar, 0, &never, nullptr, lim);
    }
  } else if (warp < 6) {
    // ---------------- epilogue ----------------
    // TMEM lane quadrant q: in phase A lanes 0..63 hold the gate rows, 64..127
    // the up rows of the same 64 intermediate features; in phase B lane =
    // down-projection row (output feature) m*128 + q*32 + lane.
    const int q = warp & 3;
    const int R = args.rows + args.T;
    int n = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++n) {
      const int g = group_of(L);
      const int j = L - item_start[g];
      int r0, nr;
      group_rows(g, r0, nr);
      if (nr > NT && warp == 2 && lane == 0) report(status, MOE_ERR_UNSUPPORTED);  // more rows than the token tile
      const int nn = min(nr, NT);
      const int a = n & 1;
      const uint32_t pa = uint32_t((n >> 1) & 1);
      // a timed-out wait in one warp must not leave the others at a named barrier
      bool ok = mbar_wait(&accA_full[a], pa, &abort_flag, status, lim);
      ok = ok && mbar_wait(&h_empty[a], pa ^ 1, &abort_flag, status, lim);
      if (!epilogue_all(ok)) break;
      tc_fence_after();
      float v[NT];
      tmem_ld16(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(a * NT), v);
      tc_fence_before();
      mbar_arrive(&accA_empty[a]);
      // rows 0..63 gate, 64..127 up pre-activations of the block's 64 features
#pragma unroll
      for (int c = 0; c < NT; ++c)
        if (c < nn) xchg[(q * 32 + lane) * XS + c] = v[c];
      epilogue_sync();
      {
        // h[c][f] = silu(gate[f][c]) * up[f][c], 16-bit, K-major 128-byte
        // swizzled: row c at c*128 bytes, 16-byte chunk (f/8) xor (c%8),
        // element f%8.  64 * nn values over the 128 threads, in a rolled loop
        // (this code runs once per item: compact code stays cached).  Token
        // columns c >= nn keep zeros or an earlier item's values: they feed
        // only accumulator columns that are never read.
        const int et = threadIdx.x - 64;
        uint8_t* ht = htile + a * H_BYTES;
#pragma unroll 1
        for (int idx = et; idx < 64 * nn; idx += 128) {
          const int f = idx & 63, c = idx >> 6;
          const float h = silu_f(xchg[f * XS + c]) * xchg[(64 + f) * XS + c];
          const uint32_t off = uint32_t(c * 128 + (((f >> 3) ^ (c & 7)) << 4) + (f & 7) * 2);
          if (args.bf16)
            *reinterpret_cast<__nv_bfloat16*>(ht + off) = __float2bfloat16_rn(h);
          else
            *reinterpret_cast<__half*>(ht + off) = __float2half_rn(h);
        }
      }
      fence_proxy_async_smem();  // the h tile is read by the tensor cores
      mbar_arrive(&h_full[a]);
      epilogue_sync();           // every thread has read xchg before the next item overwrites it
      // phase B: FP32 partials of the group's rows
      if (!epilogue_all(mbar_wait(&accB_full, uint32_t(n & 1), &abort_flag, status, lim))) break;
      tc_fence_after();
      float* P = args.partial + (size_t(j) * R + r0) * args.H + q * 32 + lane;
      const size_t H = size_t(args.H);
      const uint32_t tq = tmem_base + (uint32_t(q * 32) << 16) + ACCB_COL;
      // the accumulators' first nn columns, many blocks per TMEM load wait
      // (a load's latency is paid once per batch): 16 blocks x 4 columns, 8 x
      // 8, or 4 x 16 (addresses of blocks past the last clamped to it); the
      // AWQ kernels (fewer registers per thread) 8 x 4 or 2 x 16
      if (nn <= 4) {
        // 16 blocks per wait; 8 in the AWQ kernels, whose 576 threads have
        // fewer registers each
        constexpr int NB = WQ ? 8 : 16;
        for (int m0 = 0; m0 < MB2; m0 += NB) {
          uint32_t ta[NB], v[NB * 4];
#pragma unroll
          for (int b = 0; b < NB; ++b) ta[b] = tq + uint32_t(min(m0 + b, MB2 - 1) * NT);
          if constexpr (WQ) tmem_ld_8x4(ta, v); else tmem_ld_16x4(ta, v);
#pragma unroll
          for (int b = 0; b < NB; ++b)
            if (m0 + b < MB2)
#pragma unroll
              for (int c = 0; c < 4; ++c)
                if (c < nn) P[size_t(c) * H + size_t(m0 + b) * BM] = __uint_as_float(v[b * 4 + c]);
        }
      } else if (WQ) {
        for (int m0 = 0; m0 < MB2; m0 += 2) {
          float w0[32];
          tmem_ld32(tq + uint32_t(m0 * NT), w0);
#pragma unroll
          for (int u = 0; u < 2; ++u)
            if (m0 + u < MB2)
#pragma unroll
              for (int c = 0; c < NT; ++c)
                if (c < nn) P[size_t(c) * H + size_t(m0 + u) * BM] = w0[u * NT + c];
        }
      } else if (nn <= 8) {
        for (int m0 = 0; m0 < MB2; m0 += 8) {
          uint32_t ta[8], v[64];
#pragma unroll
          for (int b = 0; b < 8; ++b) ta[b] = tq + uint32_t(min(m0 + b, MB2 - 1) * NT);
          tmem_ld_8x8(ta, v);
#pragma unroll
          for (int b = 0; b < 8; ++b)
            if (m0 + b < MB2)
#pragma unroll
              for (int c = 0; c < 8; ++c)
                if (c < nn) P[size_t(c) * H + size_t(m0 + b) * BM] = __uint_as_float(v[b * 8 + c]);
        }
      } else {
        for (int m0 = 0; m0 < MB2; m0 += 4) {
          float w0[32], w1[32];
          // blocks m0, m0+1 and m0+2, m0+3 (32 columns each); MB2 <= 28 keeps
          // the reads past an odd last block inside the allocation
          tmem_ld32x2(tq + uint32_t(m0 * NT), tq + uint32_t(min(m0 + 2, MB2 - 1) * NT), w0, w1);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (m0 + u < MB2) {
#pragma unroll
              for (int c = 0; c < NT; ++c)
                if (c < nn) P[size_t(c) * H + size_t(m0 + u) * BM] = u < 2 ? w0[u * NT + c] : w1[(u - 2) * NT + c];
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&accB_empty);
    }
  } else if (warp < 10) {
    // ---------------- token gather: warps 6..9 ----------------
    // Thread gt copies 16-byte chunk (gt % 8) of token row gt / 8 of every
    // phase-A sub-tile into the K-major swizzled token tile; rows past the
    // group's size are zero-filled.  Phase-B stages need no tokens: the
    // threads only arrive.
    const int gt = threadIdx.x - 192;
    const int ch = gt & 7;
    const int c = gt >> 3;  // 0..15
    const uint8_t* src = static_cast<const uint8_t*>(args.x);
    const size_t pitch = size_t(args.H) * 2;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
      const int g = group_of(L);
      int r0, nr;
      group_rows(g, r0, nr);
      int row = -1;
      if (c < min(nr, NT)) {
        row = g < E ? __ldg(args.row_token + r0 + c) : c;
        if (row < 0 || row >= args.T) row = -1;
      }
      const uint8_t* base = row >= 0 ? src + size_t(row) * pitch + ch * 16 : src;
      const uint32_t bytes = row >= 0 ? 16u : 0u;
      for (int st = 0; st < NSA + NSB; ++st) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, lim)) { ok = false; break; }
        if (st < NSA) {
          for (int u = 0; u < KSUB; ++u) {
            const uint32_t dst = smem_u32(sub(stage, u) + A_BYTES) + uint32_t(c * 128 + ((ch ^ (c & 7)) << 4));
            cp_async_16_zfill(dst, base + (row >= 0 ? size_t(st * KSUB + u) * 128 : 0), bytes);
          }
        }
        cp_async_arrive_noinc(&full_bar[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // every copy has landed before the block exits
  } else if (WQ) {
    // ---------------- AWQ dequantisation: warps 10..17 ----------------
    // Thread (wc, r0): code word column wc (output columns 8wc..8wc+7 of the
    // tile: phase A wc < 8 gate, wc >= 8 up; phase B the 128 down rows of the
    // block) of K rows r0, r0 + 16, r0 + 32, r0 + 48 -> one 16-byte chunk of
    // the MN-major FP16 tile per row.  Shared-expert stages (16-bit) need
    // nothing: the threads only arrive.
    constexpr int NRW = 64 / (kDequantThreads / 16);  // rows per thread per sub-tile
    const int dt = threadIdx.x - 320;
    const int wc = dt & 15;
    const int r0 = dt >> 4;  // 0..15
    const uint32_t atom_off = uint32_t(wc >> 3) * AQ_LBO;
    const uint32_t chunk = uint32_t(wc & 7);
    const bool packed = args.qpack != nullptr;
    static_assert(NRW == 4, "a packed unit holds four K rows per thread and code word");
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
      const int g = group_of(L);
      const bool q = g < E;
      for (int st = 0; st < NSA + NSB; ++st) {
        if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status, lim)) { ok = false; break; }
        const bool pa = st < NSA;
        const int nsub = pa ? KSUB : min(KSUB, MB2 - (st - NSA) * KSUB);
        if (q) {
          // phase A: box (wc / 8) of width 8 words; phase B: one box of 16
          const int half = pa ? (wc >> 3) : 0;
          const int wl = pa ? (wc & 7) : wc;
          const int cw = pa ? 8 : 16;  // code words per K row in the box
          // every staged input of the stage first (loads before any store, so
          // that the rows' conversions overlap), then convert and store
          uint32_t cv[KSUB][NRW], z[KSUB][2];
          uint4 sv[KSUB][2];
#pragma unroll
          for (int u = 0; u < KSUB; ++u) {
            if (u < nsub) {
              const uint8_t* d = sub(stage, u);
              if (packed) {
                // packed unit: this thread's four code words are adjacent; scales and
                // zeros of word wc at column wc * 8 / word wc of each group's row
                const uint4 c4 = *reinterpret_cast<const uint4*>(d + Q_CODES + (r0 * 16 + wc) * 16);
                cv[u][0] = c4.x;
                cv[u][1] = c4.y;
                cv[u][2] = c4.z;
                cv[u][3] = c4.w;
                const uint16_t* sc = reinterpret_cast<const uint16_t*>(d + Q_SCALES) + wc * 8;
                const uint32_t* zr = reinterpret_cast<const uint32_t*>(d + Q_ZEROS) + wc;
                sv[u][0] = *reinterpret_cast<const uint4*>(sc);
                sv[u][1] = *reinterpret_cast<const uint4*>(sc + 128);
                z[u][0] = zr[0];
                z[u][1] = zr[16];
              } else {
                const uint32_t* codes = reinterpret_cast<const uint32_t*>(d + Q_CODES + half * 2048) + wl;
                const uint16_t* sc = reinterpret_cast<const uint16_t*>(d + Q_SCALES + half * 256) + wl * 8;
                const uint32_t* zr = reinterpret_cast<const uint32_t*>(d + Q_ZEROS + half * 128) + wl;
#pragma unroll
                for (int i = 0; i < NRW; ++i) cv[u][i] = codes[(r0 + 16 * i) * cw];
                sv[u][0] = *reinterpret_cast<const uint4*>(sc);
                sv[u][1] = *reinterpret_cast<const uint4*>(sc + cw * 8);
                z[u][0] = zr[0];
                z[u][1] = zr[cw];
              }
            }
          }
          // the packed copy holds codes and zero points in pair order
          auto convert = [&](auto group, auto dequant) {
#pragma unroll
            for (int u = 0; u < KSUB; ++u) {
              if (u < nsub) {
                uint8_t* at = sub(stage, u) + atom_off;
                const AwqGroup g0 = group(z[u][0], sv[u][0]), g1 = group(z[u][1], sv[u][1]);
#pragma unroll
                for (int i = 0; i < NRW; ++i) {
                  const int r = r0 + 16 * i;  // rows 0..31 use group 0, 32..63 group 1
                  const uint4 v = dequant(cv[u][i], i < NRW / 2 ? g0 : g1);
                  const uint32_t off =
                      uint32_t(r >> 3) * AQ_SBO + uint32_t(r & 7) * 128 + ((chunk ^ uint32_t(r & 7)) << 4);
                  *reinterpret_cast<uint4*>(at + off) = v;
                }
              }
            }
          };
          if (packed)
            convert([](uint32_t zz, uint4 ss) { return awq_group_paired<WQ == 2>(zz, ss); },
                    [](uint32_t w, const AwqGroup& g) { return awq_dequant8_paired<WQ == 2>(w, g); });
          else
            convert([](uint32_t zz, uint4 ss) { return awq_group<WQ == 2>(zz, ss); },
                    [](uint32_t w, const AwqGroup& g) { return awq_dequant8<WQ == 2>(w, g); });
          fence_proxy_async_smem();  // the FP16 tile is read by the tensor cores
        }
        mbar_arrive(&aready_bar[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// out[r] = sum_{j < J} P[j][r] in ascending j; rows r < rows go to f (FP32
// or 16-bit), the shared rows r >= rows to shared_out (16-bit).  Grid (R,
// ceil(H / 256)) of 64-thread blocks, so that a decode batch's few rows still
// spread over many SMs; every thread issues its first kMaxJ loads (J = I/64)
// before the first addition, which then runs in ascending j.  Launched as a
// programmatic dependent of k_decode_ffn.
constexpr int kMaxJ = 16;
template <typename T16>
__global__ void __launch_bounds__(64) k_sum_partials(const float* __restrict__ P, int J, int R, int rows, int H,
                                                     void* __restrict__ f, int f_fp32, T16* __restrict__ shared_out) {
  griddep_wait();
  griddep_launch_dependents();
  const int r = blockIdx.x;
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (c >= H) return;
  float4 p[kMaxJ];
#pragma unroll
  for (int j = 0; j < kMaxJ; ++j)
    p[j] = j < J ? *reinterpret_cast<const float4*>(P + (size_t(j) * R + r) * H + c) : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < kMaxJ; ++j) {
    if (j < J) {
      acc.x += p[j].x;
      acc.y += p[j].y;
      acc.z += p[j].z;
      acc.w += p[j].w;
    }
  }
  for (int j = kMaxJ; j < J; ++j) {  // I > 1024: the rest one by one, still in ascending j
    const float4 q = *reinterpret_cast<const float4*>(P + (size_t(j) * R + r) * H + c);
    acc.x += q.x;
    acc.y += q.y;
    acc.z += q.z;
    acc.w += q.w;
  }
  if (r < rows && f_fp32) {
    *reinterpret_cast<float4*>(static_cast<float*>(f) + size_t(r) * H + c) = acc;
    return;
  }
  T16* out = r < rows ? static_cast<T16*>(f) + size_t(r) * H + c : shared_out + size_t(r - rows) * H + c;
  uint2 v;
  v.x = Pack2<T16>::pack(acc.x, acc.y);
  v.y = Pack2<T16>::pack(acc.z, acc.w);
  *reinterpret_cast<uint2*>(out) = v;
}

template <int WQ>
int launch_fused(const Maps& maps, const Args& a, int f_fp32, void* f, void* shared_out, cudaStream_t stream) {
  using Cfg = FusedCfg<WQ>;
  static bool attr_set[64] = {false};
  int dev = 0;
  MOE_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev >= 64 || !attr_set[dev]) {
    MOE_CHECK_CUDA(cudaFuncSetAttribute(k_decode_ffn<WQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
    if (dev < 64) attr_set[dev] = true;
  }
  MOE_CHECK_CUDA(launch_pdl(k_decode_ffn<WQ>, dim3(num_sms()), dim3(Cfg::THREADS), Cfg::SMEM_BYTES, stream, maps, a));
  const int R = a.rows + a.T;
  if (R == 0) return MOE_OK;
  const dim3 grid(R, (a.H / 4 + 63) / 64);
  if (a.bf16)
    MOE_CHECK_CUDA(launch_pdl(k_sum_partials<__nv_bfloat16>, grid, dim3(64), 0, stream,
                              static_cast<const float*>(a.partial), a.I / BK, R, a.rows, a.H, f, f_fp32,
                              static_cast<__nv_bfloat16*>(shared_out)));
  else
    MOE_CHECK_CUDA(launch_pdl(k_sum_partials<__half>, grid, dim3(64), 0, stream, static_cast<const float*>(a.partial),
                              a.I / BK, R, a.rows, a.H, f, f_fp32, static_cast<__half*>(shared_out)));
  return MOE_OK;
}

int fill_args(Args& a, const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
              int E, int dtype, void* ws, size_t ws_bytes) {
  MOE_REQUIRE(T <= kFusedMaxT, MOE_ERR_UNSUPPORTED, "fused decode experts: T=%d > %d", T, kFusedMaxT);
  MOE_REQUIRE(H % BM == 0 && I % BK == 0 && H / BM <= 28, MOE_ERR_UNSUPPORTED,
              "fused decode experts: need H %% 128 == 0, H <= 3584 and I %% 64 == 0 (H=%d I=%d)", H, I);
  MOE_REQUIRE(E <= kGemmMaxGroups, MOE_ERR_UNSUPPORTED, "fused decode experts: E=%d > %d", E, kGemmMaxGroups);
  WsCarver carve(ws, ws_bytes);
  float* P = carve.take<float>(size_t(I / BK) * (rows + T) * H);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "fused decode experts: workspace of %zu bytes is too small", ws_bytes);
  a = Args{};
  a.offsets = offsets;
  a.E = E;
  a.rows = rows;
  a.T = T;
  a.H = H;
  a.I = I;
  a.row_token = row_token;
  a.x = x;
  a.partial = P;
  a.bf16 = dtype == MOE_DTYPE_BF16;
  a.status = device_status_ptr();
  a.limit_ns = wait_limit_ns();
  return MOE_OK;
}

}  // namespace

size_t decode_fused_ws_bytes(int rows, int T, int H, int I) {
  WsCounter c;
  c.take<float>(size_t(I / BK) * (rows + T) * H);
  return c.used;
}

// Routed experts (rows in permuted order, f [rows, H]) and the shared expert
// (shared_out [T, H]) for T <= 16 with 16-bit weights of width I:
// k_decode_ffn then k_sum_partials.  The FP32 partials [I/64][rows + T][H]
// live in ws.
int decode_experts_fused(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                         int E, const void* w_gu, const void* w_d, const void* w_sh_gu, const void* w_sh_d, int dtype,
                         int f_fp32, void* f, void* shared_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Args a;
  int rc = fill_args(a, x, row_token, offsets, T, rows, H, I, E, dtype, ws, ws_bytes);
  if (rc) return rc;
  Maps m;
  memset(&m, 0, sizeof(m));
  rc = make_tmap_16bit_sw128(&m.gu, w_gu, E * 2 * I, H, 64);
  if (!rc) rc = make_tmap_16bit_sw128(&m.sgu, w_sh_gu, 2 * I, H, 64);
  if (!rc) rc = make_tmap_16bit_sw128(&m.d, w_d, E * H, I, BM);
  if (!rc) rc = make_tmap_16bit_sw128(&m.sd, w_sh_d, H, I, BM);
  if (rc) return rc;
  return launch_fused<0>(m, a, f_fp32, f, shared_out, stream);
}

// The same with the routed experts in AWQ W4A16 g32 (qw_* input-major codes,
// qz_* zero points, sc_* FP16 scales) and a 16-bit shared expert: FP16
// activations, or the BF16 mode (dtype BF16: scales rounded to BF16, BF16
// weights, activations and shared expert; template WQ = 2).  qpack: the
// tile-packed copy of the routed weights (awq.cu awq_prepack) or null; when
// given, the kernel reads only it.
int decode_experts_fused_awq(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H,
                             int I, int E, const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu,
                             const int32_t* qw_d, const int32_t* qz_d, const void* sc_d, const void* w_sh_gu,
                             const void* w_sh_d, int dtype, int f_fp32, void* f, void* shared_out, void* ws,
                             size_t ws_bytes, cudaStream_t stream, const void* qpack) {
  Args a;
  int rc = fill_args(a, x, row_token, offsets, T, rows, H, I, E, dtype, ws, ws_bytes);
  if (rc) return rc;
  a.qpack = static_cast<const uint8_t*>(qpack);
  Maps m;
  memset(&m, 0, sizeof(m));
  const CUtensorMapSwizzle none = CU_TENSOR_MAP_SWIZZLE_NONE;
  rc = make_tmap_16bit_sw128(&m.sgu, w_sh_gu, 2 * I, H, 64);
  if (!rc) rc = make_tmap_16bit_sw128(&m.sd, w_sh_d, H, I, BM);
  // gate/up: input dim H, output dim 2I; down: input dim I, output dim H
  if (!rc) rc = make_tmap_2d(&m.qc_gu, qw_gu, E * H, 2 * I / 8, 4, BK, 8, none);
  if (!rc) rc = make_tmap_2d(&m.qs_gu, sc_gu, E * (H / 32), 2 * I, 2, 2, 64, none);
  if (!rc) rc = make_tmap_2d(&m.qz_gu, qz_gu, E * (H / 32), 2 * I / 8, 4, 2, 8, none);
  if (!rc) rc = make_tmap_2d(&m.qc_d, qw_d, E * I, H / 8, 4, BK, 16, none);
  if (!rc) rc = make_tmap_2d(&m.qs_d, sc_d, E * (I / 32), H, 2, 2, BM, none);
  if (!rc) rc = make_tmap_2d(&m.qz_d, qz_d, E * (I / 32), H / 8, 4, 2, 16, none);
  if (rc) return rc;
  if (a.bf16) return launch_fused<2>(m, a, f_fp32, f, shared_out, stream);
  return launch_fused<1>(m, a, f_fp32, f, shared_out, stream);
}

}  // namespace moe
