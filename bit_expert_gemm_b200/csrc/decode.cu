// Routed + shared SwiGLU experts for small batches (decode, T <= 128): a
// weight-streaming grouped GEMM on the tensor cores with the roles of the
// operands swapped.  The weights are the A operand (M = 128 weight rows per
// work item, streamed by TMA through a deep pipeline), the few tokens of a
// group are the B operand (N = token count rounded up to 16), so no MMA work
// or shared-memory traffic is spent on padded token rows.  The shared expert
// is one more group of work items in the same launch, so its weights stream
// concurrently with the routed experts'.
//
//   GEMM1 (MODE_GATE_UP): a work item is 64 gate rows and the matching 64 up
//     rows of one expert; the epilogue pairs them (gate in TMEM lanes 0..63,
//     up in 64..127, exchanged through shared memory) and writes
//     h[r, j] = silu(x_r . Wg_j) * (x_r . Wu_j) in the activation dtype.
//   GEMM2 (MODE_DOWN): a work item is 128 rows of W_d; f[r, n] = h[r] . Wd[n].
// Rows: the routed rows [0, rows) in permuted order, then the shared
// expert's T rows (identity tokens).  The token operand of both GEMMs is
// gathered with cp.async (x rows through row_token, or h rows); each gather
// thread arrives on the stage's full barrier when its copies land, the TMA
// producer's arrival carries the weight bytes, so one barrier per stage
// covers both operands and the gathers of many stages are in flight at once.
//
// Warp roles: 0 TMA producer (weights), 1 UMMA issuer (TMEM owner),
// 2..5 epilogue, 6..9 token-operand gather.
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "gemm_sm100.cuh"

namespace moe {

int make_tmap_16bit_sw128(CUtensorMap* map, const void* base, int rows, int cols, int box_rows);

namespace {

constexpr int BM = 128;             // weight rows per work item (MMA M)
constexpr int BK = 64;              // K per pipeline step (one 128-byte swizzle row)
constexpr int NMAX = 128;           // token rows per group handled in one pass (MMA N <= 128)
constexpr int A_BYTES = BM * BK * 2;  // 16 KB of weights per 64-wide K sub-tile
// A pipeline stage holds ksub K sub-tiles: ksub weight tiles and ksub token
// tiles of bn_max rows (the largest group rounded up to 16, at most NMAX).
// With N = 16 tokens an MMA does little work, and the per-stage cost of the
// issuing thread (barrier waits, commit: several hundred cycles) would cap
// the weight stream of an SM; ksub > 1 spreads that cost over more bytes.
// Smaller token tiles leave room for more stages.
constexpr int MAX_STAGES = 12;
constexpr int FULL_ARRIVALS = 1 + 128;  // producer (with the TMA bytes) + one per gather thread
constexpr int XCHG_STRIDE = 33;     // floats per row of the gate/up exchange buffer (bank-conflict padding)
constexpr int XCHG_BYTES = 64 * XCHG_STRIDE * 4;
constexpr int SMEM_BYTES = 217 * 1024;  // dynamic; + ~9 KB static stays under the 227 KB per block
constexpr int STAGE_SPACE = SMEM_BYTES - 1024 - XCHG_BYTES;
static_assert(STAGE_SPACE >= 6 * (A_BYTES + NMAX * BK * 2), "six full stages must fit");
constexpr int kThreads = 320;
constexpr uint32_t TMEM_COLS = 2 * NMAX;  // two accumulators of 128 x NMAX
enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

struct Args {
  const int* offsets;  // [E+1] routed expert offsets (device)
  int E;               // routed experts; group E is the shared expert
  int rows;            // routed rows
  int T;               // tokens (= rows of the shared group)
  int K;               // reduction length: H (GEMM1) or I (GEMM2)
  int MB;              // work items per group: I/64 (GEMM1) or H/128 (GEMM2)
  int I;               // intermediate width
  int H;               // hidden width
  // token operand: row c of group g is tok_src[token], token = row_token[r0+c]
  // for routed rows of GEMM1, c for the shared rows of GEMM1, r0+c for GEMM2
  const int* row_token;
  const void* tok_src;  // [*, K] 16-bit
  int tok_rows;         // rows of tok_src
  // outputs
  void* h_out;       // GEMM1: [rows + T, I] 16-bit
  void* f_out;       // GEMM2: routed rows [rows, H] (FP32 when f_fp32)
  void* shared_out;  // GEMM2: shared rows [T, H] (16-bit)
  int f_fp32;
  int bf16;
  int bn_max;  // token rows per sub-tile: round16(min(largest group, NMAX))
  int ksub;    // K sub-tiles (64 wide) per pipeline stage
  int stages;  // pipeline depth for that stage size
  int* status;
  unsigned long long limit_ns;
};

struct Item {
  int g;   // group (E = shared)
  int mb;  // block of 128 weight rows
};

__device__ __forceinline__ void group_rows(const int* goff, int g, int E, int rows, int T, int& r0, int& n) {
  if (g < E) {
    r0 = goff[g];
    n = goff[g + 1] - goff[g];
  } else {
    r0 = rows;
    n = T;
  }
}

__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// the four epilogue warps only
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

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_decode_gemm(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmWs, const Args args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[MAX_STAGES], empty_bar[MAX_STAGES], tfull_bar[2],
      tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int goff[kGemmMaxGroups + 2];
  __shared__ int item_start[kGemmMaxGroups + 2];
  __shared__ int warp_sums[kThreads / 32];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int STAGES = args.stages;
  const int ksub = args.ksub;
  const int b_sub_bytes = args.bn_max * BK * 2;
  const int stage_bytes = ksub * (A_BYTES + b_sub_bytes);
  // sub-tile j of stage s: weights at smA(s) + j * A_BYTES, tokens at smB(s) + j * b_sub_bytes
  auto smA = [&](int s) { return smem + s * stage_bytes; };
  auto smB = [&](int s) { return smem + s * stage_bytes + ksub * A_BYTES; };
  float* xchg = reinterpret_cast<float*>(smem + STAGES * stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E, G = E + 1;
  const int MB = args.MB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], FULL_ARRIVALS);
      mbar_init(&empty_bar[s], 1);
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
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmWs);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  // Launched as a programmatic dependent: GEMM1's routing comes from the
  // kernel just before it, so it waits here; GEMM2's routing is two kernels
  // back (complete when GEMM2 starts), so GEMM2 schedules and streams weights
  // at once and only its gather of h waits for GEMM1.
  if (MODE == MODE_GATE_UP) {
    griddep_wait();
    griddep_launch_dependents();
  }
  // work items: every group with rows contributes MB blocks of weight rows
  for (int i = threadIdx.x; i <= E; i += blockDim.x) goff[i] = args.offsets[i];
  __syncthreads();
  {
    const int per = (G + blockDim.x - 1) / blockDim.x;
    const int g0 = threadIdx.x * per;
    int local = 0;
    for (int g = g0; g < g0 + per && g < G; ++g) {
      int r0, n;
      group_rows(goff, g, E, args.rows, args.T, r0, n);
      local += n > 0 ? MB : 0;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int run = incl - local;
    for (int w = 0; w < warp; ++w) run += warp_sums[w];
    for (int g = g0; g < g0 + per && g < G; ++g) {
      item_start[g] = run;
      int r0, n;
      group_rows(goff, g, E, args.rows, args.T, r0, n);
      run += n > 0 ? MB : 0;
    }
    if (threadIdx.x == blockDim.x - 1) item_start[G] = run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  const int total = item_start[G];
  const int KB = args.K / BK;               // 64-wide K sub-tiles per work item
  const int NS = (KB + ksub - 1) / ksub;     // pipeline stages per work item (the last may be partial)
  int* status = args.status;
  const unsigned long long lim = args.limit_ns;
  auto item_of = [&](int L) {
    Item it;
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (item_start[mid] <= L) lo = mid; else hi = mid - 1;
    }
    it.g = lo;
    it.mb = L - item_start[lo];
    return it;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: weight blocks ----------------
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const Item it = item_of(L);
        const CUtensorMap* map = it.g < E ? &tmW : &tmWs;
        for (int ks = 0; ks < NS; ++ks) {
          const int nsub = min(ksub, KB - ks * ksub);
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], uint32_t(nsub * A_BYTES));
          for (int j = 0; j < nsub; ++j) {
            const int kx = (ks * ksub + j) * BK;
            uint8_t* a = smA(stage) + j * A_BYTES;
            if (MODE == MODE_GATE_UP) {
              // 64 gate rows, then the 64 up rows of the same features
              const int base = it.g < E ? it.g * 2 * args.I : 0;
              tma_load_2d(a, map, &full_bar[stage], kx, base + it.mb * 64);
              tma_load_2d(a + 64 * BK * 2, map, &full_bar[stage], kx, base + args.I + it.mb * 64);
            } else {
              const int base = it.g < E ? it.g * args.H : 0;
              tma_load_2d(a, map, &full_bar[stage], kx, base + it.mb * BM);
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
      // ---------------- UMMA issuer: D[weight row, token] ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const Item it = item_of(L);
        int r0, n;
        group_rows(goff, it.g, E, args.rows, args.T, r0, n);
        const int npad = (min(n, args.bn_max) + 15) & ~15;
        const uint32_t idesc = idesc_f16(args.bf16, BM, npad);
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, &abort_flag, status, lim)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(acc * NMAX);
        for (int ks = 0; ks < NS; ++ks) {
          const int nsub = min(ksub, KB - ks * ksub);
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status, lim)) { ok = false; break; }
          tc_fence_after();
          for (int j = 0; j < nsub; ++j) {
            const uint64_t ad = sdesc_kmajor_sw128(smem_u32(smA(stage) + j * A_BYTES));
            const uint64_t bd = sdesc_kmajor_sw128(smem_u32(smB(stage) + j * b_sub_bytes));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_f16(d, ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc, (ks | j | kk) != 0);
          }
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
  } else if (warp < 6) {
    // ---------------- epilogue: lane = weight row (output feature), column = token ----------------
    const int q = warp & 3;  // TMEM lane quadrant: GEMM1 q = 0,1 gate features, q = 2,3 up features
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      const Item it = item_of(L);
      int r0, n;
      group_rows(goff, it.g, E, args.rows, args.T, r0, n);
      const int nn = min(n, args.bn_max);
      if (n > args.bn_max && warp == 2 && lane == 0) report(status, MOE_ERR_UNSUPPORTED);  // more rows than the token tile
      // a timed-out wait in one warp must not leave the others at a named barrier
      if (!epilogue_all(mbar_wait(&tfull_bar[acc], acc_phase, &abort_flag, status, lim))) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * NMAX);
      for (int c0 = 0; c0 < nn; c0 += 32) {
        float v[32];
        tmem_ld32(tb + c0, v);
        if (MODE == MODE_GATE_UP) {
          // the up warps hand their values to the gate warps of the same features
          if (q >= 2) {
#pragma unroll
            for (int i = 0; i < 32; ++i) xchg[((q - 2) * 32 + lane) * XCHG_STRIDE + i] = v[i];
          }
          epilogue_sync();
          if (q < 2) {
            const int j = it.mb * 64 + q * 32 + lane;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int c = c0 + i;
              if (c < nn) {
                const float h = silu_f(v[i]) * xchg[(q * 32 + lane) * XCHG_STRIDE + i];
                const size_t o = size_t(r0 + c) * args.I + j;
                if (args.bf16)
                  static_cast<__nv_bfloat16*>(args.h_out)[o] = __float2bfloat16_rn(h);
                else
                  static_cast<__half*>(args.h_out)[o] = __float2half_rn(h);
              }
            }
          }
          epilogue_sync();
        } else {
          const int feat = it.mb * BM + q * 32 + lane;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c = c0 + i;
            if (c >= nn) break;
            if (it.g < E) {
              const size_t o = size_t(r0 + c) * args.H + feat;
              if (args.f_fp32)
                static_cast<float*>(args.f_out)[o] = v[i];
              else if (args.bf16)
                static_cast<__nv_bfloat16*>(args.f_out)[o] = __float2bfloat16_rn(v[i]);
              else
                static_cast<__half*>(args.f_out)[o] = __float2half_rn(v[i]);
            } else {
              const size_t o = size_t(c) * args.H + feat;
              if (args.bf16)
                static_cast<__nv_bfloat16*>(args.shared_out)[o] = __float2bfloat16_rn(v[i]);
              else
                static_cast<__half*>(args.shared_out)[o] = __float2half_rn(v[i]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  } else {
    // ---------------- token operand gather: warps 6..9 ----------------
    // Thread gt copies 16-byte chunk (gt % 8) of token rows gt/8, gt/8 + 16,
    // ... of the step into the K-major 128-byte-swizzled B tile (chunk index
    // XOR row mod 8); rows from the group size up to the next multiple of 16
    // are zero-filled.  Each thread arrives on the stage's barrier once its
    // copies have landed.
    if (MODE == MODE_DOWN) {  // h is GEMM1's output
      griddep_wait();
      griddep_launch_dependents();
    }
    const int gt = threadIdx.x - 192;
    const int ch = gt & 7;
    const int cb = gt >> 3;
    const uint8_t* src = static_cast<const uint8_t*>(args.tok_src);
    const size_t pitch = size_t(args.K) * 2;
    int stage = 0;
    uint32_t phase = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      const Item it = item_of(L);
      int r0, n;
      group_rows(goff, it.g, E, args.rows, args.T, r0, n);
      const int nn = min(n, args.bn_max);
      const int npad = (nn + 15) & ~15;
      int row[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = cb + 16 * i;
        int rr = -1;
        if (c < nn) {
          if (MODE == MODE_GATE_UP)
            rr = it.g < E ? __ldg(args.row_token + r0 + c) : c;
          else
            rr = r0 + c;
          if (rr >= args.tok_rows) rr = -1;
        }
        row[i] = rr;
      }
      bool ok = true;
      for (int ks = 0; ks < NS; ++ks) {
        const int nsub = min(ksub, KB - ks * ksub);
        if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, lim)) { ok = false; break; }
        for (int j = 0; j < nsub; ++j) {
          const uint32_t bt = smem_u32(smB(stage) + j * b_sub_bytes);
          const size_t kbyte = size_t(ks * ksub + j) * 128;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = cb + 16 * i;
            if (c < npad) {
              const uint8_t* g = src + (row[i] >= 0 ? size_t(row[i]) * pitch + kbyte + ch * 16 : 0);
              cp_async_16_zfill(bt + uint32_t(c * 128 + ((ch ^ (c & 7)) << 4)), g, row[i] >= 0 ? 16u : 0u);
            }
          }
        }
        cp_async_arrive_noinc(&full_bar[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // every copy has landed before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

int stages_for(int ksub, int bn_max) {
  const int per_stage = ksub * (A_BYTES + bn_max * BK * 2);
  return STAGE_SPACE / per_stage < MAX_STAGES ? STAGE_SPACE / per_stage : MAX_STAGES;
}

// K sub-tiles per stage: the widest of 4, 2, 1 that leaves a double-buffered
// pipeline (measured on B200: 4 sub-tiles in 2 stages stream faster than 2 in
// 4).  BIT_EXPERT_GEMM_DECODE_KSUB (1, 2 or 4) overrides it for tuning.
int decode_ksub(int bn_max) {
  static int forced = -1;
  if (forced < 0) {
    const char* s = getenv("BIT_EXPERT_GEMM_DECODE_KSUB");
    const int e = s ? atoi(s) : 0;
    forced = (e == 1 || e == 2 || e == 4) ? e : 0;
  }
  if (forced && stages_for(forced, bn_max) >= 2) return forced;
  for (int k = 4; k > 1; k >>= 1)
    if (stages_for(k, bn_max) >= 2) return k;
  return 1;
}

template <int MODE>
int launch_decode(const CUtensorMap& tw, const CUtensorMap& tws, const Args& a, cudaStream_t stream) {
  static bool attr_set[64] = {false};
  int dev = 0;
  MOE_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev >= 64 || !attr_set[dev]) {
    MOE_CHECK_CUDA(cudaFuncSetAttribute(k_decode_gemm<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    if (dev < 64) attr_set[dev] = true;
  }
  MOE_CHECK_CUDA(launch_pdl(k_decode_gemm<MODE>, dim3(num_sms()), dim3(kThreads), SMEM_BYTES, stream, tw, tws, a));
  return MOE_OK;
}

}  // namespace

size_t decode_ws_bytes(int rows, int T, int I) {
  WsCounter c;
  c.take<uint16_t>(size_t(rows + T) * I);
  return c.used;
}

// Routed experts (rows in permuted order) and the shared expert (T identity
// rows) for T <= 128, both with weights of width I; f receives the routed
// rows, shared_out the shared expert's.  h [rows + T, I] lives in ws.
int decode_experts_16bit(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                         int E, const void* w_gu, const void* w_d, const void* w_sh_gu, const void* w_sh_d, int dtype,
                         int f_fp32, void* f, void* shared_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  MOE_REQUIRE(T <= NMAX, MOE_ERR_UNSUPPORTED, "decode experts: T=%d > %d", T, NMAX);
  MOE_REQUIRE(H % BM == 0 && I % 64 == 0, MOE_ERR_UNSUPPORTED,
              "decode experts: need H %% 128 == 0 and I %% 64 == 0 (H=%d I=%d)", H, I);
  WsCarver carve(ws, ws_bytes);
  void* h = carve.take<uint16_t>(size_t(rows + T) * I);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "decode experts: workspace of %zu bytes is too small", ws_bytes);
  CUtensorMap tw1, tws1, tw2, tws2;
  int rc = make_tmap_16bit_sw128(&tw1, w_gu, E * 2 * I, H, 64);
  if (!rc) rc = make_tmap_16bit_sw128(&tws1, w_sh_gu, 2 * I, H, 64);
  if (!rc) rc = make_tmap_16bit_sw128(&tw2, w_d, E * H, I, BM);
  if (!rc) rc = make_tmap_16bit_sw128(&tws2, w_sh_d, H, I, BM);
  if (rc) return rc;
  Args a{};
  a.offsets = offsets;
  a.E = E;
  a.rows = rows;
  a.T = T;
  a.I = I;
  a.H = H;
  a.h_out = h;
  a.f_out = f;
  a.shared_out = shared_out;
  a.f_fp32 = f_fp32;
  a.bf16 = dtype == MOE_DTYPE_BF16;
  a.status = device_status_ptr();
  a.limit_ns = wait_limit_ns();
  // every group (routed: tokens that chose the expert; shared: all T) has at most T rows
  a.bn_max = ((T < NMAX ? T : NMAX) + 15) & ~15;
  a.ksub = decode_ksub(a.bn_max);
  a.stages = stages_for(a.ksub, a.bn_max);
  MOE_REQUIRE(a.stages >= 2, MOE_ERR_UNSUPPORTED, "decode experts: %d K sub-tiles per stage leave %d stages",
              a.ksub, a.stages);
  // GEMM1 (+ SwiGLU): tokens gathered from x
  a.K = H;
  a.MB = I / 64;
  a.row_token = row_token;
  a.tok_src = x;
  a.tok_rows = T;
  rc = launch_decode<MODE_GATE_UP>(tw1, tws1, a, stream);
  if (rc) return rc;
  // GEMM2: token rows of h
  a.K = I;
  a.MB = H / BM;
  a.row_token = nullptr;
  a.tok_src = h;
  a.tok_rows = rows + T;
  return launch_decode<MODE_DOWN>(tw2, tws2, a, stream);
}

}  // namespace moe
