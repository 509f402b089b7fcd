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
//     projection (H x 64, as 16 blocks of 128 rows): a split-K slice of the
//     second GEMM, whose FP32 result is the partial P[j][row][0..H).
// Phase B's weights do not depend on h, so they stream right behind phase
// A's and the whole call is one stream of weights through every SM, with no
// wait between GEMM1 and GEMM2.  A second kernel sums the I/64 partials of
// every row in a fixed order (deterministic) into f (routed rows) and
// shared_out (shared rows).
//
// Warp roles: 0 TMA producer (weights), 1 UMMA issuer (TMEM owner), 2..5
// epilogue, 6..9 token gather (cp.async, arriving on the stage's barrier).
// TMEM: two 16-column phase-A accumulators (columns 0..31) and one phase-B
// accumulator of H/128 blocks x 16 columns (from column 32).
#include "common.cuh"
#include "gemm_sm100.cuh"

namespace moe {

int make_tmap_16bit_sw128(CUtensorMap* map, const void* base, int rows, int cols, int box_rows);

constexpr int kFusedMaxT = 16;

namespace {

constexpr int BM = 128;                    // weight rows per MMA (M)
constexpr int BK = 64;                     // K per sub-tile (one 128-byte swizzle row)
constexpr int NT = 16;                     // token columns (N) of every MMA
constexpr int A_BYTES = BM * BK * 2;       // 16 KB of weights per sub-tile
constexpr int B_BYTES = NT * BK * 2;       // 2 KB of tokens per sub-tile
constexpr int SUB_BYTES = A_BYTES + B_BYTES;
constexpr int KSUB = 2;                    // sub-tiles per pipeline stage
constexpr int STAGE_BYTES = KSUB * SUB_BYTES;
constexpr int STAGES = 5;
constexpr int H_BYTES = NT * BK * 2;       // one h tile: 16 rows x 64 features
constexpr int XS = NT + 1;                 // floats per row of the accumulator exchange (bank padding)
constexpr int XCHG_BYTES = BM * XS * 4;    // all 128 phase-A rows (64 gate, 64 up)
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 2 * H_BYTES + XCHG_BYTES;
constexpr int kThreads = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACCB_COL = 32;
constexpr int FULL_ARRIVALS = 1 + 128;     // producer (with the TMA bytes) + one per gather thread
static_assert(SUB_BYTES % 1024 == 0 && H_BYTES % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(SMEM_BYTES <= 222 * 1024, "shared memory");

struct Args {
  const int* offsets;   // [E+1] routed expert offsets (device)
  int E, rows, T, H, I;
  const int* row_token; // [rows] token of each routed row
  const void* x;        // [T, H] 16-bit tokens
  float* partial;       // [I/64][rows + T][H] FP32
  int bf16;
  int* status;
  unsigned long long limit_ns;
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

__global__ void __launch_bounds__(kThreads, 1)
    k_decode_ffn(const __grid_constant__ CUtensorMap tmGU, const __grid_constant__ CUtensorMap tmGUs,
                 const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmDs, const Args args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES], accA_full[2], accA_empty[2], h_full[2],
      h_empty[2], accB_full, accB_empty, drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int goff[kGemmMaxGroups + 2];
  __shared__ int item_start[kGemmMaxGroups + 2];
  __shared__ int warp_sums[kThreads / 32];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // sub-tile u of stage s: weights at sub(s, u), tokens at sub(s, u) + A_BYTES
  auto sub = [&](int s, int u) { return smem + s * STAGE_BYTES + u * SUB_BYTES; };
  uint8_t* htile = smem + STAGES * STAGE_BYTES;  // two h tiles of H_BYTES
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
    tma_prefetch_desc(&tmGU);
    tma_prefetch_desc(&tmGUs);
    tma_prefetch_desc(&tmD);
    tma_prefetch_desc(&tmDs);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
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
    if (lane == 0) {
      // ---------------- TMA producer: phase-A then phase-B weights of every item ----------------
      const uint64_t pol = l2_policy_evict_first();  // read once per call
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const int g = group_of(L);
        const int j = L - item_start[g];
        const CUtensorMap* gu = g < E ? &tmGU : &tmGUs;
        const CUtensorMap* dn = g < E ? &tmD : &tmDs;
        const int gu_base = g < E ? g * 2 * args.I : 0;
        const int dn_base = g < E ? g * args.H : 0;
        for (int st = 0; st < NSA + NSB && ok; ++st) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, lim)) { ok = false; break; }
          if (st < NSA) {
            mbar_arrive_expect_tx(&full_bar[stage], uint32_t(KSUB * A_BYTES));
            for (int u = 0; u < KSUB; ++u) {
              const int kx = (st * KSUB + u) * BK;
              tma_load_2d_hint(sub(stage, u), gu, &full_bar[stage], kx, gu_base + j * 64, pol);
              tma_load_2d_hint(sub(stage, u) + 64 * BK * 2, gu, &full_bar[stage], kx, gu_base + args.I + j * 64, pol);
            }
          } else {
            const int m0 = (st - NSA) * KSUB;
            const int nsub = min(KSUB, MB2 - m0);
            mbar_arrive_expect_tx(&full_bar[stage], uint32_t(nsub * A_BYTES));
            for (int u = 0; u < nsub; ++u)
              tma_load_2d_hint(sub(stage, u), dn, &full_bar[stage], j * BK, dn_base + (m0 + u) * BM, pol);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {  // let the loads in flight land before the block exits
        volatile int never = 0;
        for (long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          mbar_wait(&full_bar[i % STAGES], uint32_t((i / STAGES) & 1), &never, nullptr, lim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer ----------------
      const uint32_t idesc = idesc_f16(args.bf16, BM, NT);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int n = 0;  // items of this CTA so far
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++n) {
        const int a = n & 1;                     // phase-A accumulator and h tile of this item
        const uint32_t pa = uint32_t((n >> 1) & 1);  // their phase parity
        // phase A: D_A[weight row, token] over K = H
        if (!mbar_wait(&accA_empty[a], pa ^ 1, &abort_flag, status, lim)) break;
        tc_fence_after();
        const uint32_t dA = tmem_base + uint32_t(a * NT);
        for (int st = 0; st < NSA; ++st) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status, lim)) { ok = false; break; }
          tc_fence_after();
          for (int u = 0; u < KSUB; ++u) {
            const uint64_t ad = sdesc_kmajor_sw128(smem_u32(sub(stage, u)));
            const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sub(stage, u) + A_BYTES));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_f16(dA, ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc, (st | u | kk) != 0);
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
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status, lim)) { ok = false; break; }
          tc_fence_after();
          for (int u = 0; u < nsub; ++u) {
            const uint64_t ad = sdesc_kmajor_sw128(smem_u32(sub(stage, u)));
            const uint32_t dB = tmem_base + ACCB_COL + uint32_t((m0 + u) * NT);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_f16(dB, ad + uint64_t(kk * 2), hd + uint64_t(kk * 2), idesc, kk != 0);
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
      for (int c = 0; c < NT; ++c) xchg[(q * 32 + lane) * XS + c] = v[c];
      epilogue_sync();
      {
        // h[c][f] = silu(gate[f][c]) * up[f][c], 16-bit, K-major 128-byte
        // swizzled: row c at c*128 bytes, 16-byte chunk (f/8) xor (c%8),
        // element f%8.  1024 values over the 128 threads, in a rolled loop
        // (this code runs once per item: compact code stays cached).
        const int et = threadIdx.x - 64;
        uint8_t* ht = htile + a * H_BYTES;
#pragma unroll 1
        for (int idx = et; idx < 64 * NT; idx += 128) {
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
      float* P = args.partial + (size_t(j) * R + r0) * args.H;
      // four blocks' accumulators (64 consecutive columns) per TMEM load wait
      for (int m0 = 0; m0 < MB2; m0 += 4) {
        float w0[32], w1[32];
        const uint32_t ta = tmem_base + (uint32_t(q * 32) << 16) + ACCB_COL + uint32_t(m0 * NT);
        tmem_ld32x2(ta, ta + 32, w0, w1);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (m0 + u < MB2) {
            const int feat = (m0 + u) * BM + q * 32 + lane;
#pragma unroll
            for (int c = 0; c < NT; ++c) {
              const float val = u < 2 ? w0[u * NT + c] : w1[(u - 2) * NT + c];
              if (c < nn) P[size_t(c) * args.H + feat] = val;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&accB_empty);
    }
  } else {
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
// ceil(H / 1024)); launched as a programmatic dependent of k_decode_ffn.
template <typename T16>
__global__ void __launch_bounds__(256) k_sum_partials(const float* __restrict__ P, int J, int R, int rows, int H,
                                                      void* __restrict__ f, int f_fp32, T16* __restrict__ shared_out) {
  griddep_wait();
  griddep_launch_dependents();
  const int r = blockIdx.x;
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (c >= H) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < J; ++j) {
    const float4 p = *reinterpret_cast<const float4*>(P + (size_t(j) * R + r) * H + c);
    acc.x += p.x;
    acc.y += p.y;
    acc.z += p.z;
    acc.w += p.w;
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

}  // namespace

size_t decode_fused_ws_bytes(int rows, int T, int H, int I) {
  WsCounter c;
  c.take<float>(size_t(I / BK) * (rows + T) * H);
  return c.used;
}

// Routed experts (rows in permuted order, f [rows, H]) and the shared expert
// (shared_out [T, H]) for T <= 16 with weights of width I: k_decode_ffn then
// k_sum_partials.  The FP32 partials [I/64][rows + T][H] live in ws.
int decode_experts_fused(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                         int E, const void* w_gu, const void* w_d, const void* w_sh_gu, const void* w_sh_d, int dtype,
                         int f_fp32, void* f, void* shared_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  MOE_REQUIRE(T <= kFusedMaxT, MOE_ERR_UNSUPPORTED, "fused decode experts: T=%d > %d", T, kFusedMaxT);
  MOE_REQUIRE(H % BM == 0 && I % BK == 0, MOE_ERR_UNSUPPORTED,
              "fused decode experts: need H %% 128 == 0 and I %% 64 == 0 (H=%d I=%d)", H, I);
  MOE_REQUIRE(E <= kGemmMaxGroups, MOE_ERR_UNSUPPORTED, "fused decode experts: E=%d > %d", E, kGemmMaxGroups);
  WsCarver carve(ws, ws_bytes);
  float* P = carve.take<float>(size_t(I / BK) * (rows + T) * H);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "fused decode experts: workspace of %zu bytes is too small", ws_bytes);
  CUtensorMap tgu, tgus, td, tds;
  int rc = make_tmap_16bit_sw128(&tgu, w_gu, E * 2 * I, H, 64);
  if (!rc) rc = make_tmap_16bit_sw128(&tgus, w_sh_gu, 2 * I, H, 64);
  if (!rc) rc = make_tmap_16bit_sw128(&td, w_d, E * H, I, BM);
  if (!rc) rc = make_tmap_16bit_sw128(&tds, w_sh_d, H, I, BM);
  if (rc) return rc;
  Args a{};
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
  static bool attr_set[64] = {false};
  int dev = 0;
  MOE_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev >= 64 || !attr_set[dev]) {
    MOE_CHECK_CUDA(cudaFuncSetAttribute(k_decode_ffn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    if (dev < 64) attr_set[dev] = true;
  }
  MOE_CHECK_CUDA(launch_pdl(k_decode_ffn, dim3(num_sms()), dim3(kThreads), SMEM_BYTES, stream, tgu, tgus, td, tds, a));
  const int R = rows + T;
  if (R == 0) return MOE_OK;
  const dim3 grid(R, (H / 4 + 255) / 256);
  if (a.bf16)
    MOE_CHECK_CUDA(launch_pdl(k_sum_partials<__nv_bfloat16>, grid, dim3(256), 0, stream, static_cast<const float*>(P),
                              I / BK, R, rows, H, f, f_fp32, static_cast<__nv_bfloat16*>(shared_out)));
  else
    MOE_CHECK_CUDA(launch_pdl(k_sum_partials<__half>, grid, dim3(256), 0, stream, static_cast<const float*>(P), I / BK,
                              R, rows, H, f, f_fp32, static_cast<__half*>(shared_out)));
  return MOE_OK;
}

}  // namespace moe
