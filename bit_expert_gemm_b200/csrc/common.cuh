// Shared helpers of the sm_100a kernels: status handling, PTX wrappers for
// mbarriers, TMA, tcgen05 (TMEM allocation, UMMA issue, TMEM loads), and
// small numeric helpers.  Everything here is written for sm_100a only.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// ---------------------------------------------------------------------------
// Host-side status plumbing (implemented in abi.cu)
// ---------------------------------------------------------------------------
int set_error(int code, const char* fmt, ...);
int cuda_status(cudaError_t e, const char* what);
int* device_status_ptr();            // device address of the status word of the current device
int num_sms();                       // SMs of the current device
unsigned long long wait_limit_ns();  // bound of every device-side wait
// Tile width of a grouped GEMM from host-known sizes (abi.cu).
int pick_bn(int rows, int groups, int n_out, bool swiglu);

#define MOE_CHECK_CUDA(call)                                   \
  do {                                                         \
    cudaError_t e__ = (call);                                  \
    if (e__ != cudaSuccess) return ::moe::cuda_status(e__, #call); \
  } while (0)

#define MOE_REQUIRE(cond, code, ...)                         \
  do {                                                       \
    if (!(cond)) return ::moe::set_error((code), __VA_ARGS__); \
  } while (0)

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------------------
// Programmatic dependent launch
//
// A kernel launched with launch_pdl may start while the kernel before it on
// the stream is still running.  Every kernel so launched follows one rule:
// its prologue touches no output of the previous kernel; then it executes
// griddep_wait() (the previous kernel has completed and its writes are
// visible), then griddep_launch_dependents() (its own dependent may start).
// So when a kernel starts, everything two kernels back on the stream has
// completed, and it may read those outputs before its own wait.  Without the
// launch attribute both instructions return at once.
// ---------------------------------------------------------------------------
bool pdl_enabled();  // false when the environment sets BIT_EXPERT_GEMM_PDL=0 (abi.cu)

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Optional pre-MoE RMSNorm in front of the routing (moe_norm_route_permute):
// x_norm = x / sqrt(mean x^2 + eps) * (1 + w) in 16 bits, and with gate_w
// the shared-expert gate sigmoid(x_norm . gate_w) per token.
struct RouteNorm {
  const void* w;
  float eps;
  const void* gate_w;  // may be null (no gate)
  void* x_norm;
  float* gate;         // null iff gate_w is null
};

// Carves consecutive 256-byte aligned pieces out of a workspace.
struct WsCarver {
  char* base;
  size_t cap;
  size_t used = 0;
  bool ok = true;
  WsCarver(void* b, size_t c) : base(static_cast<char*>(b)), cap(c) {}
  template <typename T>
  T* take(size_t count) {
    size_t off = align_up(used, 256);
    size_t bytes = count * sizeof(T);
    if (off + bytes > cap) {
      ok = false;
      return nullptr;
    }
    used = off + bytes;
    return reinterpret_cast<T*>(base + off);
  }
};

// Size-only twin of WsCarver, used by moe_workspace_size.
struct WsCounter {
  size_t used = 0;
  template <typename T>
  void take(size_t count) { used = align_up(used, 256) + count * sizeof(T); }
};

// ---------------------------------------------------------------------------
// Device-side status
// ---------------------------------------------------------------------------
__device__ __forceinline__ void report(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete is
// suspended (it issues nothing) until the phase completes or about 1 ms
// passes, so waiting roles leave the issue slots to the working ones.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

// Waits until the phase of `bar` with the given parity has completed.  The
// wait is bounded: after `limit_ns` (or as soon as another role of the CTA
// raised *abort) it records MOE_ERR_TIMEOUT, raises *abort and returns false.
// The deadline and the abort flag are checked every 64 suspended tries, so the
// wait ends at most about 64 ms after either.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  unsigned long long t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait_suspend(bar, parity)) return true;
    if (((++spins) & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        report(status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// TMA (tiled tensor copies global -> shared, completion on an mbarrier)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
      "%4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
// Contiguous global -> shared copy (size a multiple of 16, both addresses
// 16-byte aligned) completing on an mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Prefetch of a tensor-map box into L2 (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// generic-proxy shared-memory writes -> visible to the async proxy (UMMA, TMA)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, UMMA, commit, TMEM -> register loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (BF16 or FP16 in, FP32 accumulate)
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every previously issued tcgen05 op of this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Instruction descriptor of kind::f16: D FP32, A and B K-major,
// a/b format 0 = FP16, 1 = BF16; M = 128; N multiple of 16 in [16, 256].
__host__ __device__ constexpr uint32_t idesc_f16(int bf16, int M, int N) {
  return (1u << 4)                       // D format: FP32
         | (uint32_t(bf16) << 7)         // A format
         | (uint32_t(bf16) << 10)        // B format
         | (uint32_t(N >> 3) << 17)      // N / 8
         | (uint32_t(M >> 4) << 24);     // M / 16
}

// Shared-memory matrix descriptor of a K-major operand stored in the
// 128-byte swizzled layout that TMA writes with CU_TENSOR_MAP_SWIZZLE_128B:
// rows of 128 bytes, 8-row swizzle atoms 1024 bytes apart (the tile base
// must be 1024-byte aligned).  Advancing along K inside the 128-byte row is
// done by adding the byte offset to the start address.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFFu);   // start address
  d |= uint64_t(1) << 16;                      // leading byte offset (unused for this layout)
  d |= uint64_t(1024 >> 4) << 32;              // stride byte offset: 8 rows x 128 B
  d |= uint64_t(1) << 46;                      // descriptor version (sm_100)
  d |= uint64_t(2) << 61;                      // layout: 128-byte swizzle
  return d;
}

// 32 lanes x 32 bit, 32 consecutive columns: thread i of the warp receives
// lane (base lane + i), columns col .. col+31.  Two loads and the wait in one
// asm statement so that no consumer can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t tb, float (&a)[32], float (&b)[32]) {
  uint32_t* ra = reinterpret_cast<uint32_t*>(a);
  uint32_t* rb = reinterpret_cast<uint32_t*>(b);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
      "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%"
      "48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(ra[0]), "=r"(ra[1]), "=r"(ra[2]), "=r"(ra[3]), "=r"(ra[4]), "=r"(ra[5]), "=r"(ra[6]), "=r"(ra[7]),
        "=r"(ra[8]), "=r"(ra[9]), "=r"(ra[10]), "=r"(ra[11]), "=r"(ra[12]), "=r"(ra[13]), "=r"(ra[14]),
        "=r"(ra[15]), "=r"(ra[16]), "=r"(ra[17]), "=r"(ra[18]), "=r"(ra[19]), "=r"(ra[20]), "=r"(ra[21]),
        "=r"(ra[22]), "=r"(ra[23]), "=r"(ra[24]), "=r"(ra[25]), "=r"(ra[26]), "=r"(ra[27]), "=r"(ra[28]),
        "=r"(ra[29]), "=r"(ra[30]), "=r"(ra[31]), "=r"(rb[0]), "=r"(rb[1]), "=r"(rb[2]), "=r"(rb[3]), "=r"(rb[4]),
        "=r"(rb[5]), "=r"(rb[6]), "=r"(rb[7]), "=r"(rb[8]), "=r"(rb[9]), "=r"(rb[10]), "=r"(rb[11]), "=r"(rb[12]),
        "=r"(rb[13]), "=r"(rb[14]), "=r"(rb[15]), "=r"(rb[16]), "=r"(rb[17]), "=r"(rb[18]), "=r"(rb[19]),
        "=r"(rb[20]), "=r"(rb[21]), "=r"(rb[22]), "=r"(rb[23]), "=r"(rb[24]), "=r"(rb[25]), "=r"(rb[26]),
        "=r"(rb[27]), "=r"(rb[28]), "=r"(rb[29]), "=r"(rb[30]), "=r"(rb[31])
      : "r"(ta), "r"(tb)
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t ta, float (&a)[32]) {
  uint32_t* ra = reinterpret_cast<uint32_t*>(a);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
      "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(ra[0]), "=r"(ra[1]), "=r"(ra[2]), "=r"(ra[3]), "=r"(ra[4]), "=r"(ra[5]), "=r"(ra[6]), "=r"(ra[7]),
        "=r"(ra[8]), "=r"(ra[9]), "=r"(ra[10]), "=r"(ra[11]), "=r"(ra[12]), "=r"(ra[13]), "=r"(ra[14]),
        "=r"(ra[15]), "=r"(ra[16]), "=r"(ra[17]), "=r"(ra[18]), "=r"(ra[19]), "=r"(ra[20]), "=r"(ra[21]),
        "=r"(ra[22]), "=r"(ra[23]), "=r"(ra[24]), "=r"(ra[25]), "=r"(ra[26]), "=r"(ra[27]), "=r"(ra[28]),
        "=r"(ra[29]), "=r"(ra[30]), "=r"(ra[31])
      : "r"(ta)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t ta, float (&a)[16]) {
  uint32_t* ra = reinterpret_cast<uint32_t*>(a);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(ra[0]), "=r"(ra[1]), "=r"(ra[2]), "=r"(ra[3]), "=r"(ra[4]), "=r"(ra[5]), "=r"(ra[6]), "=r"(ra[7]),
        "=r"(ra[8]), "=r"(ra[9]), "=r"(ra[10]), "=r"(ra[11]), "=r"(ra[12]), "=r"(ra[13]), "=r"(ra[14]),
        "=r"(ra[15])
      : "r"(ta)
      : "memory");
}

// Batched TMEM reads: 16 or 8 loads of 4 columns (or 8 of 8) at independent
// addresses, then one wait, all in one asm statement, so that the load
// latency is paid once for the batch and no consumer can run before the wait.
__device__ __forceinline__ void tmem_ld_16x4(const uint32_t (&ta)[16], uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4,%5,%6,%7}, [%65];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%8,%9,%10,%11}, [%66];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%12,%13,%14,%15}, [%67];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%16,%17,%18,%19}, [%68];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%20,%21,%22,%23}, [%69];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%24,%25,%26,%27}, [%70];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%28,%29,%30,%31}, [%71];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%32,%33,%34,%35}, [%72];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%36,%37,%38,%39}, [%73];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%40,%41,%42,%43}, [%74];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%44,%45,%46,%47}, [%75];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%48,%49,%50,%51}, [%76];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%52,%53,%54,%55}, [%77];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%56,%57,%58,%59}, [%78];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%60,%61,%62,%63}, [%79];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(ta[0]), "r"(ta[1]), "r"(ta[2]), "r"(ta[3]), "r"(ta[4]), "r"(ta[5]), "r"(ta[6]), "r"(ta[7]), "r"(ta[8]), "r"(ta[9]), "r"(ta[10]), "r"(ta[11]), "r"(ta[12]), "r"(ta[13]), "r"(ta[14]), "r"(ta[15])
      : "memory");
}

__device__ __forceinline__ void tmem_ld_8x4(const uint32_t (&ta)[8], uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4,%5,%6,%7}, [%33];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%8,%9,%10,%11}, [%34];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%12,%13,%14,%15}, [%35];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%16,%17,%18,%19}, [%36];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%20,%21,%22,%23}, [%37];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%24,%25,%26,%27}, [%38];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%28,%29,%30,%31}, [%39];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(ta[0]), "r"(ta[1]), "r"(ta[2]), "r"(ta[3]), "r"(ta[4]), "r"(ta[5]), "r"(ta[6]), "r"(ta[7])
      : "memory");
}

__device__ __forceinline__ void tmem_ld_8x8(const uint32_t (&ta)[8], uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%8,%9,%10,%11,%12,%13,%14,%15}, [%65];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%16,%17,%18,%19,%20,%21,%22,%23}, [%66];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%24,%25,%26,%27,%28,%29,%30,%31}, [%67];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%32,%33,%34,%35,%36,%37,%38,%39}, [%68];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%40,%41,%42,%43,%44,%45,%46,%47}, [%69];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%48,%49,%50,%51,%52,%53,%54,%55}, [%70];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%56,%57,%58,%59,%60,%61,%62,%63}, [%71];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(ta[0]), "r"(ta[1]), "r"(ta[2]), "r"(ta[3]), "r"(ta[4]), "r"(ta[5]), "r"(ta[6]), "r"(ta[7])
      : "memory");
}

// ---------------------------------------------------------------------------
// Numeric helpers
// ---------------------------------------------------------------------------
template <typename T>
struct Pack2;
template <>
struct Pack2<__nv_bfloat16> {
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  static __device__ __forceinline__ float2 unpack(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
  }
};
template <>
struct Pack2<__half> {
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  static __device__ __forceinline__ float2 unpack(uint32_t u) {
    __half2 v = *reinterpret_cast<__half2*>(&u);
    return __half22float2(v);
  }
};

// AWQ dequantisation of one packed word: codes q_j (nibble j of W, output
// column 8w+j), zero points z_j (nibble j of Z) and FP16 scales s_j (S holds
// s_0..s_7) -> 8 16-bit weights, as 4 packed pairs (j = 2m low half, 2m+1
// high half).
//
// FP16 (BF = false): fp16_rn((q_j - z_j) * s_j).  0x6400 | q is the FP16
// value 1024 + q, so one subtraction of two such values gives q - z exactly;
// the single FP16 multiplication then rounds once, to nearest even.
// BF16 mode (BF = true; the AWQ card's stock-runtime paragraph: the FP16
// scales are rounded to BF16 on load and the arithmetic is BF16):
// bf16_rn((q_j - z_j) * bf16_rn(s_j)).  0x4300 | q is the BF16 value 128 + q
// (7 fraction bits), so the same one-subtraction trick stays exact, and the
// scales are rounded once from FP16 when the group is prepared.
//
// (W >> 4m) & 0x000F000F | magic yields the pair (q_m, q_{m+4}) in one logic
// operation, so the arithmetic runs on the pairs (m, m+4) and four byte
// permutations restore the column order.  The zero points and scales of a
// group (AwqGroup) are prepared once for its 32 rows.
struct AwqGroup {
  uint32_t z[4];  // 16-bit pairs (magic + z_m, magic + z_{m+4})
  uint32_t s[4];  // 16-bit pairs (s_m, s_{m+4}) in the operand type
};
__device__ __forceinline__ uint32_t f16x2_to_bf16x2_rn(uint32_t v) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&v));
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<const uint32_t*>(&b);
}
template <bool BF = false>
__device__ __forceinline__ AwqGroup awq_group(uint32_t Z, uint4 S) {
  constexpr uint32_t magic = BF ? 0x43004300u : 0x64006400u;
  AwqGroup g;
#pragma unroll
  for (int m = 0; m < 4; ++m) g.z[m] = ((Z >> (4 * m)) & 0x000F000Fu) | magic;
  g.s[0] = __byte_perm(S.x, S.z, 0x5410);
  g.s[1] = __byte_perm(S.x, S.z, 0x7632);
  g.s[2] = __byte_perm(S.y, S.w, 0x5410);
  g.s[3] = __byte_perm(S.y, S.w, 0x7632);
  if (BF) {
#pragma unroll
    for (int m = 0; m < 4; ++m) g.s[m] = f16x2_to_bf16x2_rn(g.s[m]);
  }
  return g;
}
template <bool BF = false>
__device__ __forceinline__ uint4 awq_dequant8(uint32_t W, const AwqGroup& g) {
  constexpr uint32_t magic = BF ? 0x43004300u : 0x64006400u;
  uint32_t d[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint32_t q = ((W >> (4 * m)) & 0x000F000Fu) | magic;
    if (BF) {
      uint32_t t;
      asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(t) : "r"(q), "r"(g.z[m]));
      asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d[m]) : "r"(t), "r"(g.s[m]));
    } else {
      __half2 t = __hsub2(*reinterpret_cast<const __half2*>(&q), *reinterpret_cast<const __half2*>(&g.z[m]));
      __half2 v = __hmul2(t, *reinterpret_cast<const __half2*>(&g.s[m]));
      d[m] = *reinterpret_cast<uint32_t*>(&v);  // (c_m, c_{m+4})
    }
  }
  return make_uint4(__byte_perm(d[0], d[1], 0x5410), __byte_perm(d[2], d[3], 0x5410), __byte_perm(d[0], d[1], 0x7632),
                    __byte_perm(d[2], d[3], 0x7632));
}
// The same for words in pair order (the tile-packed copy: output columns 2m
// and 2m + 1 in nibbles m and m + 4, zero points likewise): the pairs come
// out as consecutive columns, so the scales are the 16-bit pairs of S as
// they are and the eight values need no reordering.
template <bool BF = false>
__device__ __forceinline__ AwqGroup awq_group_paired(uint32_t Z, uint4 S) {
  constexpr uint32_t magic = BF ? 0x43004300u : 0x64006400u;
  AwqGroup g;
#pragma unroll
  for (int m = 0; m < 4; ++m) g.z[m] = ((Z >> (4 * m)) & 0x000F000Fu) | magic;
  g.s[0] = S.x;
  g.s[1] = S.y;
  g.s[2] = S.z;
  g.s[3] = S.w;
  if (BF) {
#pragma unroll
    for (int m = 0; m < 4; ++m) g.s[m] = f16x2_to_bf16x2_rn(g.s[m]);
  }
  return g;
}
template <bool BF = false>
__device__ __forceinline__ uint4 awq_dequant8_paired(uint32_t W, const AwqGroup& g) {
  constexpr uint32_t magic = BF ? 0x43004300u : 0x64006400u;
  uint32_t d[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint32_t q = ((W >> (4 * m)) & 0x000F000Fu) | magic;
    if (BF) {
      uint32_t t;
      asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(t) : "r"(q), "r"(g.z[m]));
      asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d[m]) : "r"(t), "r"(g.s[m]));
    } else {
      __half2 t = __hsub2(*reinterpret_cast<const __half2*>(&q), *reinterpret_cast<const __half2*>(&g.z[m]));
      __half2 v = __hmul2(t, *reinterpret_cast<const __half2*>(&g.s[m]));
      d[m] = *reinterpret_cast<uint32_t*>(&v);  // (c_2m, c_2m+1)
    }
  }
  return make_uint4(d[0], d[1], d[2], d[3]);
}
template <bool BF = false>
__device__ __forceinline__ uint4 awq_dequant8(uint32_t W, uint32_t Z, uint4 S) {
  return awq_dequant8<BF>(W, awq_group<BF>(Z, S));
}

// Shared-memory matrix descriptor of an MN-major operand in the 128-byte
// swizzled layout: atoms of 64 16-bit elements along MN by 8 rows along K
// (1024 bytes, 16-byte chunk index XOR (k mod 8)); atoms along K are
// `sbo` bytes apart, atoms along MN `lbo` bytes apart.
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// silu(g) = g / (1 + e^-g).  Its callers round the product silu(g) * u to a
// 16-bit type right after, so the fast division (a couple of FP32 ulp) is
// invisible there; IEEE division made the SwiGLU epilogues ALU-heavy.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ void st_global_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

}  // namespace moe
