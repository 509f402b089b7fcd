// moe_permute for callers that cannot hand the library a workspace.
//
// Some callers only receive input and output buffers from the framework that
// hosts them -- a plug-in interface that exposes no allocator, a runtime that
// owns a fixed memory pool, or a latency-critical step where a cudaMalloc
// (which may synchronise the device) is not acceptable.  This entry point
// runs the same permutation as moe_permute, with its scratch memory in a
// fixed array that lives in this library's device image instead of a
// caller-supplied workspace.  It allocates nothing.
//
// The array is file-scope static device memory of a fixed, modest size
// (kNoAllocScratchBytes below): every GPU that loads this library holds it
// until the process exits.  All calls on one device share it, and it keeps
// the contents of the last call; the permutation clears the part that must
// start at zero (the expert bitmask) on the call's stream.  Two calls whose
// kernels overlap on the GPU (different streams, no ordering between them)
// race on the array.
#include <atomic>

#include "common.cuh"

namespace moe {

size_t permute_ws_bytes(int T, int E);
int permute(const int32_t* topk_idx, int T, int ks, int E, int32_t* offsets, int32_t* row_token, int32_t* slot_row,
            void* ws, size_t ws_bytes, cudaStream_t stream);

namespace {

// Scratch of the permutation: expert bitmask and prefix words (E x ceil(T/32)
// 32-bit words each) and E counts.  Sized for E * ceil(T/32) <= 2^19 words,
// e.g. E = 512 experts and T = 32768 tokens.
constexpr long kNoAllocMaxMaskWords = 1l << 19;
constexpr size_t kNoAllocScratchBytes = size_t(kNoAllocMaxMaskWords) * 4 * 2 + 1024 * 4 + 3 * 256;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
// Per-device cache of the array's device address.  Host threads may race to
// fill an entry; they all store the same value, and the atomic makes that
// race well defined.  The cache assumes the device's primary context lives
// as long as the process: after cudaDeviceReset the library's module is
// loaded again, possibly at another address, and the cached entry is stale.
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  The array's
// name in host code is only a host-side stand-in; its device address comes
// from the runtime, once per device, with that device current.
int scratch_address(void** out) {
  int dev = 0;
  MOE_CHECK_CUDA(cudaGetDevice(&dev));
  MOE_REQUIRE(dev >= 0 && dev < kMaxDevices, MOE_ERR_UNSUPPORTED, "moe_permute_noalloc: device %d >= %d", dev,
              kMaxDevices);
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    MOE_CHECK_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    MOE_REQUIRE(p != nullptr, MOE_ERR_CUDA, "moe_permute_noalloc: no device address for the scratch array");
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_permute_noalloc(const int32_t* topk_idx, int T, int k_slots, int E, int32_t* expert_offsets,
                                   int32_t* row_token, int32_t* slot_row, void* stream) {
  MOE_REQUIRE(T >= 0 && k_slots >= 1 && k_slots <= 16 && E >= 1 && E <= 1024, MOE_ERR_UNSUPPORTED,
              "moe_permute_noalloc: need T>=0, 1<=k_slots<=16, 1<=E<=1024 (T=%d k_slots=%d E=%d)", T, k_slots, E);
  MOE_REQUIRE(long(T) * k_slots < (1l << 31), MOE_ERR_UNSUPPORTED, "moe_permute_noalloc: T*k_slots overflows int32");
  const long words = long(E) * ((long(T) + 31) / 32);
  MOE_REQUIRE(words <= kNoAllocMaxMaskWords, MOE_ERR_UNSUPPORTED,
              "moe_permute_noalloc: E * ceil(T/32) = %ld exceeds the fixed scratch limit of %ld words "
              "(use moe_permute with a workspace for larger batches)",
              words, kNoAllocMaxMaskWords);
  MOE_REQUIRE(permute_ws_bytes(T, E) <= kNoAllocScratchBytes, MOE_ERR_UNSUPPORTED,
              "moe_permute_noalloc: batch needs %zu bytes of scratch, the fixed array holds %zu",
              permute_ws_bytes(T, E), kNoAllocScratchBytes);
  MOE_REQUIRE(expert_offsets != nullptr, MOE_ERR_INVALID_ARG, "moe_permute_noalloc: expert_offsets is null");
  MOE_REQUIRE(T == 0 || (topk_idx && row_token && slot_row), MOE_ERR_INVALID_ARG,
              "moe_permute_noalloc: null pointer");
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc) return rc;
  return permute(topk_idx, T, k_slots, E, expert_offsets, row_token, slot_row, scratch, kNoAllocScratchBytes,
                 static_cast<cudaStream_t>(stream));
}
