// AWQ W4A16 g32 grouped SwiGLU (kernels follow in a later change).
#include "common.cuh"

namespace moe {

size_t awq_ws_bytes(int rows, int H, int I, int E) {
  WsCounter c;
  c.take<uint16_t>(size_t(rows) * H);
  c.take<uint16_t>(size_t(rows) * I);
  (void)E;
  return c.used;
}

int grouped_swiglu_awq(const void*, const int32_t*, const int32_t*, int, int, int, int, int, const int32_t*,
                       const int32_t*, const void*, const int32_t*, const int32_t*, const void*, int, void*, void*,
                       size_t, cudaStream_t) {
  return set_error(MOE_ERR_UNSUPPORTED, "moe_grouped_swiglu_awq_g32: not built in this library version");
}

}  // namespace moe
