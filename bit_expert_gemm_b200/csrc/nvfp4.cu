// NVFP4 W4A4 quantisation and grouped SwiGLU (kernels follow in a later change).
#include "common.cuh"

namespace moe {

size_t nvfp4_quant_ws_bytes(int batch, int rows, int K) { (void)batch; (void)rows; (void)K; return 256; }
size_t nvfp4_ws_bytes(int rows, int H, int I, int E) { (void)rows; (void)H; (void)I; (void)E; return 256; }

int nvfp4_quantize(const void*, int, int, int, int, const float*, uint8_t*, uint8_t*, float*, void*, size_t,
                   cudaStream_t) {
  return set_error(MOE_ERR_UNSUPPORTED, "moe_nvfp4_quantize: not built in this library version");
}

int grouped_swiglu_nvfp4(const void*, const int32_t*, const int32_t*, int, int, int, int, int, const uint8_t*,
                         const uint8_t*, const float*, const uint8_t*, const uint8_t*, const float*, const float*,
                         float*, int, void*, void*, size_t, cudaStream_t) {
  return set_error(MOE_ERR_UNSUPPORTED, "moe_grouped_swiglu_nvfp4: not built in this library version");
}

}  // namespace moe
