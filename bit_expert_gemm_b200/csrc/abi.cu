// extern "C" entry points declared in include/moe.h: host-side argument
// checks, workspace sizing, and dispatch to the kernels.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "gemm_sm100.cuh"

namespace moe {

// implemented in the other translation units
size_t route_ws_bytes(int T, int E);
int route_topk(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
               int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, void* ws, size_t ws_bytes,
               cudaStream_t stream);
size_t permute_ws_bytes(int T, int E);
size_t route_permute_ws_bytes(int T, int E);
int route_permute(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
                  int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, int32_t* offsets,
                  int32_t* row_token, int32_t* slot_row, void* ws, size_t ws_bytes, cudaStream_t stream, const RouteNorm* norm = nullptr);
int permute(const int32_t* topk_idx, int T, int ks, int E, int32_t* offsets, int32_t* row_token, int32_t* slot_row,
            void* ws, size_t ws_bytes, cudaStream_t stream);
int gather_rows(const void* x, const int32_t* row_token, int rows, int H, void* out, cudaStream_t stream);
int combine(const void* f, int f_fp32, const int32_t* slot_row, int ks, const float* w, const void* shared,
            const float* gate, int T, int k, int H, int dtype, void* y, cudaStream_t stream);
size_t refill_ws_bytes(int T, int k);
int refill(const void* f, int f_fp32, const int32_t* slot_row, const float* topk_logit, const int32_t* offsets, int T,
           int k, int H, int E, double* sum_sq, int64_t* count, const void* shared, void* y_out, int dtype, void* ws,
           size_t ws_bytes, cudaStream_t stream);
int select_experts(const double* sum_sq, const int64_t* count, int E, int keep, int32_t* kept, int32_t* ranking,
                   double* score, cudaStream_t stream);
size_t awq_ws_bytes(int rows, int H, int I, int E);
int grouped_swiglu_awq(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                       int E, const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu, const int32_t* qw_d,
                       const int32_t* qz_d, const void* sc_d, int dtype, int out_fp32, void* f, void* ws,
                       size_t ws_bytes, cudaStream_t stream, const void* awq_packed);
int awq_dequant(const int32_t* qweight, const int32_t* qzeros, const void* scales, int batch, int K, int N, int dtype,
                void* out, cudaStream_t stream);
size_t nvfp4_quant_ws_bytes(int batch, int rows, int K);
size_t decode_ws_bytes(int rows, int T, int I);
size_t decode_fused_ws_bytes(int rows, int T, int H, int I);
int decode_experts_fused_awq(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H,
                             int I, int E, const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu,
                             const int32_t* qw_d, const int32_t* qz_d, const void* sc_d, const void* w_sh_gu,
                             const void* w_sh_d, int dtype, int f_fp32, void* f, void* shared_out, void* ws,
                             size_t ws_bytes, cudaStream_t stream, const void* qpack);
size_t awq_packed_bytes(int E, int H, int I);
int awq_prepack(const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu, const int32_t* qw_d,
                const int32_t* qz_d, const void* sc_d, int E, int H, int I, void* out, cudaStream_t stream);
int decode_experts_fused(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                         int E, const void* w_gu, const void* w_d, const void* w_sh_gu, const void* w_sh_d, int dtype,
                         int f_fp32, void* f, void* shared_out, void* ws, size_t ws_bytes, cudaStream_t stream);
int decode_experts_16bit(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                         int E, const void* w_gu, const void* w_d, const void* w_sh_gu, const void* w_sh_d, int dtype,
                         int f_fp32, void* f, void* shared_out, void* ws, size_t ws_bytes, cudaStream_t stream);
int nvfp4_quantize(const void* v, int batch, int rows, int K, int dtype, const float* gs_in, uint8_t* codes,
                   uint8_t* sf, float* gs_out, void* ws, size_t ws_bytes, cudaStream_t stream);
size_t nvfp4_ws_bytes(int rows, int H, int I, int E);
int grouped_swiglu_nvfp4(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H,
                         int I, int E, const uint8_t* w_gu, const uint8_t* sf_gu, const float* gs_gu,
                         const uint8_t* w_d, const uint8_t* sf_d, const float* gs_d, const float* act_gs_in,
                         float* act_gs_out, int out_fp32, void* f, void* ws, size_t ws_bytes, cudaStream_t stream,
                         const uint8_t* w1sf_packed, const uint8_t* w2sf_packed);
size_t nvfp4_packed_sf_bytes(int E, int rows_per_expert, int K, int swiglu);
int nvfp4_prepack_sf(const uint8_t* sf, int E, int rows_per_expert, int K, int swiglu, uint8_t* out,
                     cudaStream_t stream);
int shared_gate(const void* x, int T, int H, const void* w_gate, int dtype, float* gate, cudaStream_t stream);
int rmsnorm(const void* x, int T, int H, const void* w, float eps, int dtype, void* y, cudaStream_t stream,
            const void* w_gate = nullptr, float* gate = nullptr);
size_t dense_gemv_ws_bytes(int T, int I);
bool dense_gemv_fits(int T, int H, int I);
int dense_swiglu_gemv(const void* x, const int32_t* offsets, int T, int H, int I, const void* w_gu, const void* w_d,
                      int dtype, int out_fp32, void* out, void* ws, size_t ws_bytes, cudaStream_t stream);
int router_norm(const void* w_router, int E, int H, int dtype, double* sum_sq, int64_t* count, cudaStream_t stream);
int slice_experts(const void* src, int E, size_t bytes_per_expert, const int32_t* kept, int keep, void* dst,
                  cudaStream_t stream);

namespace {
thread_local char g_err[1024] = "";
__device__ int g_status = 0;
constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
int g_sms[kMaxDevices] = {0};
}  // namespace

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_status(cudaError_t e, const char* what) {
  return set_error(MOE_ERR_CUDA, "%s failed: %s", what, cudaGetErrorString(e));
}

static int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return 0;
  return d < kMaxDevices ? d : 0;
}

int* device_status_ptr() {
  const int d = current_device();
  if (!g_status_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) == cudaSuccess) g_status_ptr[d] = static_cast<int*>(p);
  }
  return g_status_ptr[d];
}

int num_sms() {
  const int d = current_device();
  if (!g_sms[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    g_sms[d] = n;
  }
  return g_sms[d];
}

unsigned long long wait_limit_ns() {
  static unsigned long long lim = 0;
  if (!lim) {
    const char* s = getenv("BIT_EXPERT_GEMM_WAIT_LIMIT_MS");
    long ms = s ? atol(s) : 0;
    lim = (ms > 0 ? (unsigned long long)ms : 5000ull) * 1000000ull;
  }
  return lim;
}

bool pdl_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* s = getenv("BIT_EXPERT_GEMM_PDL");
    on = (s && s[0] == '0') ? 0 : 1;
  }
  return on != 0;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Tile-width choice of a grouped GEMM from host-known sizes only: the widest
// tile that still gives at least one tile per SM for an upper bound of the
// number of row tiles.
int pick_bn(int rows, int groups, int n_out, bool swiglu) {
  const long mt = (rows + 127) / 128 + (groups < rows ? groups : rows);
  const int cands[3] = {256, 128, 64};
  int last_ok = 0;
  for (int bn : cands) {
    const int bnh = swiglu ? bn / 2 : bn;
    if (n_out % bnh) continue;
    last_ok = bn;
    if (mt * (n_out / bnh) >= num_sms()) return bn;
  }
  return last_ok;
}

static int swiglu_bf16(const void* x, const int32_t* row_token, const int32_t* offsets, int T, int rows, int H, int I,
                       int E, const void* w_gu, const void* w_d, int dtype, int out_fp32, void* f, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
  WsCarver carve(ws, ws_bytes);
  uint16_t* h = carve.take<uint16_t>(size_t(rows) * I);
  MOE_REQUIRE(carve.ok, MOE_ERR_WORKSPACE, "moe_grouped_swiglu_bf16: workspace of %zu bytes is too small", ws_bytes);
  if (rows == 0) return MOE_OK;
  // GEMM1 gathers its A rows (x[row_token[r]]) itself: no permuted copy of x
  const void* a = x;
  GemmArgs g1{};
  g1.row_token = row_token;
  g1.a_src = x;
  g1.a_src_rows = T;
  g1.group_offsets = offsets;
  g1.G = E;
  g1.rows = rows;
  g1.K = H;
  g1.n_out = I;
  g1.b_rows_per_group = 2 * I;
  g1.up_offset = I;
  g1.out = h;
  g1.ldo = I;
  g1.out_fp32 = 0;
  g1.bias = nullptr;
  g1.bf16 = dtype == MOE_DTYPE_BF16;
  g1.status = device_status_ptr();
  g1.limit_ns = wait_limit_ns();
  int rc = launch_grouped_gemm(a, rows, w_gu, E * 2 * I, g1, EPI_SWIGLU, pick_bn(rows, E, I, true), stream);
  if (rc) return rc;
  GemmArgs g2 = g1;
  g2.row_token = nullptr;
  g2.a_src = nullptr;
  g2.a_src_rows = 0;
  g2.K = I;
  g2.n_out = H;
  g2.b_rows_per_group = H;
  g2.up_offset = 0;
  g2.out = f;
  g2.ldo = H;
  g2.out_fp32 = out_fp32;
  return launch_grouped_gemm(h, rows, w_d, E * H, g2, EPI_STORE, pick_bn(rows, E, H, false), stream);
}

// Dense SwiGLU expert on all T rows of x (the shared expert): GEMM1 + SwiGLU
// into h_ws [T, I], GEMM2 into out [T, H].
static int dense_swiglu(const void* x, int T, int H, int I, const void* w_gu, const void* w_d, int dtype, void* out,
                        uint16_t* h_ws, cudaStream_t stream) {
  GemmArgs g1{};
  g1.group_offsets = nullptr;
  g1.G = 1;
  g1.rows = T;
  g1.K = H;
  g1.n_out = I;
  g1.b_rows_per_group = 2 * I;
  g1.up_offset = I;
  g1.out = h_ws;
  g1.ldo = I;
  g1.bf16 = dtype == MOE_DTYPE_BF16;
  g1.status = device_status_ptr();
  g1.limit_ns = wait_limit_ns();
  int rc = launch_grouped_gemm(x, T, w_gu, 2 * I, g1, EPI_SWIGLU, pick_bn(T, 1, I, true), stream);
  if (rc) return rc;
  GemmArgs g2 = g1;
  g2.K = I;
  g2.n_out = H;
  g2.b_rows_per_group = H;
  g2.up_offset = 0;
  g2.out = out;
  g2.ldo = H;
  return launch_grouped_gemm(h_ws, T, w_d, H, g2, EPI_STORE, pick_bn(T, 1, H, false), stream);
}

static constexpr int kDecodeMaxT = 128;
static constexpr int kFusedMaxT = 16;

// The one-kernel split-K path for T <= 16; BIT_EXPERT_GEMM_DECODE_FUSED=0
// selects the two-GEMM decode path instead (for comparisons).
// BIT_EXPERT_GEMM_DENSE_GEMV=0 keeps a lone dense expert of a decode batch on the grouped GEMMs.
static bool dense_gemv_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* s = getenv("BIT_EXPERT_GEMM_DENSE_GEMV");
    on = (s && s[0] == '0') ? 0 : 1;
  }
  return on != 0;
}

static bool fused_decode_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* s = getenv("BIT_EXPERT_GEMM_DECODE_FUSED");
    on = (s && s[0] == '0') ? 0 : 1;
  }
  return on != 0;
}

// The split-K kernel keeps one 16-column accumulator per 128 down-projection
// rows in TMEM after 32 phase-A columns: H <= 3584 leaves room for its reads.
static constexpr int kFusedMaxH = 3584;
static bool use_fused(int T, int H) { return T <= kFusedMaxT && H <= kFusedMaxH && fused_decode_enabled(); }

// AWQ routed + 16-bit shared experts: the split-K partials for T <= 16, else
// the grouped AWQ call's workspace, reused afterwards by the shared expert's h.
static size_t experts_awq_ws_bytes(int T, int rows, int H, int I, int E) {
  if (use_fused(T, H)) return decode_fused_ws_bytes(rows, T, H, I);
  const size_t a = awq_ws_bytes(rows, H, I, E);
  const size_t b = size_t(T) * I * 2;
  return a > b ? a : b;
}

static size_t experts_ws_bytes(int T, int rows, int H, int I) {
  (void)H;
  if (use_fused(T, H)) return decode_fused_ws_bytes(rows, T, H, I);
  if (T <= kDecodeMaxT) return decode_ws_bytes(rows, T, I);
  WsCounter c;
  c.take<uint16_t>(size_t(rows > T ? rows : T) * I);
  return c.used;
}

}  // namespace moe

using namespace moe;

extern "C" {

int moe_abi_version(void) { return 2; }

const char* moe_last_error(void) { return g_err; }

int moe_device_status(int clear, void* stream) {
  MOE_CHECK_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int v = 0;
  MOE_CHECK_CUDA(cudaMemcpyFromSymbol(&v, g_status, sizeof(int)));
  if (clear) {
    const int z = 0;
    MOE_CHECK_CUDA(cudaMemcpyToSymbol(g_status, &z, sizeof(int)));
  }
  return v;
}

size_t moe_workspace_size(int op, int T, int H, int E, int k_slots, int I) {
  if (T < 0 || H < 0 || E < 0 || k_slots < 0 || I < 0) return 0;
  const int rows = T * k_slots;
  switch (op) {
    case MOE_OP_ROUTE_TOPK: return route_ws_bytes(T, E);
    case MOE_OP_PERMUTE: return permute_ws_bytes(T, E);
    case MOE_OP_ROUTE_PERMUTE: return route_permute_ws_bytes(T, E);
    case MOE_OP_SWIGLU_BF16: {
      WsCounter c;
      c.take<uint16_t>(size_t(rows) * I);
      // one dense expert on a decode batch: the GEMV path's FP32 partials
      if (E == 1 && dense_gemv_fits(T, H, I)) c.used = std::max(c.used, dense_gemv_ws_bytes(T, I));
      return c.used;
    }
    case MOE_OP_SWIGLU_AWQ_G32: return awq_ws_bytes(rows, H, I, E);
    case MOE_OP_EXPERTS_BF16: return experts_ws_bytes(T, rows, H, I);
    case MOE_OP_EXPERTS_AWQ_G32: return experts_awq_ws_bytes(T, rows, H, I, E);
    case MOE_OP_SWIGLU_NVFP4: return nvfp4_ws_bytes(rows, H, I, E);
    case MOE_OP_REFILL: return refill_ws_bytes(T, k_slots > 0 ? k_slots - 1 : 0);
    case MOE_OP_NVFP4_QUANTIZE: return nvfp4_quant_ws_bytes(1, T, H);
    default: return 0;
  }
}

int moe_route_topk(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
                   int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, void* ws, size_t ws_bytes,
                   void* stream) {
  MOE_REQUIRE(T >= 0 && H > 0 && E > 0, MOE_ERR_INVALID_ARG, "moe_route_topk: bad sizes T=%d H=%d E=%d", T, H, E);
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "moe_route_topk: dtype %d",
              dtype);
  MOE_REQUIRE(extra == 0 || extra == 1, MOE_ERR_INVALID_ARG, "moe_route_topk: extra must be 0 or 1");
  MOE_REQUIRE(k >= 1 && k + extra <= 16 && k + extra <= E, MOE_ERR_UNSUPPORTED,
              "moe_route_topk: need 1 <= k, k+extra <= 16 and <= E (k=%d extra=%d E=%d)", k, extra, E);
  MOE_REQUIRE(E <= 1024, MOE_ERR_UNSUPPORTED, "moe_route_topk: E=%d > 1024", E);
  MOE_REQUIRE(H % 64 == 0, MOE_ERR_UNSUPPORTED, "moe_route_topk: H=%d is not a multiple of 64", H);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(x && w_router && topk_idx && topk_w, MOE_ERR_INVALID_ARG, "moe_route_topk: null pointer");
  MOE_REQUIRE(aligned16(x) && aligned16(w_router), MOE_ERR_INVALID_ARG, "moe_route_topk: x / w_router not 16-byte aligned");
  return route_topk(x, T, H, w_router, bias, E, k, extra, dtype, topk_idx, topk_w, topk_logit, ws, ws_bytes,
                    static_cast<cudaStream_t>(stream));
}

int moe_permute(const int32_t* topk_idx, int T, int k_slots, int E, int32_t* expert_offsets, int32_t* row_token,
                int32_t* slot_row, void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(T >= 0 && k_slots >= 1 && k_slots <= 16 && E >= 1 && E <= 1024, MOE_ERR_UNSUPPORTED,
              "moe_permute: need T>=0, 1<=k_slots<=16, 1<=E<=1024 (T=%d k_slots=%d E=%d)", T, k_slots, E);
  MOE_REQUIRE(expert_offsets != nullptr, MOE_ERR_INVALID_ARG, "moe_permute: expert_offsets is null");
  MOE_REQUIRE(T == 0 || (topk_idx && row_token && slot_row), MOE_ERR_INVALID_ARG, "moe_permute: null pointer");
  MOE_REQUIRE(long(T) * k_slots < (1l << 31), MOE_ERR_UNSUPPORTED, "moe_permute: T*k_slots overflows int32");
  return permute(topk_idx, T, k_slots, E, expert_offsets, row_token, slot_row, ws, ws_bytes,
                 static_cast<cudaStream_t>(stream));
}

static int route_permute_entry(const char* fn, const void* x, int T, int H, const void* w_router, const float* bias,
                               int E, int k, int extra, int dtype, int32_t* topk_idx, float* topk_w,
                               float* topk_logit, int32_t* expert_offsets, int32_t* row_token, int32_t* slot_row,
                               void* ws, size_t ws_bytes, void* stream, const RouteNorm* norm) {
  MOE_REQUIRE(T >= 0 && H > 0 && E > 0, MOE_ERR_INVALID_ARG, "%s: bad sizes T=%d H=%d E=%d", fn, T, H, E);
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "%s: dtype %d", fn, dtype);
  MOE_REQUIRE(extra == 0 || extra == 1, MOE_ERR_INVALID_ARG, "%s: extra must be 0 or 1", fn);
  MOE_REQUIRE(k >= 1 && k + extra <= 16 && k + extra <= E, MOE_ERR_UNSUPPORTED,
              "%s: need 1 <= k, k+extra <= 16 and <= E (k=%d extra=%d E=%d)", fn, k, extra, E);
  MOE_REQUIRE(E <= 1024, MOE_ERR_UNSUPPORTED, "%s: E=%d > 1024", fn, E);
  MOE_REQUIRE(H % 64 == 0, MOE_ERR_UNSUPPORTED, "%s: H=%d is not a multiple of 64", fn, H);
  MOE_REQUIRE(long(T) * (k + extra) < (1l << 31), MOE_ERR_UNSUPPORTED, "%s: T*(k+extra) overflows", fn);
  MOE_REQUIRE(expert_offsets != nullptr, MOE_ERR_INVALID_ARG, "%s: expert_offsets is null", fn);
  if (norm) {
    MOE_REQUIRE(norm->w && norm->x_norm, MOE_ERR_INVALID_ARG, "%s: norm_w and x_norm must not be null", fn);
    MOE_REQUIRE((norm->gate_w == nullptr) == (norm->gate == nullptr), MOE_ERR_INVALID_ARG,
                "%s: w_shared_gate and shared_gate_out go together", fn);
    MOE_REQUIRE(norm->eps >= 0.f, MOE_ERR_INVALID_ARG, "%s: eps < 0", fn);
    MOE_REQUIRE(aligned16(norm->w) && aligned16(norm->x_norm) && (!norm->gate_w || aligned16(norm->gate_w)),
                MOE_ERR_INVALID_ARG, "%s: norm_w / x_norm / w_shared_gate not 16-byte aligned", fn);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) return permute(topk_idx, 0, k + extra, E, expert_offsets, row_token, slot_row, ws, ws_bytes, st);
  MOE_REQUIRE(x && w_router && topk_idx && topk_w && row_token && slot_row, MOE_ERR_INVALID_ARG, "%s: null pointer",
              fn);
  MOE_REQUIRE(aligned16(x) && aligned16(w_router), MOE_ERR_INVALID_ARG, "%s: x / w_router not 16-byte aligned", fn);
  return route_permute(x, T, H, w_router, bias, E, k, extra, dtype, topk_idx, topk_w, topk_logit, expert_offsets,
                       row_token, slot_row, ws, ws_bytes, st, norm);
}

int moe_route_permute(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k, int extra,
                      int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, int32_t* expert_offsets,
                      int32_t* row_token, int32_t* slot_row, void* ws, size_t ws_bytes, void* stream) {
  return route_permute_entry("moe_route_permute", x, T, H, w_router, bias, E, k, extra, dtype, topk_idx, topk_w,
                             topk_logit, expert_offsets, row_token, slot_row, ws, ws_bytes, stream, nullptr);
}

int moe_norm_route_permute(const void* x, int T, int H, const void* norm_w, float eps, const void* w_shared_gate,
                           const void* w_router, const float* bias, int E, int k, int extra, int dtype, void* x_norm,
                           float* shared_gate_out, int32_t* topk_idx, float* topk_w, float* topk_logit,
                           int32_t* expert_offsets, int32_t* row_token, int32_t* slot_row, void* ws, size_t ws_bytes,
                           void* stream) {
  RouteNorm n{norm_w, eps, w_shared_gate, x_norm, shared_gate_out};
  return route_permute_entry("moe_norm_route_permute", x, T, H, w_router, bias, E, k, extra, dtype, topk_idx, topk_w,
                             topk_logit, expert_offsets, row_token, slot_row, ws, ws_bytes, stream, &n);
}

int moe_grouped_swiglu_bf16(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T, int rows,
                            int H, int I, int E, const void* w_gate_up, const void* w_down, int dtype, int out_fp32,
                            void* f, void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(T >= 0 && rows >= 0 && E >= 1, MOE_ERR_INVALID_ARG, "moe_grouped_swiglu_bf16: bad sizes");
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_bf16: dtype %d", dtype);
  MOE_REQUIRE(H > 0 && I > 0 && H % 64 == 0 && I % 64 == 0, MOE_ERR_UNSUPPORTED,
              "moe_grouped_swiglu_bf16: H=%d and I=%d must be positive multiples of 64", H, I);
  MOE_REQUIRE(E <= kGemmMaxGroups, MOE_ERR_UNSUPPORTED, "moe_grouped_swiglu_bf16: E=%d > %d", E, kGemmMaxGroups);
  MOE_REQUIRE(row_token || rows == T, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_bf16: without row_token, rows (%d) must equal T (%d)", rows, T);
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(x && expert_offsets && w_gate_up && w_down && f, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_bf16: null pointer");
  MOE_REQUIRE(aligned16(x) && aligned16(w_gate_up) && aligned16(w_down) && aligned16(f), MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_bf16: operands must be 16-byte aligned");
  // one dense expert (E = 1, rows in order) on a decode batch: weight-streaming GEMVs
  if (E == 1 && !row_token && dense_gemv_fits(T, H, I) && dense_gemv_enabled())
    return dense_swiglu_gemv(x, expert_offsets, T, H, I, w_gate_up, w_down, dtype, out_fp32, f, ws, ws_bytes,
                             static_cast<cudaStream_t>(stream));
  return swiglu_bf16(x, row_token, expert_offsets, T, rows, H, I, E, w_gate_up, w_down, dtype, out_fp32, f, ws,
                     ws_bytes, static_cast<cudaStream_t>(stream));
}

int moe_experts_bf16(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T, int rows, int H,
                     int I, int E, const void* w_gate_up, const void* w_down, const void* w_sh_gate_up,
                     const void* w_sh_down, int dtype, int out_fp32, void* f, void* shared_out, void* ws,
                     size_t ws_bytes, void* stream) {
  MOE_REQUIRE(T >= 0 && rows >= 0 && E >= 1 && E <= kGemmMaxGroups, MOE_ERR_INVALID_ARG, "moe_experts_bf16: bad sizes");
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "moe_experts_bf16: dtype %d",
              dtype);
  MOE_REQUIRE(H > 0 && I > 0 && H % 128 == 0 && I % 64 == 0, MOE_ERR_UNSUPPORTED,
              "moe_experts_bf16: need H %% 128 == 0 and I %% 64 == 0 (H=%d I=%d)", H, I);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(x && row_token && expert_offsets && w_gate_up && w_down && w_sh_gate_up && w_sh_down && f && shared_out,
              MOE_ERR_INVALID_ARG, "moe_experts_bf16: null pointer");
  MOE_REQUIRE(aligned16(x) && aligned16(w_gate_up) && aligned16(w_down) && aligned16(w_sh_gate_up) &&
                  aligned16(w_sh_down) && aligned16(f) && aligned16(shared_out),
              MOE_ERR_INVALID_ARG, "moe_experts_bf16: operands must be 16-byte aligned");
  MOE_REQUIRE(ws_bytes >= experts_ws_bytes(T, rows, H, I), MOE_ERR_WORKSPACE,
              "moe_experts_bf16: workspace of %zu bytes is too small (need %zu)", ws_bytes,
              experts_ws_bytes(T, rows, H, I));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (use_fused(T, H))
    return decode_experts_fused(x, row_token, expert_offsets, T, rows, H, I, E, w_gate_up, w_down, w_sh_gate_up,
                                w_sh_down, dtype, out_fp32, f, shared_out, ws, ws_bytes, st);
  if (T <= kDecodeMaxT)
    return decode_experts_16bit(x, row_token, expert_offsets, T, rows, H, I, E, w_gate_up, w_down, w_sh_gate_up,
                                w_sh_down, dtype, out_fp32, f, shared_out, ws, ws_bytes, st);
  int rc = MOE_OK;
  if (rows > 0) {
    rc = swiglu_bf16(x, row_token, expert_offsets, T, rows, H, I, E, w_gate_up, w_down, dtype, out_fp32, f, ws,
                     ws_bytes, st);
    if (rc) return rc;
  }
  return dense_swiglu(x, T, H, I, w_sh_gate_up, w_sh_down, dtype, shared_out, static_cast<uint16_t*>(ws), st);
}

static int experts_awq_impl(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T, int rows,
                            int H, int I, int E, const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu,
                            const int32_t* qw_d, const int32_t* qz_d, const void* sc_d, const void* awq_packed,
                            const void* w_sh_gate_up, const void* w_sh_down, int dtype, int out_fp32, void* f,
                            void* shared_out, void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(T >= 0 && rows >= 0 && E >= 1 && E <= kGemmMaxGroups, MOE_ERR_INVALID_ARG,
              "moe_experts_awq_g32: bad sizes");
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "moe_experts_awq_g32: dtype=%d",
              dtype);
  MOE_REQUIRE(H > 0 && I > 0 && H % 128 == 0 && I % 64 == 0, MOE_ERR_UNSUPPORTED,
              "moe_experts_awq_g32: need H %% 128 == 0 and I %% 64 == 0 (H=%d I=%d)", H, I);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(x && row_token && expert_offsets && qw_gu && qz_gu && sc_gu && qw_d && qz_d && sc_d && w_sh_gate_up &&
                  w_sh_down && f && shared_out,
              MOE_ERR_INVALID_ARG, "moe_experts_awq_g32: null pointer");
  MOE_REQUIRE(aligned16(x) && aligned16(qw_gu) && aligned16(qz_gu) && aligned16(sc_gu) && aligned16(qw_d) &&
                  aligned16(qz_d) && aligned16(sc_d) && aligned16(w_sh_gate_up) && aligned16(w_sh_down) &&
                  aligned16(f) && aligned16(shared_out),
              MOE_ERR_INVALID_ARG, "moe_experts_awq_g32: operands must be 16-byte aligned");
  MOE_REQUIRE(ws_bytes >= experts_awq_ws_bytes(T, rows, H, I, E), MOE_ERR_WORKSPACE,
              "moe_experts_awq_g32: workspace of %zu bytes is too small (need %zu)", ws_bytes,
              experts_awq_ws_bytes(T, rows, H, I, E));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (use_fused(T, H))
    return decode_experts_fused_awq(x, row_token, expert_offsets, T, rows, H, I, E, qw_gu, qz_gu, sc_gu, qw_d, qz_d,
                                    sc_d, w_sh_gate_up, w_sh_down, dtype, out_fp32, f, shared_out, ws, ws_bytes, st,
                                    awq_packed);
  int rc = MOE_OK;
  if (rows > 0) {
    rc = grouped_swiglu_awq(x, row_token, expert_offsets, T, rows, H, I, E, qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d,
                            dtype, out_fp32, f, ws, ws_bytes, st, awq_packed);
    if (rc) return rc;
  }
  return dense_swiglu(x, T, H, I, w_sh_gate_up, w_sh_down, dtype, shared_out, static_cast<uint16_t*>(ws), st);
}

int moe_experts_awq_g32(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T, int rows, int H,
                        int I, int E, const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu,
                        const int32_t* qw_d, const int32_t* qz_d, const void* sc_d, const void* w_sh_gate_up,
                        const void* w_sh_down, int dtype, int out_fp32, void* f, void* shared_out, void* ws,
                        size_t ws_bytes, void* stream) {
  return experts_awq_impl(x, row_token, expert_offsets, T, rows, H, I, E, qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d,
                          nullptr, w_sh_gate_up, w_sh_down, dtype, out_fp32, f, shared_out, ws, ws_bytes, stream);
}

int moe_experts_awq_g32_prepacked(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T,
                                  int rows, int H, int I, int E, const int32_t* qw_gu, const int32_t* qz_gu,
                                  const void* sc_gu, const int32_t* qw_d, const int32_t* qz_d, const void* sc_d,
                                  const void* awq_packed, const void* w_sh_gate_up, const void* w_sh_down, int dtype,
                                  int out_fp32, void* f, void* shared_out, void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(awq_packed != nullptr || T == 0, MOE_ERR_INVALID_ARG, "moe_experts_awq_g32_prepacked: null awq_packed");
  MOE_REQUIRE(aligned16(awq_packed), MOE_ERR_INVALID_ARG,
              "moe_experts_awq_g32_prepacked: awq_packed must be 16-byte aligned");
  return experts_awq_impl(x, row_token, expert_offsets, T, rows, H, I, E, qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d,
                          awq_packed, w_sh_gate_up, w_sh_down, dtype, out_fp32, f, shared_out, ws, ws_bytes, stream);
}

size_t moe_awq_packed_bytes(int E, int H, int I) {
  if (E < 1 || H <= 0 || I <= 0 || H % 128 || I % 64) return 0;
  return awq_packed_bytes(E, H, I);
}

int moe_awq_prepack_g32(const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu, const int32_t* qw_d,
                        const int32_t* qz_d, const void* sc_d, int E, int H, int I, void* out, size_t out_bytes,
                        void* stream) {
  MOE_REQUIRE(E >= 1 && E <= kGemmMaxGroups, MOE_ERR_INVALID_ARG, "moe_awq_prepack_g32: E=%d", E);
  MOE_REQUIRE(H > 0 && I > 0 && H % 128 == 0 && I % 64 == 0, MOE_ERR_UNSUPPORTED,
              "moe_awq_prepack_g32: need H %% 128 == 0 and I %% 64 == 0 (H=%d I=%d)", H, I);
  MOE_REQUIRE(qw_gu && qz_gu && sc_gu && qw_d && qz_d && sc_d && out, MOE_ERR_INVALID_ARG,
              "moe_awq_prepack_g32: null pointer");
  MOE_REQUIRE(aligned16(out), MOE_ERR_INVALID_ARG, "moe_awq_prepack_g32: out must be 16-byte aligned");
  const size_t need = awq_packed_bytes(E, H, I);
  MOE_REQUIRE(out_bytes >= need, MOE_ERR_WORKSPACE, "moe_awq_prepack_g32: out holds %zu bytes, need %zu", out_bytes,
              need);
  return awq_prepack(qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d, E, H, I, out, static_cast<cudaStream_t>(stream));
}

int moe_grouped_swiglu_awq_g32(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T,
                               int rows, int H, int I, int E, const int32_t* qw_gu, const int32_t* qz_gu,
                               const void* sc_gu, const int32_t* qw_d, const int32_t* qz_d, const void* sc_d,
                               int dtype, int out_fp32, void* f, void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(T >= 0 && rows >= 0 && E >= 1 && E <= kGemmMaxGroups, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_awq_g32: bad sizes");
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_awq_g32: dtype=%d", dtype);
  MOE_REQUIRE(H > 0 && I > 0 && H % 64 == 0 && I % 64 == 0, MOE_ERR_UNSUPPORTED,
              "moe_grouped_swiglu_awq_g32: H=%d and I=%d must be positive multiples of 64", H, I);
  MOE_REQUIRE(row_token || rows == T, MOE_ERR_INVALID_ARG, "moe_grouped_swiglu_awq_g32: without row_token rows must equal T");
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(x && expert_offsets && qw_gu && qz_gu && sc_gu && qw_d && qz_d && sc_d && f, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_awq_g32: null pointer");
  return grouped_swiglu_awq(x, row_token, expert_offsets, T, rows, H, I, E, qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d,
                            dtype, out_fp32, f, ws, ws_bytes, static_cast<cudaStream_t>(stream), nullptr);
}

int moe_awq_dequant_g32(const int32_t* qweight, const int32_t* qzeros, const void* scales, int batch, int K, int N,
                        int dtype, void* out, void* stream) {
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "moe_awq_dequant_g32: dtype=%d",
              dtype);
  MOE_REQUIRE(batch >= 0 && K >= 0 && N >= 0 && K % 32 == 0 && N % 8 == 0, MOE_ERR_UNSUPPORTED,
              "moe_awq_dequant_g32: need K %% 32 == 0 and N %% 8 == 0 (K=%d N=%d)", K, N);
  if (long(batch) * K * N == 0) return MOE_OK;
  MOE_REQUIRE(qweight && qzeros && scales && out, MOE_ERR_INVALID_ARG, "moe_awq_dequant_g32: null pointer");
  MOE_REQUIRE(aligned16(scales) && aligned16(out), MOE_ERR_INVALID_ARG,
              "moe_awq_dequant_g32: scales / out must be 16-byte aligned");
  return awq_dequant(qweight, qzeros, scales, batch, K, N, dtype, out, static_cast<cudaStream_t>(stream));
}

int moe_nvfp4_quantize(const void* v, int batch, int rows, int K, int dtype, const float* global_scale_in,
                       uint8_t* codes, uint8_t* sf, float* global_scale_out, void* ws, size_t ws_bytes,
                       void* stream) {
  MOE_REQUIRE(batch >= 0 && rows >= 0 && K > 0 && K % 16 == 0, MOE_ERR_UNSUPPORTED,
              "moe_nvfp4_quantize: need K a positive multiple of 16 (K=%d)", K);
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "moe_nvfp4_quantize: dtype");
  if (batch == 0 || rows == 0) return MOE_OK;
  MOE_REQUIRE(v && codes && sf && global_scale_out, MOE_ERR_INVALID_ARG, "moe_nvfp4_quantize: null pointer");
  return nvfp4_quantize(v, batch, rows, K, dtype, global_scale_in, codes, sf, global_scale_out, ws, ws_bytes,
                        static_cast<cudaStream_t>(stream));
}

int moe_grouped_swiglu_nvfp4(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T, int rows,
                             int H, int I, int E, const uint8_t* w_gu, const uint8_t* sf_gu, const float* gs_gu,
                             const uint8_t* w_d, const uint8_t* sf_d, const float* gs_d, const float* act_gs_in,
                             float* act_gs_out, int out_fp32, void* f, void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(T >= 0 && rows >= 0 && E >= 1 && E <= kGemmMaxGroups, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_nvfp4: bad sizes");
  MOE_REQUIRE(H > 0 && I > 0 && H % 128 == 0 && I % 128 == 0, MOE_ERR_UNSUPPORTED,
              "moe_grouped_swiglu_nvfp4: H=%d and I=%d must be positive multiples of 128", H, I);
  MOE_REQUIRE(row_token || rows == T, MOE_ERR_INVALID_ARG, "moe_grouped_swiglu_nvfp4: without row_token rows must equal T");
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(x && expert_offsets && w_gu && sf_gu && gs_gu && w_d && sf_d && gs_d && f, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_nvfp4: null pointer");
  return grouped_swiglu_nvfp4(x, row_token, expert_offsets, T, rows, H, I, E, w_gu, sf_gu, gs_gu, w_d, sf_d, gs_d,
                              act_gs_in, act_gs_out, out_fp32, f, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                              nullptr, nullptr);
}

size_t moe_nvfp4_packed_sf_bytes(int E, int rows_per_expert, int K, int swiglu) {
  if (E < 1 || rows_per_expert <= 0 || K <= 0 || rows_per_expert % 128 || K % 128) return 0;
  return nvfp4_packed_sf_bytes(E, rows_per_expert, K, swiglu);
}

int moe_nvfp4_prepack_sf(const uint8_t* sf, int E, int rows_per_expert, int K, int swiglu, uint8_t* out,
                         size_t out_bytes, void* stream) {
  MOE_REQUIRE(E >= 1 && E <= kGemmMaxGroups, MOE_ERR_INVALID_ARG, "moe_nvfp4_prepack_sf: E=%d", E);
  MOE_REQUIRE(rows_per_expert > 0 && K > 0 && rows_per_expert % 128 == 0 && K % 128 == 0, MOE_ERR_UNSUPPORTED,
              "moe_nvfp4_prepack_sf: rows_per_expert=%d and K=%d must be positive multiples of 128",
              rows_per_expert, K);
  MOE_REQUIRE(swiglu == 0 || swiglu == 1, MOE_ERR_INVALID_ARG, "moe_nvfp4_prepack_sf: swiglu=%d", swiglu);
  MOE_REQUIRE(sf && out, MOE_ERR_INVALID_ARG, "moe_nvfp4_prepack_sf: null pointer");
  const size_t need = nvfp4_packed_sf_bytes(E, rows_per_expert, K, swiglu);
  MOE_REQUIRE(out_bytes >= need, MOE_ERR_WORKSPACE, "moe_nvfp4_prepack_sf: out holds %zu bytes, need %zu",
              out_bytes, need);
  return nvfp4_prepack_sf(sf, E, rows_per_expert, K, swiglu, out, static_cast<cudaStream_t>(stream));
}

int moe_grouped_swiglu_nvfp4_prepacked(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T,
                                       int rows, int H, int I, int E, const uint8_t* w_gu, const uint8_t* sf_gu_packed,
                                       const float* gs_gu, const uint8_t* w_d, const uint8_t* sf_d_packed,
                                       const float* gs_d, const float* act_gs_in, float* act_gs_out, int out_fp32,
                                       void* f, void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(T >= 0 && rows >= 0 && E >= 1 && E <= kGemmMaxGroups, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_nvfp4_prepacked: bad sizes");
  MOE_REQUIRE(H > 0 && I > 0 && H % 128 == 0 && I % 128 == 0, MOE_ERR_UNSUPPORTED,
              "moe_grouped_swiglu_nvfp4_prepacked: H=%d and I=%d must be positive multiples of 128", H, I);
  MOE_REQUIRE(row_token || rows == T, MOE_ERR_INVALID_ARG,
              "moe_grouped_swiglu_nvfp4_prepacked: without row_token rows must equal T");
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(x && expert_offsets && w_gu && sf_gu_packed && gs_gu && w_d && sf_d_packed && gs_d && f,
              MOE_ERR_INVALID_ARG, "moe_grouped_swiglu_nvfp4_prepacked: null pointer");
  return grouped_swiglu_nvfp4(x, row_token, expert_offsets, T, rows, H, I, E, w_gu, nullptr, gs_gu, w_d, nullptr, gs_d,
                              act_gs_in, act_gs_out, out_fp32, f, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                              sf_gu_packed, sf_d_packed);
}

int moe_combine(const void* f, int f_fp32, const int32_t* slot_row, int k_slots, const float* topk_w,
                const void* shared_out, const float* shared_gate, int T, int k, int H, int dtype, void* y,
                void* stream) {
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= k_slots && k_slots <= 16, MOE_ERR_INVALID_ARG,
              "moe_combine: need 1 <= k <= k_slots <= 16");
  MOE_REQUIRE(H > 0 && H % 8 == 0, MOE_ERR_UNSUPPORTED, "moe_combine: H=%d must be a multiple of 8", H);
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "moe_combine: dtype %d", dtype);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(f && slot_row && topk_w && y, MOE_ERR_INVALID_ARG, "moe_combine: null pointer");
  return combine(f, f_fp32, slot_row, k_slots, topk_w, shared_out, shared_gate, T, k, H, dtype, y,
                 static_cast<cudaStream_t>(stream));
}

int razor_refill_rms_accumulate(const void* f, int f_fp32, const int32_t* slot_row, const int32_t* topk_idx,
                                const float* topk_logit, const int32_t* expert_offsets, int T, int k, int H, int E,
                                double* sum_sq, int64_t* count, const void* shared_out, void* y_out, int dtype,
                                void* ws, size_t ws_bytes, void* stream) {
  (void)topk_idx;  // the expert of each row is implied by expert_offsets
  MOE_REQUIRE(T >= 0 && k >= 1 && k + 1 <= 16 && E >= 1 && E <= 1024, MOE_ERR_UNSUPPORTED,
              "razor_refill_rms_accumulate: need 1 <= k, k+1 <= 16, 1 <= E <= 1024");
  MOE_REQUIRE(H > 0 && H % 8 == 0, MOE_ERR_UNSUPPORTED, "razor_refill_rms_accumulate: H=%d must be a multiple of 8", H);
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG,
              "razor_refill_rms_accumulate: dtype %d", dtype);
  MOE_REQUIRE(sum_sq && count && expert_offsets, MOE_ERR_INVALID_ARG, "razor_refill_rms_accumulate: null pointer");
  MOE_REQUIRE(T == 0 || (f && slot_row && topk_logit), MOE_ERR_INVALID_ARG,
              "razor_refill_rms_accumulate: null pointer");
  return refill(f, f_fp32, slot_row, topk_logit, expert_offsets, T, k, H, E, sum_sq, count, shared_out, y_out, dtype,
                ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int razor_select(const double* sum_sq, const int64_t* count, int E, int keep, int32_t* kept_idx, int32_t* ranking,
                 double* score, void* stream) {
  MOE_REQUIRE(E >= 1 && E <= 1024, MOE_ERR_UNSUPPORTED, "razor_select: E=%d outside [1, 1024]", E);
  MOE_REQUIRE(keep >= 0 && keep <= E, MOE_ERR_INVALID_ARG, "razor_select: keep=%d outside [0, E]", keep);
  MOE_REQUIRE(sum_sq && count && (kept_idx || keep == 0), MOE_ERR_INVALID_ARG, "razor_select: null pointer");
  return select_experts(sum_sq, count, E, keep, kept_idx, ranking, score, static_cast<cudaStream_t>(stream));
}

int moe_shared_gate(const void* x, int T, int H, const void* w_gate, int dtype, float* gate, void* stream) {
  MOE_REQUIRE(T >= 0 && H >= 8 && H % 8 == 0, MOE_ERR_UNSUPPORTED, "moe_shared_gate: T=%d H=%d (need H %% 8 == 0)", T,
              H);
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "moe_shared_gate: dtype=%d",
              dtype);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(x && w_gate && gate, MOE_ERR_INVALID_ARG, "moe_shared_gate: null pointer");
  MOE_REQUIRE(aligned16(x) && aligned16(w_gate), MOE_ERR_INVALID_ARG,
              "moe_shared_gate: x and w_gate must be 16-byte aligned");
  return shared_gate(x, T, H, w_gate, dtype, gate, static_cast<cudaStream_t>(stream));
}

int moe_rmsnorm(const void* x, int T, int H, const void* w, float eps, int dtype, void* y, void* stream) {
  MOE_REQUIRE(T >= 0 && H >= 8 && H % 8 == 0, MOE_ERR_UNSUPPORTED, "moe_rmsnorm: T=%d H=%d (need H %% 8 == 0)", T,
              H);
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "moe_rmsnorm: dtype=%d", dtype);
  MOE_REQUIRE(eps >= 0.0f, MOE_ERR_INVALID_ARG, "moe_rmsnorm: eps must be >= 0");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(x && w && y, MOE_ERR_INVALID_ARG, "moe_rmsnorm: null pointer");
  MOE_REQUIRE(aligned16(x) && aligned16(w) && aligned16(y), MOE_ERR_INVALID_ARG,
              "moe_rmsnorm: x, w and y must be 16-byte aligned");
  return rmsnorm(x, T, H, w, eps, dtype, y, static_cast<cudaStream_t>(stream));
}

int razor_router_norm(const void* w_router, int E, int H, int dtype, double* sum_sq, int64_t* count, void* stream) {
  MOE_REQUIRE(E >= 1 && H >= 1, MOE_ERR_INVALID_ARG, "razor_router_norm: E=%d H=%d must be positive", E, H);
  MOE_REQUIRE(dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_F16, MOE_ERR_INVALID_ARG, "razor_router_norm: dtype=%d",
              dtype);
  MOE_REQUIRE(w_router && sum_sq, MOE_ERR_INVALID_ARG, "razor_router_norm: null pointer");
  return router_norm(w_router, E, H, dtype, sum_sq, count, static_cast<cudaStream_t>(stream));
}

int razor_slice(const void* src, int E, size_t bytes_per_expert, const int32_t* kept_idx, int keep, void* dst,
                void* stream) {
  MOE_REQUIRE(E >= 1, MOE_ERR_INVALID_ARG, "razor_slice: E=%d must be positive", E);
  MOE_REQUIRE(keep >= 0 && keep <= E && keep <= 65535, MOE_ERR_INVALID_ARG,
              "razor_slice: keep=%d outside [0, min(E, 65535)]", keep);
  if (keep == 0 || bytes_per_expert == 0) return MOE_OK;
  MOE_REQUIRE(src && dst && kept_idx, MOE_ERR_INVALID_ARG, "razor_slice: null pointer");
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
  const uintptr_t s1 = s0 + uintptr_t(E) * bytes_per_expert, d1 = d0 + uintptr_t(keep) * bytes_per_expert;
  MOE_REQUIRE(d1 <= s0 || s1 <= d0, MOE_ERR_INVALID_ARG, "razor_slice: dst overlaps src");
  return slice_experts(src, E, bytes_per_expert, kept_idx, keep, dst, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
