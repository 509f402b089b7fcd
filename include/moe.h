/*
 * bit_expert_gemm_b200 -- C ABI of the routed-expert MoE layer and RAZOR
 * Refill-RMS scoring on one NVIDIA B200 (sm_100a).
 *
 * The operations follow these pages (cited by page title and section):
 *   [ARCH]  Qwen3.8-Flash-Next architecture fact sheet (archdb model page):
 *           entries "Routed experts per MoE layer" (512), "Routed experts
 *           selected per token" (10), "Always-on experts per MoE layer" (1),
 *           "Intermediate width of one routed expert" (640), "Gating function
 *           over expert logits" (softmax), "Selected expert weights are
 *           renormalized to sum to 1" (yes), "FFN activation" (SwiGLU),
 *           "Clamping of GLU gate / up activations" (none), "FFN projections
 *           have bias terms" (no).
 *   [AWQ]   Qwen3.8-Flash-Next-AWQ-g32 card, sections "Checkpoint" (format:
 *           asymmetric W4A16, group 32, integer zero point, GEMM packing, FP16
 *           expert scales) and "Calibration" (code rule
 *           clip(round(w/scale + zero), 0, 15)).
 *   [NVFP4] Qwen3.8-Flash-Next-RAZOR-96B-A6B-NVFP4 card, component table
 *           (routed experts in NVFP4 for weights and activations: FP4 values
 *           in groups of 16, an FP8 scale per group, an FP32 scale per
 *           tensor; the shared expert and the router stay BF16).
 *   [RAZOR] Qwen3.8-Flash-Next-RAZOR-65B-A6B-E256of512 card, section
 *           "Selection and calibration" (Refill-RMS score, conditional RMS
 *           aggregation, keep the top 256 / 384, additive statistics) and the
 *           opening paragraphs (experts and router rows sliced in matching
 *           order; keep manifest in output order).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every function returns an int status (MOE_OK or an MOE_ERR_* code).  On
 *    error, moe_last_error() returns a message for the calling host thread.
 *    Argument checks happen on the host before anything is launched; a call
 *    that fails its checks launches nothing.
 *  - Tensor arguments are DEVICE pointers owned by the caller, contiguous,
 *    row-major, unless a comment says otherwise.  The library never allocates
 *    or frees device memory and never synchronises the host; all work is
 *    enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *    default stream).
 *  - Scratch memory is passed as (ws, ws_bytes); its required size is
 *    returned by moe_workspace_size().  The workspace must be 256-byte
 *    aligned and must not be used by another call that may run concurrently.
 *  - "dtype" is MOE_DTYPE_BF16 or MOE_DTYPE_F16 and describes the 16-bit
 *    activations and 16-bit weights of the call.
 *  - Weights are stored out x in (row j of a projection produces output
 *    feature j).  The stacked gate/up projection of an expert holds the gate
 *    rows 0..I-1 followed by the up rows I..2I-1.
 *  - Device-side waits are bounded.  A wait that runs out records
 *    MOE_ERR_TIMEOUT in a device status word that moe_device_status() reads.
 */
#ifndef BIT_EXPERT_GEMM_B200_MOE_H_
#define BIT_EXPERT_GEMM_B200_MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, negative size, index out of range   */
  MOE_ERR_UNSUPPORTED = 2, /* a shape the kernels do not handle (see each call) */
  MOE_ERR_WORKSPACE = 3,   /* ws too small or misaligned                          */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime call failed                          */
  MOE_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out                  */
};

enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_F16 = 1 };

/* Operation ids for moe_workspace_size(). */
enum {
  MOE_OP_ROUTE_TOPK = 0,
  MOE_OP_PERMUTE = 1,
  MOE_OP_SWIGLU_BF16 = 2,
  MOE_OP_SWIGLU_AWQ_G32 = 3,
  MOE_OP_SWIGLU_NVFP4 = 4,
  MOE_OP_REFILL = 5,
  MOE_OP_NVFP4_QUANTIZE = 6,
  MOE_OP_EXPERTS_BF16 = 7,
  MOE_OP_ROUTE_PERMUTE = 8,
  MOE_OP_EXPERTS_AWQ_G32 = 9
};

/* Version of this header's ABI. */
MOE_API int moe_abi_version(void);

/* Message of the last failed call on this host thread ("" if none). */
MOE_API const char* moe_last_error(void);

/* Synchronises `stream`, returns the device status word of the current
 * device (MOE_OK, or MOE_ERR_TIMEOUT if a bounded device-side wait ran out,
 * or MOE_ERR_INVALID_ARG if a kernel met an out-of-range index), and clears
 * it when `clear` is non-zero.  This is the only call that synchronises. */
MOE_API int moe_device_status(int clear, void* stream);

/* Self-test of the bounded device-side waits (failure handling; the pages
 * have no counterpart).  Launches one CTA that does what a TMA / tcgen05
 * kernel of this library does when a wait never completes: one role starts
 * a bulk copy, then waits on an mbarrier that nothing completes, with a
 * limit of limit_us microseconds; the wait runs out, records MOE_ERR_TIMEOUT
 * in the device status word and raises the CTA's abort flag, and the role
 * waits (bounded) for its copy to land.  A second role waiting on the same
 * barrier with a 100x longer limit stops on the abort flag, drains the
 * tensor core, and the CTA frees its tensor memory and exits.  result [2]
 * int32 on the device: result[0] = 1 if the first role's wait gave up,
 * result[1] = 1 if the second role's did.  The launch ends about 64 ms
 * after limit_us at most (the flags are polled every 64 suspended tries).
 * Clear the status word (moe_device_status(1, ...)) before the call and read
 * it after; the GPU context stays usable.  Limits: 100 <= limit_us <=
 * 1000000, else MOE_ERR_UNSUPPORTED with nothing launched. */
MOE_API int moe_selftest_bounded_wait(int limit_us, int32_t* result, void* stream);

/* Bytes of workspace that operation `op` needs for the given sizes
 * (T tokens, hidden size H, E experts, k_slots selected slots per token,
 * intermediate width I).  Returns 0 for an unknown op.  The result is an
 * upper bound valid for any routing of those sizes. */
MOE_API size_t moe_workspace_size(int op, int T, int H, int E, int k_slots, int I);

/* ---------------------------------------------------------------------------
 * Router, softmax over all E experts, top-k, renormalised weights [ARCH].
 *
 *   l[t, e]  = sum_h x[t, h] * w_router[e, h] + bias[e]      (FP32 accumulate)
 *   S_t      = the k experts of largest l (equivalently of largest softmax
 *              probability), ties to the lower expert index, in descending
 *              order; with extra = 1 the rank-(k+1) expert r_t is appended
 *              (the expert Refill-RMS promotes [RAZOR]).
 *   topk_w   = softmax(l)[S] / sum softmax(l)[S]  (sums to 1 over the k slots)
 *
 * x [T, H] and w_router [E, H] are 16-bit (dtype); bias [E] FP32 or NULL.
 * Outputs: topk_idx [T, k+extra] int32, topk_w [T, k] FP32, topk_logit
 * [T, k+extra] FP32 (the logits l of the selected experts, bias included; may
 * be NULL).  Limits: 1 <= k, k + extra <= 16, k + extra <= E <= 1024,
 * H % 64 == 0.  Workspace: MOE_OP_ROUTE_TOPK.
 * ------------------------------------------------------------------------- */
MOE_API int moe_route_topk(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k,
                   int extra, int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit, void* ws,
                   size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Permutation of the (token, slot) assignments by expert, so that each
 * routed expert [ARCH] ("Routed experts selected per token") runs once over
 * the rows of all tokens that selected it: histogram, exclusive scan,
 * scatter.  The pages fix no order; this one is deterministic: expert blocks in
 * ascending expert id, and inside one expert ascending token index (every
 * token selects an expert at most once).
 *
 * topk_idx [T, k_slots] int32 in [0, E) -> expert_offsets [E+1] int32
 * (expert e owns permuted rows expert_offsets[e] .. expert_offsets[e+1]-1),
 * row_token [T*k_slots] int32 (token of each permuted row), slot_row
 * [T, k_slots] int32 (permuted row of each assignment).  An index outside
 * [0, E) is skipped and recorded as MOE_ERR_INVALID_ARG in the device status
 * word; duplicate experts within one token's slots are not allowed.
 * Limits: E <= 1024, k_slots <= 16.  Workspace: MOE_OP_PERMUTE.
 * ------------------------------------------------------------------------- */
MOE_API int moe_permute(const int32_t* topk_idx, int T, int k_slots, int E, int32_t* expert_offsets, int32_t* row_token,
                int32_t* slot_row, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_route_topk followed by moe_permute of its topk_idx (k_slots = k +
 * extra), in one call, with the arguments and outputs of both ([ARCH]
 * gating and selection; [RAZOR] rank k + 1 when extra = 1).  For T <= 128
 * (decode) everything runs in one cooperative kernel (grid-wide barriers
 * between the logits, the top-k and the permutation); larger T takes the two
 * calls' kernels in sequence.  Outputs equal those of the two calls, except
 * that a near-tie among logits may resolve differently, as the logits are
 * summed in another order.  Limits: those of both calls; for T <= 128 also
 * 8 * H <= 204800 (the staged router rows).  Workspace: MOE_OP_ROUTE_PERMUTE.
 * ------------------------------------------------------------------------- */
MOE_API int moe_route_permute(const void* x, int T, int H, const void* w_router, const float* bias, int E, int k,
                              int extra, int dtype, int32_t* topk_idx, float* topk_w, float* topk_logit,
                              int32_t* expert_offsets, int32_t* row_token, int32_t* slot_row, void* ws,
                              size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Pre-MoE RMSNorm, the optional shared-expert gate and moe_route_permute in
 * one call [ARCH] (normalisation entries: RMSNorm before the block, gain
 * 1 + w, epsilon 1e-6; [AWQ] "Checkpoint": the shared-expert gate tensor).
 *
 *   x_norm[t, h] = x[t, h] / sqrt(mean_h x[t, :]^2 + eps) * (1 + norm_w[h])
 *                  (FP32, rounded to dtype: the block's 16-bit input)
 *   shared_gate_out[t] = 1 / (1 + exp(-x_norm[t, :] . w_shared_gate))
 *   then moe_route_permute of x_norm (same outputs and limits).
 *
 * x, x_norm [T, H] dtype (x_norm may be x); norm_w [H] dtype; w_shared_gate
 * [H] dtype or NULL, and shared_gate_out [T] FP32 then NULL too.  The experts
 * and the shared expert of the layer take x_norm as their input.  For T <=
 * 128 the normalisation is a first phase of the cooperative routing kernel
 * (one more grid barrier); larger T run one normalisation kernel (one read
 * of x, the gate from the values it writes) before the routing of x_norm.
 * Workspace: MOE_OP_ROUTE_PERMUTE.
 * ------------------------------------------------------------------------- */
MOE_API int moe_norm_route_permute(const void* x, int T, int H, const void* norm_w, float eps,
                                   const void* w_shared_gate, const void* w_router, const float* bias, int E, int k,
                                   int extra, int dtype, void* x_norm, float* shared_gate_out, int32_t* topk_idx,
                                   float* topk_w, float* topk_logit, int32_t* expert_offsets, int32_t* row_token,
                                   int32_t* slot_row, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism over `world` ranks ([NVFP4] serving example: expert
 * parallelism over eight GPUs).  Rank d owns the routed experts
 * [d * E/world, (d+1) * E/world).  A rank's permuted rows (moe_permute:
 * experts ascending) are therefore already grouped by destination rank.
 *
 * moe_ep_plan: expert_offsets [E+1] (device) -> row_local_expert [rows] int32,
 * the index of each permuted row's expert among its destination's experts
 * (e mod E/world), and send_counts [world] int32, the rows each destination
 * receives (offsets[(d+1) E/world] - offsets[d E/world]).  Limits: E a
 * multiple of world.
 *
 * moe_gather_rows: out[r] = src[index[r]] for whole 16-bit rows of H
 * elements: src [src_rows, H], index [rows] int32, out [rows, H] (H % 8 == 0,
 * 16-byte aligned rows).  An index outside [0, src_rows) writes a zero row
 * and records MOE_ERR_INVALID_ARG in the device status word.  Used for the x
 * rows of the send order and for the experts' outputs in the received order.
 * ------------------------------------------------------------------------- */
MOE_API int moe_ep_plan(const int32_t* expert_offsets, int E, int world, int rows, int32_t* row_local_expert,
                        int32_t* send_counts, void* stream);
MOE_API int moe_gather_rows(const void* src, int src_rows, int H, const int32_t* index, int rows, void* out,
                            void* stream);

/* ---------------------------------------------------------------------------
 * moe_permute without a workspace argument.  The pages have no counterpart:
 * this exists for callers that only receive input and output buffers from
 * the framework hosting them (a plug-in interface without an allocator, a
 * runtime with its own fixed memory pool, a latency-critical step where a
 * cudaMalloc could synchronise the device) and so cannot pass scratch memory.
 * Same arguments, outputs and order as moe_permute.  Its scratch is a fixed
 * array of about 4 MiB inside the library's device image, held on every GPU
 * that loads the library until the process exits; the call allocates and
 * frees nothing.  Limit: E * ceil(T/32) <= 524288 (e.g. E = 512 experts,
 * T = 32768 tokens); larger batches are rejected with MOE_ERR_UNSUPPORTED
 * (use moe_permute with a workspace).  The first call on a device looks up
 * the array's device address with that device current; make that first call
 * before any stream capture.  The address is cached per device for the life
 * of the process (host threads may make the first call concurrently): a
 * process that resets a device (cudaDeviceReset) must not call this on that
 * device afterwards.  All calls on a device share the array and it
 * keeps the last call's contents (the part that must start at zero is
 * cleared on the call's stream); calls whose work overlaps on the GPU, e.g.
 * on unordered streams, race on it.
 * ------------------------------------------------------------------------- */
MOE_API int moe_permute_noalloc(const int32_t* topk_idx, int T, int k_slots, int E, int32_t* expert_offsets,
                                int32_t* row_token, int32_t* slot_row, void* stream);

/* ---------------------------------------------------------------------------
 * Grouped SwiGLU expert FFN with 16-bit weights [ARCH]:
 *   for every expert e and every permuted row r of e (expert_offsets):
 *     g = x[row_token[r]] . Wg_e^T,  u = x[row_token[r]] . Wu_e^T   (FP32 acc)
 *     h = silu(g) * u,  silu(g) = g / (1 + exp(-g)), rounded to dtype
 *     f[r] = h . Wd_e^T                                            (FP32 acc)
 *
 * x [T, H] dtype; row_token [rows] int32, or NULL for the identity (rows
 * must then equal T: this computes a dense expert such as the shared expert
 * with E = 1 and expert_offsets = {0, T}); expert_offsets [E+1] int32 on the
 * device, expert_offsets[E] == rows; w_gate_up [E, 2I, H] dtype; w_down
 * [E, H, I] dtype; f [rows, H], FP32 when out_fp32 != 0, else dtype.
 * A dense expert (E = 1, row_token NULL) on T <= 16 tokens with H % 256 == 0
 * runs as two weight-streaming GEMV launches over all SMs (FP32 sums, h
 * rounded to dtype) instead of the tiled GEMMs.
 * Limits: H % 64 == 0, I % 64 == 0, E <= 1024.  Workspace:
 * MOE_OP_SWIGLU_BF16 (holds h, or the GEMV path's FP32 partials).
 * ------------------------------------------------------------------------- */
MOE_API int moe_grouped_swiglu_bf16(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T,
                            int rows, int H, int I, int E, const void* w_gate_up, const void* w_down, int dtype,
                            int out_fp32, void* f, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Routed experts and the shared expert of one layer in one call [ARCH]: the
 * routed part is moe_grouped_swiglu_bf16 (f [rows, H]), the shared part the
 * same SwiGLU on every token with w_sh_gate_up [2I, H] and w_sh_down [H, I]
 * (shared_out [T, H] dtype; the shared expert has the routed experts' width
 * I).  Decode-sized batches run as weight-streaming tensor-core GEMMs with
 * the weights as the M operand and the few tokens as N, routed and shared
 * work items in the same launches: for T <= 16 one kernel computes, per
 * block of 64 intermediate features, gate/up, SwiGLU and that block's slice
 * of the down projection, FP32 partials that a second kernel sums in a fixed
 * order (no wait between the two GEMMs); for 16 < T <= 128 the first GEMM
 * applies SwiGLU in its epilogue and writes h [rows + T, I] (dtype) to the
 * workspace, the second reads it back.  Larger T uses the grouped prefill
 * GEMMs.  row_token is required.
 * Limits: H % 128 == 0, I % 64 == 0.  Workspace: MOE_OP_EXPERTS_BF16.
 * ------------------------------------------------------------------------- */
MOE_API int moe_experts_bf16(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T, int rows,
                             int H, int I, int E, const void* w_gate_up, const void* w_down, const void* w_sh_gate_up,
                             const void* w_sh_down, int dtype, int out_fp32, void* f, void* shared_out, void* ws,
                             size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Grouped SwiGLU expert FFN with AWQ W4A16 asymmetric group-32 weights [AWQ].
 * Same maths as moe_grouped_swiglu_bf16 with 16-bit activations of `dtype`,
 * h rounded to that type, and each weight dequantised exactly as
 *     MOE_DTYPE_F16:  W[k, n] = fp16_rn((q[k, n] - z[k/32, n]) * s[k/32, n])
 * (the inverse of the card's code rule), or in the BF16 mode the card's
 * stock-runtime paragraph describes (FP16 scales rounded to BF16 on load,
 * BF16 arithmetic, at most 0.4 % relative change per scale):
 *     MOE_DTYPE_BF16: W[k, n] = bf16_rn((q - z) * bf16_rn(s)).
 * The stored scales are FP16 in both modes.  Layout per projection with input
 * dim K and output dim N, input-major ("GEMM" orientation):
 *     qweight [K, N/8] int32: word w of row k holds the codes of output
 *             columns 8w .. 8w+7, column 8w+i in bits 4i .. 4i+3;
 *     qzeros  [K/32, N/8] int32, packed the same way;
 *     scales  [K/32, N] FP16.
 * Gate/up projection: K = H, N = 2I (gate columns 0..I-1, up I..2I-1):
 *   qw_gu [E, H, 2I/8], qz_gu [E, H/32, 2I/8], sc_gu [E, H/32, 2I].
 * Down projection: K = I, N = H: qw_d [E, I, H/8], qz_d [E, I/32, H/8],
 *   sc_d [E, I/32, H].
 * x [T, H] dtype; f [rows, H], FP32 when out_fp32 != 0, else dtype.
 * Limits: H % 64 == 0, I % 64 == 0.  Workspace: MOE_OP_SWIGLU_AWQ_G32.
 * ------------------------------------------------------------------------- */
MOE_API int moe_grouped_swiglu_awq_g32(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T,
                               int rows, int H, int I, int E, const int32_t* qw_gu, const int32_t* qz_gu,
                               const void* sc_gu, const int32_t* qw_d, const int32_t* qz_d, const void* sc_d,
                               int dtype, int out_fp32, void* f, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Routed AWQ experts and the 16-bit shared expert of one layer in one call
 * [AWQ] [ARCH]: the routed part is moe_grouped_swiglu_awq_g32 (f [rows, H]),
 * the shared part the SwiGLU of every token with w_sh_gate_up [2I, H] and
 * w_sh_down [H, I] of `dtype` (shared_out [T, H] dtype: FP16, or BF16 in the
 * BF16 mode).  For T <= 16 (decode) both
 * run in one weight-streaming kernel: the routed weights stream as packed
 * codes, zero points and scales and are dequantised in shared memory, the
 * second GEMM is split along I into FP32 partials in the workspace that a
 * second kernel sums in a fixed order.  Larger T uses the grouped AWQ GEMMs
 * and then the dense shared expert.  Layouts, exact dequantisation and x as
 * in moe_grouped_swiglu_awq_g32; row_token is required.  Limits: H % 128 ==
 * 0, I % 64 == 0.  Workspace: MOE_OP_EXPERTS_AWQ_G32.
 * ------------------------------------------------------------------------- */
MOE_API int moe_experts_awq_g32(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T,
                                int rows, int H, int I, int E, const int32_t* qw_gu, const int32_t* qz_gu,
                                const void* sc_gu, const int32_t* qw_d, const int32_t* qz_d, const void* sc_d,
                                const void* w_sh_gate_up, const void* w_sh_down, int dtype, int out_fp32, void* f,
                                void* shared_out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Tile-packed copy of one layer's routed AWQ weights [AWQ], made once, for
 * moe_experts_awq_g32_prepacked (decode and prefill): the same codes, zero
 * points and scales (no value changes, same total size) regrouped so that
 * every 64-input-row sub-tile the decode kernel streams is one contiguous
 * 4736-byte unit.  Inputs as in moe_grouped_swiglu_awq_g32; out: device
 * buffer of moe_awq_packed_bytes(E, H, I) bytes, 16-byte aligned, owned by
 * the caller (its layout is internal to the library).
 * moe_awq_packed_bytes returns 0 for unsupported sizes.
 * Limits: H % 128 == 0, I % 64 == 0; out_bytes large enough
 * (MOE_ERR_WORKSPACE otherwise).
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_awq_packed_bytes(int E, int H, int I);
MOE_API int moe_awq_prepack_g32(const int32_t* qw_gu, const int32_t* qz_gu, const void* sc_gu, const int32_t* qw_d,
                                const int32_t* qz_d, const void* sc_d, int E, int H, int I, void* out,
                                size_t out_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_experts_awq_g32 with the routed weights also given tile-packed
 * (awq_packed, from moe_awq_prepack_g32 on the same qw/qz/sc): for T <= 16
 * the decode kernel reads only awq_packed (one bulk copy per sub-tile
 * instead of six tensor-map boxes); larger T reads awq_packed too in the
 * grouped GEMMs whose tiles are 128 or 256 columns wide (one bulk copy per
 * 128-column unit), qw/qz/sc otherwise, and its GEMM1 gathers the x rows
 * through row_token itself (no separate gather launch).
 * Results are identical to moe_experts_awq_g32's.  All other arguments,
 * limits and the workspace as there; awq_packed must not be NULL.
 * ------------------------------------------------------------------------- */
MOE_API int moe_experts_awq_g32_prepacked(const void* x, const int32_t* row_token, const int32_t* expert_offsets,
                                          int T, int rows, int H, int I, int E, const int32_t* qw_gu,
                                          const int32_t* qz_gu, const void* sc_gu, const int32_t* qw_d,
                                          const int32_t* qz_d, const void* sc_d, const void* awq_packed,
                                          const void* w_sh_gate_up, const void* w_sh_down, int dtype, int out_fp32,
                                          void* f, void* shared_out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * AWQ dequantisation [AWQ], the same device code the grouped GEMM runs on
 * each weight tile: out[b, k, n] = fp16_rn((q - z) * s) (dtype F16) or
 * bf16_rn((q - z) * bf16_rn(s)) (dtype BF16) for `batch` stacked projections
 * in the layout above (qweight [batch, K, N/8], qzeros [batch, K/32, N/8],
 * scales [batch, K/32, N] FP16); out [batch, K, N] of dtype, input-major
 * like the stored codes.  Limits: K % 32 == 0, N % 8 == 0.
 * ------------------------------------------------------------------------- */
MOE_API int moe_awq_dequant_g32(const int32_t* qweight, const int32_t* qzeros, const void* scales, int batch, int K,
                                int N, int dtype, void* out, void* stream);

/* ---------------------------------------------------------------------------
 * NVFP4 quantisation of `batch` tensors [rows, K] of 16-bit values [NVFP4]
 * (decode-direction scales, every rounding decision in FP32 IEEE
 * round-to-nearest-even, in this order):
 *     s_g = amax(|V|) / 2688            (or global_scale_in[b] when given)
 *     s_b = e4m3_rn_satfinite(amax(|block of 16 along K|) / (6 * s_g))
 *     c   = e2m1_rn_satfinite(v / (e4m3(s_b) * s_g)),  c = +0 if e4m3(s_b)*s_g == 0
 * v [batch, rows, K] dtype; codes [batch, rows, K/2] uint8 (element 2j in the
 * low nibble); sf [batch, rows, K/16] uint8 E4M3; global_scale_out [batch]
 * FP32 (device).  global_scale_in [batch] FP32 device or NULL (dynamic).
 * Limits: K % 16 == 0.  Workspace: MOE_OP_NVFP4_QUANTIZE.
 * ------------------------------------------------------------------------- */
MOE_API int moe_nvfp4_quantize(const void* v, int batch, int rows, int K, int dtype, const float* global_scale_in,
                       uint8_t* codes, uint8_t* sf, float* global_scale_out, void* ws, size_t ws_bytes,
                       void* stream);

/* ---------------------------------------------------------------------------
 * Grouped SwiGLU expert FFN with NVFP4 W4A4 weights [NVFP4].  The gathered
 * activations are quantised to NVFP4 on the fly (moe_nvfp4_quantize's rule
 * over the whole [rows, H] input), GEMM1 runs on FP4 x FP4 with E4M3 block
 * scales and FP32 accumulation, h = silu(g) * u is quantised again (over the
 * whole [rows, I] intermediate) and GEMM2 runs the same way.
 * Weights as produced by moe_nvfp4_quantize:
 *   w_gu [E, 2I, H/2], sf_gu [E, 2I, H/16], gs_gu [E, 2] (gate, up);
 *   w_d  [E, H, I/2],  sf_d  [E, H, I/16],  gs_d  [E].
 * act_gs_in [2] FP32 device (static global scales of x and h) or NULL
 * (dynamic amax); act_gs_out [2] receives the scales used (may be NULL).
 * x [T, H] BF16; f [rows, H], FP32 when out_fp32 != 0, else BF16.
 * Limits: H % 128 == 0, I % 128 == 0.  Workspace: MOE_OP_SWIGLU_NVFP4.
 * ------------------------------------------------------------------------- */
MOE_API int moe_grouped_swiglu_nvfp4(const void* x, const int32_t* row_token, const int32_t* expert_offsets, int T,
                             int rows, int H, int I, int E, const uint8_t* w_gu, const uint8_t* sf_gu,
                             const float* gs_gu, const uint8_t* w_d, const uint8_t* sf_d, const float* gs_d,
                             const float* act_gs_in, float* act_gs_out, int out_fp32, void* f, void* ws,
                             size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Weight block scales of one NVFP4 projection, rearranged once into the order
 * in which the FP4 GEMM's B tiles read them, so that moe_grouped_swiglu_nvfp4
 * need not rearrange static scales on every call [NVFP4] (the scale values
 * are unchanged: this is layout only).
 * sf [E, rows_per_expert, K/16] uint8 E4M3 (moe_nvfp4_quantize's layout);
 * swiglu = 1 for a gate/up projection whose rows are [gate I | up I]
 * (rows_per_expert = 2I, each tile pairs 64 gate with the matching 64 up
 * rows), 0 for a plain projection (128 consecutive rows per tile).
 * out: device buffer of moe_nvfp4_packed_sf_bytes(...) bytes, owned by the
 * caller; the layout is opaque and is only read by
 * moe_grouped_swiglu_nvfp4_prepacked.  moe_nvfp4_packed_sf_bytes returns 0
 * for unsupported sizes.
 * Limits: rows_per_expert % 128 == 0, K % 128 == 0, out_bytes large enough
 * (MOE_ERR_WORKSPACE otherwise).
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_nvfp4_packed_sf_bytes(int E, int rows_per_expert, int K, int swiglu);
MOE_API int moe_nvfp4_prepack_sf(const uint8_t* sf, int E, int rows_per_expert, int K, int swiglu, uint8_t* out,
                                 size_t out_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_grouped_swiglu_nvfp4 [NVFP4] with the weight scales given already
 * rearranged by moe_nvfp4_prepack_sf (sf_gu_packed from sf_gu with swiglu = 1,
 * rows_per_expert = 2I, K = H; sf_d_packed from sf_d with swiglu = 0,
 * rows_per_expert = H, K = I).  Results are identical to
 * moe_grouped_swiglu_nvfp4's; all other arguments, limits and the workspace
 * are the same.
 * ------------------------------------------------------------------------- */
MOE_API int moe_grouped_swiglu_nvfp4_prepacked(const void* x, const int32_t* row_token, const int32_t* expert_offsets,
                                               int T, int rows, int H, int I, int E, const uint8_t* w_gu,
                                               const uint8_t* sf_gu_packed, const float* gs_gu, const uint8_t* w_d,
                                               const uint8_t* sf_d_packed, const float* gs_d,
                                               const float* act_gs_in, float* act_gs_out, int out_fp32, void* f,
                                               void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Weighted combine [ARCH]:
 *   y[t] = sum_{j<k} topk_w[t, j] * f[slot_row[t, j]]  (+ gate[t] * shared[t])
 * summed in FP32 in slot order, rounded once to dtype.
 * f [rows, H] (FP32 when f_fp32 != 0, else dtype); slot_row [T, k_slots]
 * (k <= k_slots; extra slots are ignored); topk_w [T, k] FP32; shared_out
 * [T, H] dtype or NULL; shared_gate [T] FP32 or NULL (gate 1); y [T, H] dtype.
 * Limits: H % 8 == 0.
 * ------------------------------------------------------------------------- */
MOE_API int moe_combine(const void* f, int f_fp32, const int32_t* slot_row, int k_slots, const float* topk_w,
                const void* shared_out, const float* shared_gate, int T, int k, int H, int dtype, void* y,
                void* stream);

/* ---------------------------------------------------------------------------
 * Pre-MoE RMSNorm [ARCH] (normalisation entries: RMSNorm whose gain is
 * 1 + w, applied before the block, epsilon 1e-6):
 *   y[t, h] = x[t, h] / sqrt(mean_h x[t, :]^2 + eps) * (1 + w[h])
 * with FP32 sums, rounded once to dtype.  x, y [T, H] dtype (y may be x);
 * w [H] dtype; all 16-byte aligned.  The fact sheet's eps is 1e-6.
 * Limits: H % 8 == 0.
 * ------------------------------------------------------------------------- */
MOE_API int moe_rmsnorm(const void* x, int T, int H, const void* w, float eps, int dtype, void* y, void* stream);

/* ---------------------------------------------------------------------------
 * Shared-expert gate [AWQ] ("Checkpoint": a shared-expert gate tensor is
 * stored with the router and the shared expert; the card gives no formula,
 * so this is the plainest reading):
 *   gate[t] = 1 / (1 + exp(-sum_h x[t, h] * w_gate[h]))     (FP32 accumulate)
 * to be passed as moe_combine's shared_gate.  x [T, H] and w_gate [H] dtype,
 * both 16-byte aligned; gate [T] FP32.  Limits: H % 8 == 0.
 * ------------------------------------------------------------------------- */
MOE_API int moe_shared_gate(const void* x, int T, int H, const void* w_gate, int dtype, float* gate, void* stream);

/* ---------------------------------------------------------------------------
 * Refill-RMS accumulation, fused with the combine of a (k+1)-slot pass
 * [RAZOR].  For token t with selected set S (slots 0..k-1) and promoted
 * expert r (slot k), with p_j = exp(l_j - l_0) from topk_logit:
 *   Z = sum_S p,  U = sum_S p_j f_j,  y = U / Z
 *   for each e in S:  delta_e = (U - p_e f_e + p_r f_r) / (Z - p_e + p_r) - y
 *                     sum_sq[e] += ||delta_e||_2^2,  count[e] += 1
 * (the layer output change when e is removed and r promoted; the shared
 * expert cancels).  Statistics are additive across calls: sum_sq [E] FP64 and
 * count [E] int64 are read and updated in place and must be initialised by
 * the caller (zeros for a fresh pass).  The per-expert sums are formed in a
 * fixed order (deterministic for a given routing).
 * f [rows, H] (FP32 when f_fp32 != 0, else dtype), rows = T*(k+1) permuted
 * rows of the (k+1)-slot pass; slot_row, topk_idx, topk_logit [T, k+1];
 * expert_offsets [E+1] of that pass.  y_out [T, H] dtype or NULL receives
 * y (+ shared_out when given).  Limits: k + 1 <= 16, H % 8 == 0.
 * Workspace: MOE_OP_REFILL.
 * ------------------------------------------------------------------------- */
MOE_API int razor_refill_rms_accumulate(const void* f, int f_fp32, const int32_t* slot_row, const int32_t* topk_idx,
                                const float* topk_logit, const int32_t* expert_offsets, int T, int k, int H, int E,
                                double* sum_sq, int64_t* count, const void* shared_out, void* y_out, int dtype,
                                void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Refill-RMS selection [RAZOR]: score_e = sqrt(sum_sq[e] / count[e]) (0 when
 * count[e] == 0), rank by (score descending, expert index ascending), keep the
 * first `keep`.  kept_idx [keep] int32 receives the kept original indices in
 * ascending order ("output order" of the sliced checkpoint); ranking [E]
 * int32 (the full order) and score [E] FP64 may be NULL.
 * Limits: 1 <= E <= 1024, 0 <= keep <= E.
 * ------------------------------------------------------------------------- */
MOE_API int razor_select(const double* sum_sq, const int64_t* count, int E, int keep, int32_t* kept_idx, int32_t* ranking,
                 double* score, void* stream);

/* ---------------------------------------------------------------------------
 * Router-norm keep policy [RAZOR] ("Selection and calibration", MTP item: the
 * MTP layer's experts are kept by the L2 norm of their original router rows,
 * mtp_policy=router_norm).  Writes sum_sq[e] = sum_h w_router[e, h]^2 (the
 * 16-bit weights squared exactly in FP64 and summed in a fixed order) and,
 * when count is not NULL, count[e] = 1: statistics in the form Refill-RMS
 * produces, so razor_select with the same keep ranks the experts by
 * sqrt(sum_sq / count) = ||w_router[e, :]||_2, ties to the lower index.
 * Both outputs are overwritten, not accumulated.
 * w_router [E, H] dtype; sum_sq [E] FP64; count [E] int64 or NULL.
 * ------------------------------------------------------------------------- */
MOE_API int razor_router_norm(const void* w_router, int E, int H, int dtype, double* sum_sq, int64_t* count,
                              void* stream);

/* ---------------------------------------------------------------------------
 * Slice of the kept experts [RAZOR] (opening paragraphs: the surviving
 * kept experts' weights and router rows are cut from the original checkpoint
 * in the same order; the manifest lists the original indices in the order of
 * the pruned layer).
 *
 *   dst[j] = src[kept_idx[j]]     for j < keep, whole blocks of
 *                                 bytes_per_expert bytes
 *
 * src holds E per-expert blocks back to back ([E, ...] with the expert index
 * leading: router rows, a router bias, every expert weight, scale and zero
 * tensor of any format, the tile-ordered copies of moe_awq_prepack_g32 and
 * moe_nvfp4_prepack_sf); dst receives keep blocks.  Passing the same
 * kept_idx (razor_select's ascending kept set) to every tensor of a layer
 * slices them in matching order.  The copy is byte-exact; 16-byte vectors
 * are used when both pointers and bytes_per_expert are multiples of 16.
 * kept_idx [keep] int32 device array, any order; an index outside [0, E) is
 * skipped (its dst block is left untouched) and recorded as
 * MOE_ERR_INVALID_ARG in the device status word.  dst must not overlap src.
 * Limits: 0 <= keep <= min(E, 65535).
 * ------------------------------------------------------------------------- */
MOE_API int razor_slice(const void* src, int E, size_t bytes_per_expert, const int32_t* kept_idx, int keep, void* dst,
                        void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BIT_EXPERT_GEMM_B200_MOE_H_ */
