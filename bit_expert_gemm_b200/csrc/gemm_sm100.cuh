// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05 /
// TMEM), fed by TMA.  Used for the expert GEMMs of the MoE layer (gate/up
// with a fused SwiGLU epilogue, and down), for dense experts (one group) and
// for the router logits (one group, FP32 output plus bias).
//
//   for every group g (an expert) with rows R_g = [off[g], off[g+1]) of A:
//     D[r, n] = sum_k A[r, k] * B[g * b_rows + n, k]          (FP32 in TMEM)
//
// Tiles are 128 rows of A by BN rows of B, K stepped by 64 (one 128-byte
// swizzle row of 16-bit elements).  Warp roles: warp 0 = TMA producer,
// warp 1 = UMMA issuer (and TMEM owner), warps 2..5 = epilogue, one TMEM
// lane quadrant each.  The accumulator is double-buffered in TMEM so the
// epilogue of one tile overlaps the main loop of the next.
#pragma once

#include "common.cuh"

namespace moe {

enum { EPI_SWIGLU = 0, EPI_STORE = 1 };
constexpr int kGemmMaxGroups = 1024;

struct GemmArgs {
  const int* group_offsets;  // [G+1] on the device, or nullptr: one group of `rows` rows
  int G;
  int rows;
  int K;                 // multiple of 64
  int n_out;             // output columns per group (SwiGLU: I; store: N)
  int b_rows_per_group;  // rows of B per group (SwiGLU: 2I; store: N)
  int up_offset;         // SwiGLU: row offset of the up rows (I)
  void* out;
  int ldo;               // output leading dimension (elements)
  int out_fp32;          // store: 1 -> FP32 output, 0 -> 16-bit of the input dtype
  const float* bias;     // store: per output column, may be nullptr
  int bf16;              // 1: BF16 operands, 0: FP16
  int* status;
  unsigned long long limit_ns;
  // Row gather of A (optional): A row r of the grouped problem is row
  // row_token[r] of a_src [a_src_rows, K]; nullptr: A is read as stored.
  const int* row_token;
  const void* a_src;
  int a_src_rows;
  // AWQ only (optional): the tile-packed copy of the weights (awq.cu
  // awq_prepack, codes and zero points in pair order); the kernel then reads
  // it, one bulk copy per 128-column unit, instead of the checkpoint arrays.
  const uint8_t* awq_packed;
};

// Host launcher (gemm_sm100.cu).  A [a_rows, K] and B [b_rows_total, K] are
// row-major 16-bit device arrays.  bn selects the tile width (64/128/256).
int launch_grouped_gemm(const void* A, int a_rows, const void* B, int b_rows_total, const GemmArgs& args, int epi,
                        int bn, cudaStream_t stream);

// Same GEMM with AWQ W4A16 group-32 weights as B.  Per group the stored
// projection has K input rows and n_total output columns: qweight [G*K,
// n_total/8] int32, qzeros [G*K/32, n_total/8] int32, scales [G*K/32,
// n_total] FP16.  Dequantisation warps turn each staged tile of codes into
// 16-bit weights in shared memory that the tensor cores read MN-major:
// exactly fp16_rn((q-z)*s) with FP16 operands (args.bf16 = 0), or
// bf16_rn((q-z)*bf16_rn(s)) in the BF16 mode (args.bf16 = 1).  args.up_offset is the column of the up
// half (SwiGLU); args.b_rows_per_group is unused.
// awq_packed (may be NULL): the tile-packed copy of the same weights, read
// instead of them for tile widths 128 and 256.
int launch_grouped_gemm_awq(const void* A, int a_rows, const int32_t* qweight, const int32_t* qzeros,
                            const void* scales, int n_total, const GemmArgs& args, int epi, int bn,
                            cudaStream_t stream, const void* awq_packed = nullptr);

}  // namespace moe
