/* Declarations of the CPU oracle (test infrastructure only; see dq_oracle.cpp).
 * This header belongs to the oracle alone: the CUDA library neither includes
 * it nor shares any of its constants. */
#ifndef DQ_ORACLE_H
#define DQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element storage types of floating-point inputs */
enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };
/* output code containers */
enum { ORACLE_Y_INT8 = 0, ORACLE_Y_INT4X2 = 1, ORACLE_Y_INT32 = 2 };
/* quantization mode */
enum { ORACLE_SYMMETRIC = 0, ORACLE_ASYMMETRIC = 1 };
/* status */
enum {
  ORACLE_OK = 0,
  ORACLE_ERR_SHAPE = -1,
  ORACLE_ERR_DTYPE = -2,
  ORACLE_ERR_ARGUMENT = -3,
  ORACLE_ERR_GROUP_INDEX = -4
};

/* Per-token dynamic quantization (aclnnDynamicQuantV2, Formula).
 * x: [rows, cols] row-major; smooth: NULL, [cols] or [num_groups, cols];
 * group_index: NULL or [num_groups] cumulative end rows; y: int8 [rows, cols],
 * packed uint8 [rows, cols/2] or uint32 [rows, cols/8]; scale: [rows];
 * offset: [rows] (asymmetric only, else may be NULL). */
int oracle_dynamic_quant(const void* x, int x_dtype, int64_t rows, int64_t cols,
                         const void* smooth, int smooth_dtype,
                         const int32_t* group_index, int32_t num_groups,
                         int mode, int y_dtype,
                         void* y, float* scale, float* offset);

/* AdaLayerNorm prologue (aclnnAdaLayerNormQuant, Formula steps 1-3): writes the
 * fp32 value that is quantized, plus per-row mean and sqrt(var+eps). */
int oracle_ada_layernorm_pre(const void* x, int x_dtype, int64_t batch, int64_t seq, int64_t hidden,
                             const void* ada_scale, const void* ada_shift,
                             const void* weight, const void* bias, const void* smooth,
                             int param_dtype, float epsilon,
                             float* y, float* mean_out, float* std_out);

/* Fused AdaLayerNormQuant (aclnnAdaLayerNormQuant, Formula steps 1-5). */
int oracle_ada_layernorm_quant(const void* x, int x_dtype, int64_t batch, int64_t seq, int64_t hidden,
                               const void* ada_scale, const void* ada_shift,
                               const void* weight, const void* bias, const void* smooth,
                               int param_dtype, float epsilon,
                               int8_t* out, float* quant_scale);

/* Per-token dequantization (AntiQuantize, PER_TOKEN policy: one scale and
 * offset per row of an [m, n] source). The pages print no formula for it; the
 * reading is the inverse of aclnnDynamicQuantV2's quantizer:
 *   out[r,c] = (code[r,c] - offset[r]) * scale[r]   (binary32, each operation
 *   rounded; the subtraction only when offset is given), then rounded to
 *   out_dtype (round to nearest even).
 * y: codes in a container of y_dtype (ORACLE_Y_*), [rows, cols] codes;
 * scale, offset (NULL allowed): [rows] of scale_dtype; out: [rows, cols] of
 * out_dtype (float, or the uint16 bit patterns of binary16 / bfloat16). */
int oracle_dequant_per_token(const void* y, int y_dtype, int64_t rows, int64_t cols,
                             const void* scale, const void* offset, int scale_dtype,
                             int out_dtype, void* out);

/* Per-group dequantization (AntiQuantize, PER_GROUP policy, int8 source):
 * every group_size elements along the k axis share one scale and offset.
 * k_dim = 1 (k runs along a row): scale/offset [rows, ceil(cols/group_size)],
 * element (i, j) uses entry (i, j / group_size); k_dim = 0 (k runs down a
 * column): scale/offset [ceil(rows/group_size), cols], element (i, j) uses
 * entry (i / group_size, j). group_size > 0 and a multiple of 32. The value is
 * computed as in oracle_dequant_per_token with that element's scale/offset. */
int oracle_dequant_per_group(const void* y, int y_dtype, int64_t rows, int64_t cols,
                             const void* scale, const void* offset, int scale_dtype,
                             int64_t group_size, int k_dim, int out_dtype, void* out);

/* W8A8 GEMM with per-token x per-channel scales (the quantized matrix
 * product that consumes the codes; aclnnQuantBatchMatmulInplaceAdd,
 * "计算公式", T-T form, with scale1 per row of x1 and scale2 per column of
 * the product):
 *   acc[m,n] = sum_k a[m,k] * b[n,k]            (exact integer)
 *   t        = float(acc[m,n]) * (a_scale[m] * b_scale[n])   (binary32: the
 *              int32 -> float conversion, the scale product and the multiply
 *              are each rounded once, in the formula's order)
 *   out[m,n] = accumulate ? t + out[m,n] : t     (then narrowed to out_dtype)
 * a: int8 [M, K]; b: int8 [N, K] (each output column's weights contiguous);
 * a_scale [M], b_scale [N] float; out [M, N] of out_dtype (accumulate only
 * with ORACLE_F32). */
int oracle_w8a8_gemm(const int8_t* a, const int8_t* b, int64_t m, int64_t n, int64_t k,
                     const float* a_scale, const float* b_scale, int out_dtype, int accumulate, void* out);

/* binary32 -> binary16 / bfloat16 bit patterns, round to nearest even (the
 * narrowing the dequantizer ends with; exported for its pins). */
uint16_t oracle_float_to_half_bits(float f);
uint16_t oracle_float_to_bfloat16_bits(float f);

#ifdef __cplusplus
}
#endif

#endif /* DQ_ORACLE_H */
