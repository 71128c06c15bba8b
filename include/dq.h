/*
 * dq.h — C ABI of the B200 (sm_100a) per-token dynamic quantization library.
 *
 * Five operations, launched asynchronously on the caller's stream:
 *
 *   dq_dynamic_quant        aclnnDynamicQuantV2, "Formula" and "Description":
 *                           per-row (per-token) symmetric or asymmetric
 *                           quantization of x, optionally multiplied by a
 *                           per-channel smooth-scale vector that, for MoE,
 *                           is chosen per expert through a group index.
 *   dq_ada_layernorm_quant  aclnnAdaLayerNormQuant, "Formula" steps 1-5:
 *                           LayerNorm with optional weight/bias, then
 *                           y * (1 + scale) + shift, optional smooth scales,
 *                           then symmetric INT8 dynamic quantization.
 *   dq_dequant_per_token    AntiQuantize, PER_TOKEN policy: codes back to
 *                           floats with one scale (and offset) per row.
 *   dq_dequant_per_group    AntiQuantize, PER_GROUP policy: one scale (and
 *                           offset) per group of elements along a row or
 *                           down a column.
 *   dq_w8a8_gemm            aclnnQuantBatchMatmulInplaceAdd: the consumer of
 *                           the codes, a W8A8 product with per-token x
 *                           per-channel scales on the tensor cores.
 *
 * plus the workspace queries of the two-phase calling convention both pages
 * describe ("...GetWorkspaceSize" first, then the run): dq_get_workspace_size
 * and dq_ada_layernorm_quant_get_workspace_size.
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer (cudaMalloc'd or equivalent),
 *     owned by the caller. The library allocates nothing, keeps no state
 *     between calls and never synchronizes the stream.
 *   - Tensors are dense and row-major; the last dimension is the row
 *     ("token") that one scale covers. Leading dimensions are flattened.
 *   - Outputs must not overlap inputs or each other.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream). The
 *     returned status covers argument validation, done on the host before
 *     anything is launched (no launch happens when it is not DQ_OK), and
 *     the launch itself (DQ_ERR_CUDA). Faults that happen later surface
 *     through the CUDA stream like any other kernel's.
 *   - Results are deterministic: the same inputs give the same bytes on
 *     every call (both pages state deterministic implementations).
 *   - Quantization rows are streamed through shared memory with bulk (TMA)
 *     copies; every wait in the kernels is bounded. If a copy never completes (a device
 *     fault, never a data-dependent condition) the affected rows get NaN
 *     scales instead of the kernel hanging.
 *
 * Arithmetic (fixed by the formulas; identical to the CPU oracle):
 *   IEEE binary32 throughout; x and smooth scales are widened exactly;
 *   input = x * smooth is one rounded multiply; scale = absmax / 127 (or
 *   (max - min) / scale_opt) and x / scale are IEEE divisions; "round" is
 *   round-half-to-even; codes saturate to the output range.
 */
#ifndef DQ_H
#define DQ_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. DQ_OK is 0; everything else is an error and means nothing was
 * launched (except DQ_ERR_CUDA, which reports a failed launch). */
typedef enum dq_status {
  DQ_OK = 0,
  DQ_ERR_NULL_POINTER = 1,        /* a required pointer is NULL */
  DQ_ERR_BAD_SHAPE = 2,           /* negative/zero sizes, odd cols for INT4, ... */
  DQ_ERR_BAD_DTYPE = 3,           /* dtype not allowed in that argument */
  DQ_ERR_UNSUPPORTED = 4,         /* valid request this library does not implement */
  DQ_ERR_MISALIGNED = 5,          /* pointer below its element's natural alignment */
  DQ_ERR_WORKSPACE_TOO_SMALL = 6, /* workspace missing or smaller than queried */
  DQ_ERR_CUDA = 7,                /* the CUDA launch failed (cudaGetLastError) */
  DQ_ERR_BAD_ARGUMENT = 8         /* any other invalid argument value */
} dq_status;

/* Element types. DQ_INT4X2: two signed 4-bit codes per byte, element 2j in
 * bits 0-3 and element 2j+1 in bits 4-7 of byte j. DQ_INT32: eight signed
 * 4-bit codes per 32-bit word, element 8j+k in bits 4k..4k+3 of word j
 * (aclnnDynamicQuantV2, "Constraints": INT32 output packs int4 codes and
 * needs a last dimension divisible by 8). On a little-endian host the two
 * packed layouts are the same bytes. */
typedef enum dq_dtype {
  DQ_F32 = 0,
  DQ_F16 = 1,
  DQ_BF16 = 2,
  DQ_INT8 = 3,
  DQ_INT4X2 = 4,
  DQ_INT32 = 5
} dq_dtype;

/* aclnnDynamicQuantV2, "Formula": symmetric or asymmetric quantization. */
typedef enum dq_mode { DQ_SYMMETRIC = 0, DQ_ASYMMETRIC = 1 } dq_mode;

/* Bits of the 32-bit status word at the start of the workspace (MoE calls). */
#define DQ_WS_ROWS_PAST_LAST_GROUP 0x1u /* rows >= group_index[E-1]: zero codes, scale 0 */
#define DQ_WS_GROUP_INDEX_INVALID 0x2u  /* group_index decreasing or negative */

/* Largest expert count a group index may have. */
#define DQ_MAX_GROUPS 1024

/* Human-readable name of a status code (static string, never NULL). */
const char* dq_status_string(dq_status status);

/* Workspace query — the first phase of the two-phase convention
 * (aclnnDynamicQuantV2 and aclnnAdaLayerNormQuant, "...GetWorkspaceSize").
 *
 * Validates the sizes and dtypes of a dq_dynamic_quant call and writes the
 * number of bytes of device workspace it needs to *workspace_bytes: 0 without
 * a group index, 4 with one (a status word the kernel writes on every call,
 * see DQ_WS_*). Pointers are not inspected. Host only; no CUDA call.
 *   rows >= 0, cols >= 1; x_dtype in {DQ_F16, DQ_BF16};
 *   y_dtype in {DQ_INT8, DQ_INT4X2 (cols even), DQ_INT32 (cols % 8 == 0)};
 *   0 <= num_groups <= DQ_MAX_GROUPS.
 * Returns DQ_ERR_NULL_POINTER if workspace_bytes is NULL. */
dq_status dq_get_workspace_size(int64_t rows, int64_t cols, dq_dtype x_dtype,
                                dq_mode mode, dq_dtype y_dtype, int32_t num_groups,
                                size_t* workspace_bytes);

/* Per-token dynamic quantization (aclnnDynamicQuantV2, "Formula").
 *
 * For every row r of x [rows, cols]:
 *   input[c] = x[r,c] * smooth[e(r), c]     (when smooth != NULL; else x[r,c])
 *   symmetric:  scale[r] = max_c |input| / 127    (7 for 4-bit outputs)
 *               y[r,c]   = round(input[c] / scale[r])          in [-127, 127]
 *   asymmetric: scale[r] = (max_c input - min_c input) / scale_opt
 *               offset[r] = offset_opt - max_c input / scale[r]
 *               y[r,c]   = round(input[c] / scale[r] + offset[r])
 *   (scale_opt, offset_opt) = (255, 127) for DQ_INT8, (15, 7) for DQ_INT4X2 and
 *   DQ_INT32; asymmetric codes lie in [-128, 127] or [-8, 7].
 *   A symmetric row with absmax 0 gets scale 0 and codes 0; an asymmetric row
 *   with max == min gets scale 0, offset offset_opt and codes offset_opt.
 *
 * Arguments
 *   x            device, [rows, cols] of x_dtype (DQ_F16 or DQ_BF16).
 *   smooth       device or NULL. [cols] without a group index, [num_groups,
 *                cols] with one; smooth_dtype in {DQ_F32, DQ_F16, DQ_BF16}.
 *                Ignored (smooth_dtype too) when NULL.
 *   group_index  device int32 [num_groups] or NULL (aclnnDynamicQuantV2,
 *                "Description": MoE expert selection). Entry e is the
 *                cumulative END row (exclusive) of expert e, so the list is
 *                non-decreasing and e(r) is the smallest e with
 *                r < group_index[e]; empty experts are equal neighbours.
 *                Requires smooth. Rows at or past group_index[E-1] get codes 0,
 *                scale 0 (and offset 0) and set DQ_WS_ROWS_PAST_LAST_GROUP in
 *                the workspace status word. num_groups is 0 iff it is NULL.
 *   mode         DQ_SYMMETRIC or DQ_ASYMMETRIC.
 *   y_dtype      DQ_INT8 (y is int8 [rows, cols]), DQ_INT4X2 (uint8
 *                [rows, cols/2]) or DQ_INT32 (int32 [rows, cols/8]).
 *   y, scale     device outputs; scale is float [rows].
 *   offset       device float [rows], required for DQ_ASYMMETRIC; ignored (may
 *                be NULL) for DQ_SYMMETRIC.
 *   workspace    device, at least the bytes dq_get_workspace_size returned,
 *                4-byte aligned; may be NULL when that is 0. With a group
 *                index its first word is overwritten on every call with the
 *                DQ_WS_* bits of this call (no clearing needed).
 *   stream       CUDA stream to launch on.
 * Alignment: x, smooth 2-byte (4 for fp32); scale, offset, group_index,
 * workspace 4-byte; y 4-byte for DQ_INT32. Rows whose data are 16-byte
 * aligned take a vectorised path; others a scalar one — same results.
 * rows == 0 is a valid no-op (pointers are then not checked).
 * Errors: DQ_ERR_NULL_POINTER, DQ_ERR_BAD_SHAPE, DQ_ERR_BAD_DTYPE,
 * DQ_ERR_BAD_ARGUMENT, DQ_ERR_MISALIGNED, DQ_ERR_WORKSPACE_TOO_SMALL,
 * DQ_ERR_UNSUPPORTED (num_groups > DQ_MAX_GROUPS), DQ_ERR_CUDA. */
dq_status dq_dynamic_quant(const void* x, dq_dtype x_dtype, int64_t rows, int64_t cols,
                           const void* smooth, dq_dtype smooth_dtype,
                           const int32_t* group_index, int32_t num_groups,
                           dq_mode mode, dq_dtype y_dtype,
                           void* y, float* scale, float* offset,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Workspace query for dq_ada_layernorm_quant (the first phase of
 * aclnnAdaLayerNormQuant's two-phase convention). Writes the bytes of device
 * workspace the call needs: batch * hidden * 8 (room for a folded table of
 * the affine parameters, rebuilt by any call that keeps the table in global
 * memory), or 0 when batch * seq == 0. Host only.
 * Errors: DQ_ERR_NULL_POINTER, DQ_ERR_BAD_SHAPE, DQ_ERR_BAD_DTYPE. */
dq_status dq_ada_layernorm_quant_get_workspace_size(int64_t batch, int64_t seq, int64_t hidden,
                                                    dq_dtype x_dtype, dq_dtype param_dtype,
                                                    size_t* workspace_bytes);

/* Fused AdaLayerNorm + symmetric INT8 quantization (aclnnAdaLayerNormQuant,
 * "Formula"; the page fuses only DynamicQuant, i.e. symmetric INT8).
 *
 * For every row (b, s) of x [batch, seq, hidden]:
 *   1. LN = (x - E(x)) / sqrt(Var(x) + epsilon) * weight + bias
 *      (E, Var over the row; Var is biased, dividing by hidden)
 *   2. y  = LN * (1 + ada_scale[b]) + ada_shift[b]
 *   3. y  = y * smooth                                   (when smooth != NULL)
 *   4. quant_scale[b,s] = max |y| / 127
 *   5. out[b,s,:] = round(y / quant_scale[b,s])          in [-127, 127]
 * Arguments
 *   x                  device [batch, seq, hidden], x_dtype DQ_F16 or DQ_BF16.
 *   ada_scale, ada_shift  device [batch, hidden] of param_dtype (required).
 *   weight, bias, smooth  device [hidden] of param_dtype, or NULL (weight 1,
 *                      bias 0, no smoothing).
 *   param_dtype        DQ_F32, DQ_F16 or DQ_BF16 (all parameters share it).
 *   epsilon            finite, >= 0.
 *   out                device int8 [batch, seq, hidden]; quant_scale device
 *                      float [batch, seq].
 *   workspace          device, 16-byte aligned, at least the bytes
 *                      dq_ada_layernorm_quant_get_workspace_size returned.
 *                      Its contents are scratch, which a call may overwrite;
 *                      calls that run concurrently need separate workspaces.
 * Steps 1-3's parameters are folded into y = n * A + B (A, B per batch and
 * column). When the table rows of the batches one CTA processes fit in 64 KB
 * of shared memory, one kernel is launched on `stream` and folds them there;
 * otherwise a first kernel writes the table into the workspace and the row
 * kernel, launched second, overlaps its start with it.
 * The row statistics are reduced in a different order than a sequential loop
 * and steps 1-3 are folded, so a result may differ from a sequential fp32
 * evaluation in the last bits: quant_scale by a relative 1e-5 at most, and
 * rarely a code by 1.
 * Errors: as dq_dynamic_quant (DQ_ERR_BAD_ARGUMENT for a bad epsilon). */
dq_status dq_ada_layernorm_quant(const void* x, dq_dtype x_dtype,
                                 int64_t batch, int64_t seq, int64_t hidden,
                                 const void* ada_scale, const void* ada_shift,
                                 const void* weight, const void* bias, const void* smooth,
                                 dq_dtype param_dtype, float epsilon,
                                 int8_t* out, float* quant_scale,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Per-token dequantization (AntiQuantize, PER_TOKEN policy: every row of an
 * [m, n] code matrix shares one scale and one offset, shapes [m, 1]).
 *
 * The page's formula images were lost; the operation is read as the inverse
 * of dq_dynamic_quant (whose codes are round(input / scale + offset)):
 *   out[r,c] = (code[r,c] - offset[r]) * scale[r]
 * evaluated in IEEE binary32 with one rounding per operation (the subtraction
 * only when offset is given), then rounded to nearest even into out_dtype.
 * Arguments
 *   y            device codes: DQ_INT8 int8 [rows, cols]; DQ_INT4X2 uint8
 *                [rows, cols/2] (element 2j in the low nibble of byte j);
 *                DQ_INT32 int32 [rows, cols/8] (the same bytes).
 *   scale        device [rows] of scale_dtype (DQ_F32, DQ_F16 or DQ_BF16).
 *   offset       device [rows] of scale_dtype, or NULL for no offset.
 *   out          device [rows, cols] of out_dtype (DQ_F32, DQ_F16, DQ_BF16).
 * The page lists int8 codes with half scales to half output, bfloat16 to
 * bfloat16, and float scales to float, half or bfloat16 output; every
 * combination of the three float types is accepted here.
 * Alignment: scale/offset to their element size, out to its element size,
 * y 4-byte for DQ_INT32. Rows whose codes and outputs are 16-byte aligned
 * and a whole number of 16-byte code vectors take a vectorised path; others
 * a scalar one, with the same results. rows == 0 is a no-op.
 * Errors: DQ_ERR_NULL_POINTER, DQ_ERR_BAD_SHAPE (cols < 1, odd cols for
 * DQ_INT4X2, cols % 8 for DQ_INT32), DQ_ERR_BAD_DTYPE, DQ_ERR_MISALIGNED,
 * DQ_ERR_CUDA. */
dq_status dq_dequant_per_token(const void* y, dq_dtype y_dtype, int64_t rows, int64_t cols,
                               const void* scale, const void* offset, dq_dtype scale_dtype,
                               void* out, dq_dtype out_dtype, cudaStream_t stream);

/* Per-group dequantization (AntiQuantize, PER_GROUP policy): along the k
 * axis every group_size elements share one scale and one offset.
 *   k_dim = 1 (k runs along a row): scale/offset tables [rows, ceil(cols/g)];
 *             element (i, j) uses entry (i, j / g).
 *   k_dim = 0 (k runs down a column): tables [ceil(rows/g), cols]; element
 *             (i, j) uses entry (i / g, j).
 * group_size > 0 and a multiple of 32 (the page's constraint). The value is
 * computed as in dq_dequant_per_token with the element's scale and offset;
 * the page's formula images were lost, so that is a reading (the inverse of
 * the quantizer). The page's int8 ("b8") source scenario is covered, with
 * the int4 / INT32 containers accepted as well; its fp4 / fp8 / hifloat8
 * scenarios are not (their formats are not defined on the pages).
 * Arguments, alignment and errors as dq_dequant_per_token, plus
 * DQ_ERR_BAD_ARGUMENT for a bad group_size or k_dim. With k_dim = 0, tables
 * that are 16-byte aligned take the vectorised path. */
dq_status dq_dequant_per_group(const void* y, dq_dtype y_dtype, int64_t rows, int64_t cols,
                               const void* scale, const void* offset, dq_dtype scale_dtype,
                               int64_t group_size, int32_t k_dim,
                               void* out, dq_dtype out_dtype, cudaStream_t stream);

/* W8A8 product with per-token x per-channel scales, on the tensor cores
 * (aclnnQuantBatchMatmulInplaceAdd, "计算公式", T-T form: the quantized
 * product times (scale1 * scale2), plus y), with scale1 per row of a (per
 * token, as dq_dynamic_quant produces it) and scale2 per output column:
 *   acc[m,n] = sum_k a[m,k] * b[n,k]                     (exact int32)
 *   out[m,n] = float(acc) * (a_scale[m] * b_scale[n])  (+ out[m,n] when
 *              accumulate), each binary32 operation rounded once in that
 *              order, then narrowed to out_dtype (round to nearest even).
 * Arguments
 *   a        device int8 [m, k] (the quantized activations, rows contiguous).
 *   b        device int8 [n, k] (each output column's weights contiguous).
 *   a_scale  device float [m]; b_scale device float [n].
 *   out      device [m, n] of out_dtype (DQ_F32, DQ_F16, DQ_BF16);
 *            accumulate = 1 adds into it (DQ_F32 only), 0 overwrites.
 * k < 2^17 (|sum| <= k * 128 * 128 < 2^31: int32 sums cannot overflow, even
 * with every code at -128). With k a multiple of 16 and
 * 16-byte aligned a and b, any m and n run on tcgen05 tensor cores
 * (128 x 256 or 128 x 128 tiles, ragged edges zero-filled and masked); other
 * shapes run a CUDA-core kernel with the same results.
 * Errors: DQ_ERR_BAD_SHAPE, DQ_ERR_BAD_DTYPE, DQ_ERR_BAD_ARGUMENT,
 * DQ_ERR_NULL_POINTER, DQ_ERR_MISALIGNED, DQ_ERR_CUDA. */
dq_status dq_w8a8_gemm(const int8_t* a, const int8_t* b, int64_t m, int64_t n, int64_t k,
                       const float* a_scale, const float* b_scale, void* out, dq_dtype out_dtype,
                       int32_t accumulate, cudaStream_t stream);

/* Largest batch * hidden that dq_ada_layernorm_quant_noalloc accepts (its
 * fixed table holds this many 8-byte entries: 1 MiB per device). */
#define DQ_ADA_NOALLOC_MAX_TABLE 131072

/* dq_ada_layernorm_quant without a workspace argument: the same computation
 * and results, with the scratch table kept in a fixed device array inside the
 * library. The pages have no counterpart to this entry point (their two-phase
 * calls always take a workspace); it exists for callers that cannot allocate
 * device memory: a plain C host program that links only this library, or code
 * that runs where allocating would re-enter the caller's own allocator (for
 * example an out-of-memory handler).
 *   - Allocates nothing: no cudaMalloc/cudaFree, no library allocation.
 *   - Checks in dq_ada_layernorm_quant's order (shapes and dtypes, epsilon,
 *     batch * seq == 0 returns DQ_OK, required pointers), then
 *     batch * hidden <= DQ_ADA_NOALLOC_MAX_TABLE, else DQ_ERR_UNSUPPORTED
 *     (where dq_ada_layernorm_quant checks its workspace); nothing is
 *     launched on an error.
 *   - The first call on each device (with that device current) looks up the
 *     array's address with cudaGetSymbolAddress and caches it with the
 *     identity of the device's context; the first call after a device reset
 *     (cudaDeviceReset) looks it up again. Make such a call before any stream
 *     capture. A failed lookup returns DQ_ERR_CUDA.
 *   - Nothing needs clearing beforehand: each call writes every table entry it
 *     reads.
 *   - The array is shared by all calls on a device: calls whose executions
 *     overlap (other streams, other host threads) race on it and must use
 *     dq_ada_layernorm_quant with separate workspaces instead. */
dq_status dq_ada_layernorm_quant_noalloc(const void* x, dq_dtype x_dtype,
                                         int64_t batch, int64_t seq, int64_t hidden,
                                         const void* ada_scale, const void* ada_shift,
                                         const void* weight, const void* bias, const void* smooth,
                                         dq_dtype param_dtype, float epsilon,
                                         int8_t* out, float* quant_scale, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DQ_H */
