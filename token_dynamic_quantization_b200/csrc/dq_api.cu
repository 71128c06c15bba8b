// C ABI of the per-token dynamic quantization library (declared in include/dq.h).
//
// Host side of the two-phase convention of aclnnDynamicQuantV2 and
// aclnnAdaLayerNormQuant: every call validates its arguments on the host
// before anything is launched (the pages' "first-phase API implements input
// parameter verification"), then launches its kernels on the caller's
// stream through the dispatchers of dq_launch.cuh (one translation unit per
// kernel family). The library allocates nothing and keeps no per-call
// state; the only cached values are per-device launch facts (SM count,
// occupancy).

#include <cmath>
#include <cstdint>

#include "dq.h"
#include "dq_args.cuh"
#include "dq_launch.cuh"

namespace {

using dq_host::aligned;

size_t float_size(dq_dtype t) { return t == DQ_F32 ? 4 : 2; }

bool is_input_float(dq_dtype t) { return t == DQ_F16 || t == DQ_BF16; }
bool is_param_float(dq_dtype t) { return t == DQ_F32 || t == DQ_F16 || t == DQ_BF16; }
bool is_code_type(dq_dtype t) { return t == DQ_INT8 || t == DQ_INT4X2 || t == DQ_INT32; }

size_t ada_table_bytes(int64_t batch, int64_t hidden) { return static_cast<size_t>(batch * hidden) * 8; }

// Shared validation and dispatch of the two dequantization entry points.
dq_status dequantize(int layout, const void* y, dq_dtype y_dtype, int64_t rows, int64_t cols, const void* scale,
                     const void* offset, dq_dtype scale_dtype, int64_t group_size, int64_t table_cols, void* out,
                     dq_dtype out_dtype, bool table_vec_ok, cudaStream_t stream) {
  if (rows < 0 || cols < 1 || cols > (int64_t(1) << 31) || rows > (int64_t(1) << 40)) return DQ_ERR_BAD_SHAPE;
  if (!is_code_type(y_dtype) || !is_param_float(scale_dtype) || !is_param_float(out_dtype)) return DQ_ERR_BAD_DTYPE;
  if (y_dtype == DQ_INT4X2 && cols % 2 != 0) return DQ_ERR_BAD_SHAPE;
  if (y_dtype == DQ_INT32 && cols % 8 != 0) return DQ_ERR_BAD_SHAPE;
  if (rows == 0) return DQ_OK;
  if (y == nullptr || scale == nullptr || out == nullptr) return DQ_ERR_NULL_POINTER;
  const size_t ss = float_size(scale_dtype), os = float_size(out_dtype);
  if (!aligned(scale, ss) || (offset && !aligned(offset, ss)) || !aligned(out, os) ||
      (y_dtype == DQ_INT32 && !aligned(y, 4)))
    return DQ_ERR_MISALIGNED;
  dq::DequantArgs a{};
  a.y = y;
  a.rows = rows;
  a.cols = cols;
  a.scale = scale;
  a.offset = offset;
  a.scale_dtype = static_cast<int>(scale_dtype);
  a.out = out;
  a.group_size = group_size;
  a.table_cols = table_cols;
  const bool four = y_dtype != DQ_INT8;
  const int out_kind = out_dtype == DQ_F32 ? dq::kOutF32 : (out_dtype == DQ_F16 ? dq::kOutF16 : dq::kOutBF16);
  const int64_t per_vec = four ? 32 : 16;
  const bool vec = cols % per_vec == 0 && aligned(y, 16) && aligned(out, 16) && table_vec_ok;
  return dq_host::dequant(a, layout, out_kind, four, offset != nullptr, vec, stream);
}

dq_status check_ada(int64_t batch, int64_t seq, int64_t hidden, dq_dtype x_dtype, dq_dtype param_dtype) {
  if (batch < 0 || seq < 0 || hidden < 1) return DQ_ERR_BAD_SHAPE;
  if (hidden > (int64_t(1) << 31) || batch > (int64_t(1) << 40) || seq > (int64_t(1) << 40)) return DQ_ERR_BAD_SHAPE;
  if (batch > 0 && seq > (int64_t(1) << 40) / batch) return DQ_ERR_BAD_SHAPE;
  if (!is_input_float(x_dtype) || !is_param_float(param_dtype)) return DQ_ERR_BAD_DTYPE;
  return DQ_OK;
}

dq_status check_sizes(int64_t rows, int64_t cols, dq_dtype x_dtype, dq_mode mode, dq_dtype y_dtype,
                      int32_t num_groups) {
  if (rows < 0 || cols < 1) return DQ_ERR_BAD_SHAPE;
  if (rows > (int64_t(1) << 40) || cols > (int64_t(1) << 31)) return DQ_ERR_BAD_SHAPE;
  if (!is_input_float(x_dtype)) return DQ_ERR_BAD_DTYPE;
  if (mode != DQ_SYMMETRIC && mode != DQ_ASYMMETRIC) return DQ_ERR_BAD_ARGUMENT;
  if (!is_code_type(y_dtype)) return DQ_ERR_BAD_DTYPE;
  if (y_dtype == DQ_INT4X2 && (cols % 2) != 0) return DQ_ERR_BAD_SHAPE;
  if (y_dtype == DQ_INT32 && (cols % 8) != 0) return DQ_ERR_BAD_SHAPE;
  if (num_groups < 0) return DQ_ERR_BAD_ARGUMENT;
  if (num_groups > DQ_MAX_GROUPS) return DQ_ERR_UNSUPPORTED;
  return DQ_OK;
}

}  // namespace

extern "C" {

const char* dq_status_string(dq_status s) {
  switch (s) {
    case DQ_OK: return "DQ_OK";
    case DQ_ERR_NULL_POINTER: return "DQ_ERR_NULL_POINTER: a required pointer is NULL";
    case DQ_ERR_BAD_SHAPE: return "DQ_ERR_BAD_SHAPE: invalid sizes for this call";
    case DQ_ERR_BAD_DTYPE: return "DQ_ERR_BAD_DTYPE: element type not allowed for this argument";
    case DQ_ERR_UNSUPPORTED: return "DQ_ERR_UNSUPPORTED: request not implemented by this library";
    case DQ_ERR_MISALIGNED: return "DQ_ERR_MISALIGNED: pointer below its element alignment";
    case DQ_ERR_WORKSPACE_TOO_SMALL: return "DQ_ERR_WORKSPACE_TOO_SMALL: workspace missing or too small";
    case DQ_ERR_CUDA: return "DQ_ERR_CUDA: the kernel launch failed";
    case DQ_ERR_BAD_ARGUMENT: return "DQ_ERR_BAD_ARGUMENT: invalid argument value";
  }
  return "unknown dq_status";
}

dq_status dq_get_workspace_size(int64_t rows, int64_t cols, dq_dtype x_dtype, dq_mode mode, dq_dtype y_dtype,
                                int32_t num_groups, size_t* workspace_bytes) {
  if (workspace_bytes == nullptr) return DQ_ERR_NULL_POINTER;
  const dq_status st = check_sizes(rows, cols, x_dtype, mode, y_dtype, num_groups);
  if (st != DQ_OK) return st;
  *workspace_bytes = num_groups > 0 ? sizeof(uint32_t) : 0;
  return DQ_OK;
}

dq_status dq_dynamic_quant(const void* x, dq_dtype x_dtype, int64_t rows, int64_t cols, const void* smooth,
                           dq_dtype smooth_dtype, const int32_t* group_index, int32_t num_groups, dq_mode mode,
                           dq_dtype y_dtype, void* y, float* scale, float* offset, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream) {
  dq_status st = check_sizes(rows, cols, x_dtype, mode, y_dtype, num_groups);
  if (st != DQ_OK) return st;
  if ((group_index != nullptr) != (num_groups > 0)) return DQ_ERR_BAD_ARGUMENT;
  if (group_index != nullptr && smooth == nullptr) return DQ_ERR_BAD_ARGUMENT;
  if (smooth != nullptr && !is_param_float(smooth_dtype)) return DQ_ERR_BAD_DTYPE;
  const size_t needed = num_groups > 0 ? sizeof(uint32_t) : 0;
  if (rows == 0) return DQ_OK;
  if (x == nullptr || y == nullptr || scale == nullptr) return DQ_ERR_NULL_POINTER;
  if (mode == DQ_ASYMMETRIC && offset == nullptr) return DQ_ERR_NULL_POINTER;
  if (needed > 0 && (workspace == nullptr || workspace_bytes < needed)) return DQ_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(x, 2) || !aligned(scale, 4)) return DQ_ERR_MISALIGNED;
  if (mode == DQ_ASYMMETRIC && !aligned(offset, 4)) return DQ_ERR_MISALIGNED;
  if (smooth != nullptr && !aligned(smooth, float_size(smooth_dtype))) return DQ_ERR_MISALIGNED;
  if (group_index != nullptr && !aligned(group_index, 4)) return DQ_ERR_MISALIGNED;
  if (needed > 0 && !aligned(workspace, 4)) return DQ_ERR_MISALIGNED;
  if (y_dtype == DQ_INT32 && !aligned(y, 4)) return DQ_ERR_MISALIGNED;

  dq::RowQuantArgs a{};
  a.x = x;
  a.rows = rows;
  a.cols = cols;
  a.smooth = smooth;
  a.smooth_dtype = static_cast<int>(smooth_dtype);
  a.group_index = group_index;
  a.num_groups = num_groups;
  a.y = y;
  a.scale = scale;
  a.offset = mode == DQ_ASYMMETRIC ? offset : nullptr;
  a.status = needed > 0 ? static_cast<uint32_t*>(workspace) : nullptr;

  // bulk-copy path: 16-byte rows of x, 16-byte aligned smooth rows and
  // naturally aligned code vectors; anything else takes the generic kernel
  const uintptr_t y_align = y_dtype == DQ_INT8 ? 8 : 4;
  const bool vec = (cols % 8) == 0 && aligned(x, 16) && aligned(y, y_align) &&
                   (smooth == nullptr || aligned(smooth, 16));
  const bool four = y_dtype != DQ_INT8;
  if (x_dtype == DQ_F16) {
    return mode == DQ_SYMMETRIC ? dq_host::quant_f16_sym(a, four, vec, stream)
                                : dq_host::quant_f16_asym(a, four, vec, stream);
  }
  return mode == DQ_SYMMETRIC ? dq_host::quant_bf16_sym(a, four, vec, stream)
                              : dq_host::quant_bf16_asym(a, four, vec, stream);
}

dq_status dq_ada_layernorm_quant_get_workspace_size(int64_t batch, int64_t seq, int64_t hidden, dq_dtype x_dtype,
                                                    dq_dtype param_dtype, size_t* workspace_bytes) {
  if (workspace_bytes == nullptr) return DQ_ERR_NULL_POINTER;
  const dq_status st = check_ada(batch, seq, hidden, x_dtype, param_dtype);
  if (st != DQ_OK) return st;
  *workspace_bytes = batch * seq > 0 ? ada_table_bytes(batch, hidden) : 0;
  return DQ_OK;
}

dq_status dq_ada_layernorm_quant(const void* x, dq_dtype x_dtype, int64_t batch, int64_t seq, int64_t hidden,
                                 const void* ada_scale, const void* ada_shift, const void* weight,
                                 const void* bias, const void* smooth, dq_dtype param_dtype, float epsilon,
                                 int8_t* out, float* quant_scale, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
  const dq_status st = check_ada(batch, seq, hidden, x_dtype, param_dtype);
  if (st != DQ_OK) return st;
  if (!std::isfinite(epsilon) || epsilon < 0.0f) return DQ_ERR_BAD_ARGUMENT;
  const int64_t rows = batch * seq;
  if (rows == 0) return DQ_OK;
  if (x == nullptr || ada_scale == nullptr || ada_shift == nullptr || out == nullptr || quant_scale == nullptr)
    return DQ_ERR_NULL_POINTER;
  if (workspace == nullptr || workspace_bytes < ada_table_bytes(batch, hidden)) return DQ_ERR_WORKSPACE_TOO_SMALL;
  const size_t ps = float_size(param_dtype);
  if (!aligned(x, 2) || !aligned(quant_scale, 4) || !aligned(ada_scale, ps) || !aligned(ada_shift, ps) ||
      (weight && !aligned(weight, ps)) || (bias && !aligned(bias, ps)) || (smooth && !aligned(smooth, ps)) ||
      !aligned(workspace, 16))
    return DQ_ERR_MISALIGNED;

  dq::AdaArgs a{};
  a.x = x;
  a.batch = batch;
  a.seq = seq;
  a.hidden = hidden;
  a.ada_scale = ada_scale;
  a.ada_shift = ada_shift;
  a.weight = weight;
  a.bias = bias;
  a.smooth = smooth;
  a.param_dtype = static_cast<int>(param_dtype);
  a.epsilon = epsilon;
  a.inv_hidden = 1.0 / static_cast<double>(hidden);
  a.table = static_cast<float*>(workspace);
  a.out = out;
  a.quant_scale = quant_scale;
  const bool vec = (hidden % 8) == 0 && aligned(x, 16) && aligned(out, 8);
  if (x_dtype == DQ_F16) return dq_host::ada_f16(a, vec, stream);
  return dq_host::ada_bf16(a, vec, stream);
}

dq_status dq_dequant_per_token(const void* y, dq_dtype y_dtype, int64_t rows, int64_t cols, const void* scale,
                               const void* offset, dq_dtype scale_dtype, void* out, dq_dtype out_dtype,
                               cudaStream_t stream) {
  return dequantize(dq::kPerToken, y, y_dtype, rows, cols, scale, offset, scale_dtype, 0, 1, out, out_dtype, true,
                    stream);
}

dq_status dq_dequant_per_group(const void* y, dq_dtype y_dtype, int64_t rows, int64_t cols, const void* scale,
                               const void* offset, dq_dtype scale_dtype, int64_t group_size, int32_t k_dim,
                               void* out, dq_dtype out_dtype, cudaStream_t stream) {
  if (group_size <= 0 || group_size % 32 != 0 || (k_dim != 0 && k_dim != 1)) return DQ_ERR_BAD_ARGUMENT;
  if (k_dim == 1) {
    const int64_t groups = (cols + group_size - 1) / group_size;
    return dequantize(dq::kGroupAlongRow, y, y_dtype, rows, cols, scale, offset, scale_dtype, group_size, groups,
                      out, out_dtype, true, stream);
  }
  // per-column tables are read as 16-byte vectors on the vectorised path
  const bool table_vec_ok = aligned(scale, 16) && (offset == nullptr || aligned(offset, 16));
  return dequantize(dq::kGroupDownColumn, y, y_dtype, rows, cols, scale, offset, scale_dtype, group_size, cols, out,
                    out_dtype, table_vec_ok, stream);
}

}  // extern "C"
