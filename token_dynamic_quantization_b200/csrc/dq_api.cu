// C ABI of the per-token dynamic quantization library (declared in include/dq.h).
//
// Host side of the two-phase convention of aclnnDynamicQuantV2 and
// aclnnAdaLayerNormQuant: every call validates its arguments on the host
// before anything is launched (the pages' "first-phase API implements input
// parameter verification"), then launches exactly one kernel on the caller's
// stream. The library allocates nothing and keeps no per-call state; the only
// cached values are per-device launch facts (SM count, occupancy).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "ada_layernorm_quant_kernels.cuh"
#include "dq.h"
#include "dynamic_quant_kernels.cuh"

namespace {

// ---------------------------------------------------------------- launch facts

constexpr int kMaxDevices = 64;

int sm_count(int device) {
  static int cache[kMaxDevices] = {0};
  if (device < 0 || device >= kMaxDevices) return 148;
  if (cache[device] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0) n = 148;
    cache[device] = n;
  }
  return cache[device];
}

// Resident CTAs per SM for (kernel, block, dynamic smem); cached.
int blocks_per_sm(const void* kernel, int block, size_t smem, int device) {
  struct Entry {
    const void* k;
    int block;
    size_t smem;
    int device;
    int value;
  };
  static Entry cache[256];
  static int used = 0;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
      const Entry& e = cache[i];
      if (e.k == kernel && e.block == block && e.smem == smem && e.device == device) return e.value;
    }
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, block, smem) != cudaSuccess || n <= 0) {
    cudaGetLastError();  // clear; fall back to one resident CTA
    n = 1;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (used < 256) cache[used++] = Entry{kernel, block, smem, device, n};
  return n;
}

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) {
    cudaGetLastError();
    d = 0;
  }
  return d;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t float_size(dq_dtype t) { return t == DQ_F32 ? 4 : 2; }

bool is_input_float(dq_dtype t) { return t == DQ_F16 || t == DQ_BF16; }
bool is_param_float(dq_dtype t) { return t == DQ_F32 || t == DQ_F16 || t == DQ_BF16; }
bool is_code_type(dq_dtype t) { return t == DQ_INT8 || t == DQ_INT4X2 || t == DQ_INT32; }

dq_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

// ---------------------------------------------------------------- dynamic quant dispatch

template <typename InT, int MODE, int OUT>
dq_status launch_dynamic_quant(dq::RowQuantArgs a, bool vector_ok, cudaStream_t stream) {
  const int device = current_device();
  const int sms = sm_count(device);
  const int64_t nvec = a.cols >> 3;
  const size_t smem = a.group_index ? static_cast<size_t>(a.num_groups) * sizeof(int32_t) : 0;
  if (vector_ok) {
    const int vpt = nvec >= 128 ? 4 : (nvec >= 64 ? 2 : 1);
    const int64_t tpr64 = ((nvec + vpt - 1) / vpt + 31) / 32 * 32;
    if (tpr64 <= dq::kMaxBlock) {
      a.tpr = static_cast<int>(tpr64);
      a.groups = a.tpr >= 256 ? 1 : 256 / a.tpr;
      const int block = a.tpr * a.groups;
      const void* k = vpt == 4 ? reinterpret_cast<const void*>(dq::dynamic_quant_vec_kernel<InT, MODE, OUT, 4>)
                    : vpt == 2 ? reinterpret_cast<const void*>(dq::dynamic_quant_vec_kernel<InT, MODE, OUT, 2>)
                               : reinterpret_cast<const void*>(dq::dynamic_quant_vec_kernel<InT, MODE, OUT, 1>);
      const int64_t wanted = (a.rows + a.groups - 1) / a.groups;
      const int64_t resident = static_cast<int64_t>(sms) * blocks_per_sm(k, block, smem, device);
      const int grid = static_cast<int>(wanted < resident ? wanted : resident);
      if (vpt == 4) {
        dq::dynamic_quant_vec_kernel<InT, MODE, OUT, 4><<<grid, block, smem, stream>>>(a);
      } else if (vpt == 2) {
        dq::dynamic_quant_vec_kernel<InT, MODE, OUT, 2><<<grid, block, smem, stream>>>(a);
      } else {
        dq::dynamic_quant_vec_kernel<InT, MODE, OUT, 1><<<grid, block, smem, stream>>>(a);
      }
      return launch_status();
    }
  }
  const void* k = reinterpret_cast<const void*>(dq::dynamic_quant_generic_kernel<InT, MODE, OUT>);
  const int64_t resident = static_cast<int64_t>(sms) * blocks_per_sm(k, dq::kGenericBlock, 0, device);
  const int grid = static_cast<int>(a.rows < resident ? a.rows : resident);
  dq::dynamic_quant_generic_kernel<InT, MODE, OUT><<<grid, dq::kGenericBlock, 0, stream>>>(a);
  return launch_status();
}

template <typename InT>
dq_status dispatch_mode_out(const dq::RowQuantArgs& a, dq_mode mode, dq_dtype y_dtype, bool vec,
                            cudaStream_t s) {
  const bool four = y_dtype != DQ_INT8;
  if (mode == DQ_SYMMETRIC) {
    return four ? launch_dynamic_quant<InT, dq::kSym, dq::kOutInt4>(a, vec, s)
                : launch_dynamic_quant<InT, dq::kSym, dq::kOutInt8>(a, vec, s);
  }
  return four ? launch_dynamic_quant<InT, dq::kAsym, dq::kOutInt4>(a, vec, s)
              : launch_dynamic_quant<InT, dq::kAsym, dq::kOutInt8>(a, vec, s);
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
    case DQ_ERR_UNSUPPORTED: return "DQ_ERR_UNSUPPORTED: request not implemented by this build";
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

  // vector path: 16-byte rows of x and naturally aligned code vectors
  const uintptr_t y_align = y_dtype == DQ_INT8 ? 8 : 4;
  const bool vec = (cols % 8) == 0 && aligned(x, 16) && aligned(y, y_align);
  if (x_dtype == DQ_F16) return dispatch_mode_out<__half>(a, mode, y_dtype, vec, stream);
  return dispatch_mode_out<__nv_bfloat16>(a, mode, y_dtype, vec, stream);
}

dq_status dq_ada_layernorm_quant(const void* x, dq_dtype x_dtype, int64_t batch, int64_t seq, int64_t hidden,
                                 const void* ada_scale, const void* ada_shift, const void* weight,
                                 const void* bias, const void* smooth, dq_dtype param_dtype, float epsilon,
                                 int8_t* out, float* quant_scale, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (batch < 0 || seq < 0 || hidden < 1) return DQ_ERR_BAD_SHAPE;
  if (hidden > (int64_t(1) << 31) || batch > (int64_t(1) << 40) || seq > (int64_t(1) << 40))
    return DQ_ERR_BAD_SHAPE;
  if (!is_input_float(x_dtype) || !is_param_float(param_dtype)) return DQ_ERR_BAD_DTYPE;
  if (!std::isfinite(epsilon) || epsilon < 0.0f) return DQ_ERR_BAD_ARGUMENT;
  const int64_t rows = batch * seq;
  if (rows == 0) return DQ_OK;
  if (x == nullptr || ada_scale == nullptr || ada_shift == nullptr || out == nullptr || quant_scale == nullptr)
    return DQ_ERR_NULL_POINTER;
  const size_t ps = float_size(param_dtype);
  if (!aligned(x, 2) || !aligned(quant_scale, 4) || !aligned(ada_scale, ps) || !aligned(ada_shift, ps) ||
      (weight && !aligned(weight, ps)) || (bias && !aligned(bias, ps)) || (smooth && !aligned(smooth, ps)))
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
  a.out = out;
  a.quant_scale = quant_scale;

  const int device = current_device();
  const int sms = sm_count(device);
  const int64_t nvec = hidden / 8;
  const bool vec = (hidden % 8) == 0 && aligned(x, 16) && aligned(out, 8) && nvec <= dq::kAdaMaxBlock;
  if (vec) {
    a.tpr = static_cast<int>((nvec + 31) / 32 * 32);
    a.groups = a.tpr >= 256 ? 1 : 256 / a.tpr;
    const int block = a.tpr * a.groups;
    const void* k = x_dtype == DQ_F16 ? reinterpret_cast<const void*>(dq::ada_layernorm_quant_vec_kernel<__half>)
                                      : reinterpret_cast<const void*>(dq::ada_layernorm_quant_vec_kernel<__nv_bfloat16>);
    const int64_t wanted = (rows + a.groups - 1) / a.groups;
    const int64_t resident = static_cast<int64_t>(sms) * blocks_per_sm(k, block, 0, device);
    const int grid = static_cast<int>(wanted < resident ? wanted : resident);
    if (x_dtype == DQ_F16) {
      dq::ada_layernorm_quant_vec_kernel<__half><<<grid, block, 0, stream>>>(a);
    } else {
      dq::ada_layernorm_quant_vec_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(a);
    }
    return launch_status();
  }
  const void* k = x_dtype == DQ_F16 ? reinterpret_cast<const void*>(dq::ada_layernorm_quant_generic_kernel<__half>)
                                    : reinterpret_cast<const void*>(dq::ada_layernorm_quant_generic_kernel<__nv_bfloat16>);
  const int64_t resident = static_cast<int64_t>(sms) * blocks_per_sm(k, dq::kAdaGenericBlock, 0, device);
  const int grid = static_cast<int>(rows < resident ? rows : resident);
  if (x_dtype == DQ_F16) {
    dq::ada_layernorm_quant_generic_kernel<__half><<<grid, dq::kAdaGenericBlock, 0, stream>>>(a);
  } else {
    dq::ada_layernorm_quant_generic_kernel<__nv_bfloat16><<<grid, dq::kAdaGenericBlock, 0, stream>>>(a);
  }
  return launch_status();
}

}  // extern "C"
