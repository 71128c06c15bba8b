// Host-side launch plumbing shared by the library's translation units:
// cached per-device launch facts (SM count, occupancy, shared-memory opt-in),
// programmatic dependent launches, and the internal dispatch entry points
// that dq_api.cu calls after validating a request.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "dq.h"

namespace dq {
struct RowQuantArgs;
struct AdaArgs;
struct DequantArgs;
}  // namespace dq

namespace dq_host {

constexpr int kMaxDevices = 64;
constexpr size_t kMaxDynamicSmem = 200 * 1024;

// Internal status of the bulk-copy launchers: the configuration cannot run on
// this device (shared memory or occupancy); the caller uses the generic kernel.
constexpr dq_status kNotLaunchable = static_cast<dq_status>(-1);

inline int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) {
    cudaGetLastError();
    d = 0;
  }
  return d;
}

inline int sm_count(int device) {
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
inline int blocks_per_sm(const void* kernel, int block, size_t smem, int device) {
  struct Entry {
    const void* k;
    int block;
    size_t smem;
    int device;
    int value;
  };
  static Entry cache[512];
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
  if (used < 512) cache[used++] = Entry{kernel, block, smem, device, n};
  return n;
}

// Allow `kernel` the dynamic shared memory it needs (once per kernel/device).
inline bool allow_smem(const void* kernel, int device) {
  struct Entry {
    const void* k;
    int device;
  };
  static Entry done[512];
  static int used = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i) {
    if (done[i].k == kernel && done[i].device == device) return true;
  }
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kMaxDynamicSmem)) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (used < 512) done[used++] = Entry{kernel, device};
  return true;
}

// The same opt-in for an explicit number of bytes.
inline bool allow_smem_bytes(const void* kernel, int device, size_t bytes) {
  struct Entry {
    const void* k;
    int device;
    size_t bytes;
  };
  static Entry done[512];
  static int used = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i) {
    if (done[i].k == kernel && done[i].device == device && done[i].bytes >= bytes) return true;
  }
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
      cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (used < 512) done[used++] = Entry{kernel, device, bytes};
  return true;
}

// Largest block a compiled kernel can be launched with (its registers per
// thread, rounded as the hardware allocates them; 0 if unknown); cached.
inline int kernel_max_threads(const void* kernel, int device) {
  struct Entry {
    const void* k;
    int device;
    int threads;
  };
  static Entry cache[512];
  static int used = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i) {
    if (cache[i].k == kernel && cache[i].device == device) return cache[i].threads;
  }
  cudaFuncAttributes attr{};
  if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (used < 512) cache[used++] = Entry{kernel, device, attr.maxThreadsPerBlock};
  return attr.maxThreadsPerBlock;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline dq_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

// Launch `kernel` as a programmatic dependent of the previous work in
// `stream`: it may start before that work finishes and waits for it
// (griddepcontrol.wait) before it reads or writes global memory (the ring
// kernels issue only L2 prefetch hints before the wait).
template <typename Args>
dq_status launch_programmatic(void (*kernel)(const Args), const Args& a, int grid, int block, size_t smem,
                              cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, a) != cudaSuccess) {
    cudaGetLastError();
    return DQ_ERR_CUDA;
  }
  return launch_status();
}

// ---- internal dispatchers (one translation unit each; arguments validated)

// DynamicQuant for one input type and mode; `four`: 4-bit codes (INT4X2 or
// INT32), `vec`: the bulk-copy path's alignment holds.
dq_status quant_bf16_sym(const dq::RowQuantArgs& a, bool four, bool vec, cudaStream_t s);
dq_status quant_bf16_asym(const dq::RowQuantArgs& a, bool four, bool vec, cudaStream_t s);
dq_status quant_f16_sym(const dq::RowQuantArgs& a, bool four, bool vec, cudaStream_t s);
dq_status quant_f16_asym(const dq::RowQuantArgs& a, bool four, bool vec, cudaStream_t s);

// AdaLayerNormQuant (both launches) for one input type.
dq_status ada_bf16(const dq::AdaArgs& a, bool vec, cudaStream_t s);
dq_status ada_f16(const dq::AdaArgs& a, bool vec, cudaStream_t s);

// Dequantization; `layout` is dq::kPerToken, kGroupAlongRow or kGroupDownColumn.
dq_status dequant(const dq::DequantArgs& a, int layout, int out_kind, bool four, bool has_offset, bool vec,
                  cudaStream_t s);

}  // namespace dq_host
