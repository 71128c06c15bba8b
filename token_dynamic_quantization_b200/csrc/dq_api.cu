// C ABI of the per-token dynamic quantization library (declared in include/dq.h).
//
// Host side of the two-phase convention of aclnnDynamicQuantV2 and
// aclnnAdaLayerNormQuant: every call validates its arguments on the host
// before anything is launched (the pages' "first-phase API implements input
// parameter verification"), then launches exactly one kernel on the caller's
// stream. The library allocates nothing and keeps no per-call state; the only
// cached values are per-device launch facts (SM count, occupancy).

#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "ada_layernorm_quant_kernels.cuh"
#include "dequant_kernels.cuh"
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

// ---------------------------------------------------------------- launch shapes

// Row-group shape: VPT 16-byte vectors per thread, tpr = 32 * G threads per row.
struct GroupShape {
  int vpt;
  int tpr;
};

constexpr size_t kMaxDynamicSmem = 200 * 1024;

// Allow `kernel` the dynamic shared memory it needs (once per kernel/device).
bool allow_smem(const void* kernel, int device) {
  struct Entry {
    const void* k;
    int device;
  };
  static Entry done[256];
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
  // (the shared-memory carveout is left to the driver: the smooth-scale
  // tables are read through L1 and need it to stay resident)
  if (used < 256) done[used++] = Entry{kernel, device};
  return true;
}

// Launch `kernel` as a programmatic dependent of the previous work in
// `stream`: it may start before that work finishes and waits for it
// (griddepcontrol.wait) before touching global memory.
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

// ---------------------------------------------------------------- dynamic quant dispatch

// Row-group geometry of the bulk-copy DynamicQuant kernel: a group of
// tpr = 32 * G threads owns a row, VPT in {2, 4, 8} vectors per thread; the
// shape wasting the fewest lanes wins, then the one whose VPT is closest to
// the target VPT (8 by default: more elements per thread amortize the
// per-row work; with smooth scales the fp32 products of pass 1 stay in
// registers for pass 2). DQ_WARP_STAGES row buffers per group; groups per CTA so that
// a CTA holds about DQ_WARP_CTA_BYTES_SMOOTH / _PLAIN of rows (measured: the
// smooth-scale path prefers several groups sharing a CTA, the plain path
// smaller CTAs).
#ifndef DQ_TARGET_VPT_SMOOTH
#define DQ_TARGET_VPT_SMOOTH 8
#endif
#ifndef DQ_TARGET_VPT_PLAIN
#define DQ_TARGET_VPT_PLAIN 8
#endif
#ifndef DQ_WARP_STAGES
#define DQ_WARP_STAGES 2
#endif
#ifndef DQ_WARP_CTA_BYTES_SMOOTH
#define DQ_WARP_CTA_BYTES_SMOOTH 65536
#endif
#ifndef DQ_WARP_CTA_BYTES_PLAIN
#define DQ_WARP_CTA_BYTES_PLAIN 32768
#endif

GroupShape pick_dq_shape(int64_t nvec, int target_vpt) {
  GroupShape best{0, 0};
  double best_eff = -1.0;
  static const int kVpts[5] = {2, 4, 6, 7, 8};
  for (int vpt : kVpts) {
    const int64_t warps = (nvec + 32 * vpt - 1) / (32 * vpt);
    if (warps > 16) continue;
    const int64_t tpr = warps * 32;
    const double eff = static_cast<double>(nvec) / static_cast<double>(tpr * vpt);
    const bool better = eff > best_eff + 1e-9 ||
                        (eff > best_eff - 1e-9 && std::abs(vpt - target_vpt) < std::abs(best.vpt - target_vpt));
    if (better) {
      best_eff = eff;
      best = GroupShape{vpt, static_cast<int>(tpr)};
    }
  }
  return best;
}

// Internal status of the bulk-copy launchers: the configuration cannot run on
// this device (shared memory or occupancy); the caller uses the generic kernel.
constexpr dq_status kNotLaunchable = static_cast<dq_status>(-1);

template <typename InT, int MODE, int OUT, int SMK, int VPT, bool kRagged>
dq_status launch_dq_tma(dq::RowQuantArgs a, int device, int sms, cudaStream_t stream) {
  const void* k = reinterpret_cast<const void*>(dq::dynamic_quant_tma_kernel<InT, MODE, OUT, SMK, VPT, kRagged>);
  const size_t smem = dq::dq_smem_bytes(a.groups, a.stages, a.stage_stride, a.group_index ? a.num_groups : 0);
  if (smem > kMaxDynamicSmem || !allow_smem(k, device)) return kNotLaunchable;
  const int block = a.tpr * a.groups;
  const int64_t wanted = (a.rows + a.groups - 1) / a.groups;
  const int64_t resident = static_cast<int64_t>(sms) * blocks_per_sm(k, block, smem, device);
  if (resident < 1) return kNotLaunchable;
  const int grid = static_cast<int>(wanted < resident ? wanted : resident);
  return launch_programmatic(dq::dynamic_quant_tma_kernel<InT, MODE, OUT, SMK, VPT, kRagged>, a, grid, block, smem,
                             stream);
}

template <typename InT, int MODE, int OUT, int SMK, int VPT>
dq_status launch_dq_ragged(dq::RowQuantArgs a, int device, int sms, cudaStream_t stream) {
  // exact tiling (the row is G * 32 * VPT vectors) needs no per-vector bounds checks
  if ((a.cols >> 3) == static_cast<int64_t>(a.tpr) * VPT)
    return launch_dq_tma<InT, MODE, OUT, SMK, VPT, false>(a, device, sms, stream);
  return launch_dq_tma<InT, MODE, OUT, SMK, VPT, true>(a, device, sms, stream);
}

template <typename InT, int MODE, int OUT, int SMK>
dq_status launch_dq_vpt(dq::RowQuantArgs a, int vpt, int device, int sms, cudaStream_t stream) {
  switch (vpt) {
    case 2: return launch_dq_ragged<InT, MODE, OUT, SMK, 2>(a, device, sms, stream);
    case 4: return launch_dq_ragged<InT, MODE, OUT, SMK, 4>(a, device, sms, stream);
    case 6: return launch_dq_ragged<InT, MODE, OUT, SMK, 6>(a, device, sms, stream);
    case 7: return launch_dq_ragged<InT, MODE, OUT, SMK, 7>(a, device, sms, stream);
    default: return launch_dq_ragged<InT, MODE, OUT, SMK, 8>(a, device, sms, stream);
  }
}

template <typename InT, int MODE, int OUT>
dq_status launch_dynamic_quant(dq::RowQuantArgs a, bool vector_ok, cudaStream_t stream) {
  const int device = current_device();
  const int sms = sm_count(device);
  if (vector_ok) {
    const GroupShape gs =
        pick_dq_shape(a.cols >> 3, a.smooth != nullptr ? DQ_TARGET_VPT_SMOOTH : DQ_TARGET_VPT_PLAIN);
    if (gs.vpt > 0) {
      const int64_t row_bytes = a.cols * 2;
      const uint32_t stride = static_cast<uint32_t>((row_bytes + 127) / 128 * 128);
      const int stages = DQ_WARP_STAGES;
      const int64_t cta_bytes = a.smooth != nullptr ? DQ_WARP_CTA_BYTES_SMOOTH : DQ_WARP_CTA_BYTES_PLAIN;
      int64_t groups = cta_bytes / (static_cast<int64_t>(stages) * stride);
      const int64_t max_groups = dq::kWarpKernelMaxThreads / gs.tpr;
      groups = groups < 1 ? 1 : (groups > max_groups ? max_groups : groups);
      groups = groups > 15 ? 15 : groups;  // named barriers 1..15
      a.groups = static_cast<int>(groups);
      a.stages = stages;
      a.stage_stride = stride;
      a.tpr = gs.tpr;
      if (dq::dq_smem_bytes(a.groups, stages, stride, a.group_index ? a.num_groups : 0) <= kMaxDynamicSmem) {
        dq_status st;
        if (a.smooth == nullptr) {
          st = launch_dq_vpt<InT, MODE, OUT, dq::kSmNone>(a, gs.vpt, device, sms, stream);
        } else if (a.smooth_dtype == dq::kF32) {
          st = launch_dq_vpt<InT, MODE, OUT, dq::kSmF32>(a, gs.vpt, device, sms, stream);
        } else if (a.smooth_dtype == dq::kF16) {
          st = launch_dq_vpt<InT, MODE, OUT, dq::kSmF16>(a, gs.vpt, device, sms, stream);
        } else {
          st = launch_dq_vpt<InT, MODE, OUT, dq::kSmBF16>(a, gs.vpt, device, sms, stream);
        }
        if (st != kNotLaunchable) return st;
      }
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

// ---------------------------------------------------------------- AdaLayerNormQuant dispatch

size_t ada_table_bytes(int64_t batch, int64_t hidden) { return static_cast<size_t>(batch * hidden) * 8; }

// Affine-table kernel (ordinary launch), then the row kernel as its
// programmatic dependent (it may start before the table is finished and waits
// for it with griddepcontrol.wait).
dq_status launch_ada_table(const dq::AdaArgs& a, int sms, cudaStream_t stream) {
  const int64_t total = a.batch * a.hidden;
  int64_t grid = (total + dq::kTableBlock - 1) / dq::kTableBlock;
  if (grid > 2 * sms) grid = 2 * sms;
  return launch_programmatic(dq::ada_affine_table_kernel, a, static_cast<int>(grid), dq::kTableBlock, 0, stream);
}

template <typename InT, int VPT, bool kRagged>
dq_status launch_ada_tma(dq::AdaArgs a, int device, int sms, cudaStream_t stream) {
  void (*kfn)(const dq::AdaArgs) = dq::ada_layernorm_quant_tma_kernel<InT, VPT, kRagged>;
  const void* k = reinterpret_cast<const void*>(kfn);
  const size_t smem = dq::ada_smem_bytes(a.groups, a.stages, a.stage_stride);
  if (smem > kMaxDynamicSmem || !allow_smem(k, device)) return kNotLaunchable;
  const int block = a.tpr * a.groups;
  const int64_t rows = a.batch * a.seq;
  const int64_t wanted = (rows + a.groups - 1) / a.groups;
  const int64_t resident = static_cast<int64_t>(sms) * blocks_per_sm(k, block, smem, device);
  if (resident < 1) return kNotLaunchable;
  const int grid = static_cast<int>(wanted < resident ? wanted : resident);
  dq_status st = launch_ada_table(a, sms, stream);
  if (st != DQ_OK) return st;
  return launch_programmatic(kfn, a, grid, block, smem, stream);
}

template <typename InT, int VPT>
dq_status launch_ada_ragged(dq::AdaArgs a, int device, int sms, cudaStream_t stream) {
  // exact tiling (the row is G * 32 * VPT vectors) needs no per-vector bounds checks
  if ((a.hidden >> 3) == static_cast<int64_t>(a.tpr) * VPT) return launch_ada_tma<InT, VPT, false>(a, device, sms, stream);
  return launch_ada_tma<InT, VPT, true>(a, device, sms, stream);
}

// AdaLayerNorm row-group shape: VPT in {2, 3, 4, 6, 8}, fewest wasted lanes,
// then VPT closest to DQ_ADA_TARGET_VPT (more elements per thread amortize the
// two row reductions; the row share stays in registers). DQ_ADA_STAGES row
// buffers per group, one of them holding the row being processed.
#ifndef DQ_ADA_TARGET_VPT
#define DQ_ADA_TARGET_VPT 6  // hidden 3072: 2 warps x 6 vectors per row (2811 GB/s) over 3 x 4 (2652)
#endif
#ifndef DQ_ADA_CTA_BYTES
#define DQ_ADA_CTA_BYTES 147456  // 8 row groups of 64 threads at hidden 3072: 16 warps per SM
#endif
#ifndef DQ_ADA_STAGES
#define DQ_ADA_STAGES 3
#endif

GroupShape pick_ada_shape(int64_t nvec) {
  GroupShape best{0, 0};
  double best_eff = -1.0;
  static const int kVpts[5] = {2, 3, 4, 6, 8};
  for (int vpt : kVpts) {
    const int64_t warps = (nvec + 32 * vpt - 1) / (32 * vpt);
    if (warps > 16) continue;
    const int64_t tpr = warps * 32;
    const double eff = static_cast<double>(nvec) / static_cast<double>(tpr * vpt);
    const bool better = eff > best_eff + 1e-9 || (eff > best_eff - 1e-9 && std::abs(vpt - DQ_ADA_TARGET_VPT) <
                                                                             std::abs(best.vpt - DQ_ADA_TARGET_VPT));
    if (better) {
      best_eff = eff;
      best = GroupShape{vpt, static_cast<int>(tpr)};
    }
  }
  return best;
}

template <typename InT>
dq_status launch_ada(dq::AdaArgs a, bool vector_ok, cudaStream_t stream) {
  const int device = current_device();
  const int sms = sm_count(device);
  if (vector_ok) {
    const GroupShape gs = pick_ada_shape(a.hidden >> 3);
    if (gs.vpt > 0) {
      const uint32_t stride = static_cast<uint32_t>((a.hidden * 2 + 127) / 128 * 128);
      const int stages = DQ_ADA_STAGES;
      int64_t groups = DQ_ADA_CTA_BYTES / (static_cast<int64_t>(stages) * stride);
      const int64_t max_groups = dq::kAdaMaxBlock / gs.tpr;
      groups = groups < 1 ? 1 : (groups > max_groups ? max_groups : groups);
      groups = groups > 15 ? 15 : groups;
      a.tpr = gs.tpr;
      a.groups = static_cast<int>(groups);
      a.stages = stages;
      a.stage_stride = stride;
      if (dq::ada_smem_bytes(a.groups, stages, stride) <= kMaxDynamicSmem) {
        dq_status st;
        switch (gs.vpt) {
          case 2: st = launch_ada_ragged<InT, 2>(a, device, sms, stream); break;
          case 3: st = launch_ada_ragged<InT, 3>(a, device, sms, stream); break;
          case 4: st = launch_ada_ragged<InT, 4>(a, device, sms, stream); break;
          case 6: st = launch_ada_ragged<InT, 6>(a, device, sms, stream); break;
          default: st = launch_ada_ragged<InT, 8>(a, device, sms, stream); break;
        }
        if (st != kNotLaunchable) return st;
      }
    }
  }
  dq_status st = launch_ada_table(a, sms, stream);
  if (st != DQ_OK) return st;
  const void* k = reinterpret_cast<const void*>(dq::ada_layernorm_quant_generic_kernel<InT>);
  const int64_t rows = a.batch * a.seq;
  const int64_t resident = static_cast<int64_t>(sms) * blocks_per_sm(k, dq::kAdaGenericBlock, 0, device);
  const int grid = static_cast<int>(rows < resident ? rows : resident);
  dq::ada_layernorm_quant_generic_kernel<InT><<<grid, dq::kAdaGenericBlock, 0, stream>>>(a);
  return launch_status();
}

// ---------------------------------------------------------------- dequantization dispatch

template <int OUT, bool kFour, bool kOff, int LAYOUT>
dq_status launch_dequant(const dq::DequantArgs& a, bool vec, cudaStream_t stream) {
  if (vec) {
    // one warp per row chunk, a grid that covers every chunk (capped: the
    // kernel loops beyond the cap)
    void (*kfn)(const dq::DequantArgs) = dq::dequant_vec_kernel<OUT, kFour, kOff, LAYOUT>;
    const int64_t nvec = a.cols / (kFour ? 32 : 16);
    constexpr int kUnroll = dq::dequant_unroll<LAYOUT>();
    const int64_t chunks = (nvec + 32 * kUnroll - 1) / (32 * kUnroll);
    const int64_t warps_per_block = dq::kDequantBlock / 32;
    int64_t grid = (a.rows * chunks + warps_per_block - 1) / warps_per_block;
    if (grid > (int64_t(1) << 30)) grid = int64_t(1) << 30;
    return launch_programmatic(kfn, a, static_cast<int>(grid), dq::kDequantBlock, 0, stream);
  }
  const int device = current_device();
  const int sms = sm_count(device);
  void (*gfn)(const dq::DequantArgs) = dq::dequant_generic_kernel<OUT, kFour, kOff, LAYOUT>;
  const int64_t resident =
      static_cast<int64_t>(sms) * blocks_per_sm(reinterpret_cast<const void*>(gfn), dq::kDequantBlock, 0, device);
  const int64_t g = a.rows < resident ? a.rows : resident;
  return launch_programmatic(gfn, a, static_cast<int>(g < 1 ? 1 : g), dq::kDequantBlock, 0, stream);
}

// Shared validation and dispatch of the two dequantization entry points.
template <int LAYOUT>
dq_status dequantize(const void* y, dq_dtype y_dtype, int64_t rows, int64_t cols, const void* scale,
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
  const bool has_offset = offset != nullptr;
  const int64_t per_vec = four ? 32 : 16;
  const bool vec = cols % per_vec == 0 && aligned(y, 16) && aligned(out, 16) && table_vec_ok;
  switch (out_kind * 4 + (four ? 2 : 0) + (has_offset ? 1 : 0)) {
#define DQ_DEQ_CASE(O, F, H)              \
  case O * 4 + (F ? 2 : 0) + (H ? 1 : 0): \
    return launch_dequant<O, F, H, LAYOUT>(a, vec, stream);
    DQ_DEQ_CASE(0, false, false) DQ_DEQ_CASE(0, false, true) DQ_DEQ_CASE(0, true, false) DQ_DEQ_CASE(0, true, true)
    DQ_DEQ_CASE(1, false, false) DQ_DEQ_CASE(1, false, true) DQ_DEQ_CASE(1, true, false) DQ_DEQ_CASE(1, true, true)
    DQ_DEQ_CASE(2, false, false) DQ_DEQ_CASE(2, false, true) DQ_DEQ_CASE(2, true, false) DQ_DEQ_CASE(2, true, true)
#undef DQ_DEQ_CASE
    default:
      return DQ_ERR_BAD_DTYPE;
  }
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
  if (x_dtype == DQ_F16) return dispatch_mode_out<__half>(a, mode, y_dtype, vec, stream);
  return dispatch_mode_out<__nv_bfloat16>(a, mode, y_dtype, vec, stream);
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
  if (x_dtype == DQ_F16) return launch_ada<__half>(a, vec, stream);
  return launch_ada<__nv_bfloat16>(a, vec, stream);
}

dq_status dq_dequant_per_token(const void* y, dq_dtype y_dtype, int64_t rows, int64_t cols, const void* scale,
                               const void* offset, dq_dtype scale_dtype, void* out, dq_dtype out_dtype,
                               cudaStream_t stream) {
  return dequantize<dq::kPerToken>(y, y_dtype, rows, cols, scale, offset, scale_dtype, 0, 1, out, out_dtype, true,
                                   stream);
}

dq_status dq_dequant_per_group(const void* y, dq_dtype y_dtype, int64_t rows, int64_t cols, const void* scale,
                               const void* offset, dq_dtype scale_dtype, int64_t group_size, int32_t k_dim,
                               void* out, dq_dtype out_dtype, cudaStream_t stream) {
  if (group_size <= 0 || group_size % 32 != 0 || (k_dim != 0 && k_dim != 1)) return DQ_ERR_BAD_ARGUMENT;
  if (k_dim == 1) {
    const int64_t groups = (cols + group_size - 1) / group_size;
    return dequantize<dq::kGroupAlongRow>(y, y_dtype, rows, cols, scale, offset, scale_dtype, group_size, groups,
                                          out, out_dtype, true, stream);
  }
  // per-column tables are read as 16-byte vectors on the vectorised path
  const bool table_vec_ok = aligned(scale, 16) && (offset == nullptr || aligned(offset, 16));
  return dequantize<dq::kGroupDownColumn>(y, y_dtype, rows, cols, scale, offset, scale_dtype, group_size, cols, out,
                                          out_dtype, table_vec_ok, stream);
}

}  // extern "C"
