// DynamicQuant launch selection (aclnnDynamicQuantV2): the bulk-copy row
// kernel's shape for a row width, or the generic kernel. Included by one
// translation unit per (input type, mode) so the instantiations compile in
// parallel.
#pragma once

#include <cstdlib>

#include "dq_launch.cuh"
#include "dynamic_quant_kernels.cuh"

namespace dq_host {

// Row-group shape: VPT 16-byte vectors per thread, tpr = 32 * G threads per row.
struct GroupShape {
  int vpt;
  int tpr;
};

// Row-group geometry of the bulk-copy DynamicQuant kernel: a group of
// tpr = 32 * G threads owns a row, VPT in {2, 4, 6, 7, 8} vectors per thread;
// the shape wasting the fewest lanes wins, then the one whose VPT is closest
// to the target VPT (8 by default: more elements per thread amortize the
// per-row work; with smooth scales the fp32 products of pass 1 stay in
// registers for pass 2). DQ_WARP_STAGES row buffers per group; groups per CTA
// so that a CTA holds about DQ_WARP_CTA_BYTES_SMOOTH / _PLAIN of rows
// (measured: the smooth-scale path prefers several groups sharing a CTA, the
// plain path smaller CTAs).
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

inline GroupShape pick_dq_shape(int64_t nvec, int target_vpt) {
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

}  // namespace dq_host

// One translation unit per (input type, mode): both code widths.
#define DQ_DEFINE_QUANT_DISPATCH(NAME, INT, MODE)                                                         \
  dq_status dq_host::NAME(const dq::RowQuantArgs& a, bool four, bool vec, cudaStream_t s) {            \
    return four ? launch_dynamic_quant<INT, MODE, dq::kOutInt4>(a, vec, s)                              \
                : launch_dynamic_quant<INT, MODE, dq::kOutInt8>(a, vec, s);                             \
  }
