// DynamicQuant launch selection (aclnnDynamicQuantV2): the ring kernel's
// shape for a row width, or the generic kernel. Included by one
// translation unit per (input type, mode) so the instantiations compile in
// parallel.
#pragma once

#include <cstdlib>

#include "dq_launch.cuh"
#include "dynamic_quant_kernels.cuh"
#include "dynamic_quant_ring.cuh"

namespace dq_host {

// Row-group shape: VPT 16-byte vectors per thread, tpr = 32 * G threads per row.
struct GroupShape {
  int vpt;
  int tpr;
};

// Row-group geometry of the ring kernel: a group of tpr = 32 * G threads owns
// a row, VPT in {2, 4, 6, 7, 8} 16-byte vectors per thread; the shape wasting
// the fewest lanes wins, then the one whose VPT is closest to the target VPT
// (8: more elements per thread amortize the per-row work, and with smooth
// scales the fp32 products of pass 1 stay in registers for pass 2).
#ifndef DQ_TARGET_VPT_SMOOTH
#define DQ_TARGET_VPT_SMOOTH 8
#endif
#ifndef DQ_TARGET_VPT_PLAIN
#define DQ_TARGET_VPT_PLAIN 8
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

// Largest dynamic shared memory of one CTA on sm_100 (227 KB), less the
// ring kernel's static shared memory and a reserve.
constexpr size_t kRingSmemBudget = 232448 - 1024;
#ifndef DQ_RING_MAX_SLOTS
#define DQ_RING_MAX_SLOTS 32
#endif
// Bytes of row slots per CTA. Measured on the 8192 x 4096 workload (one CTA
// per SM, 8 row groups): 12 slots of 8 KB 20.1 us, 16 slots 22.2 us, 26 slots
// 23.6 us; on 32768 rows 8 slots 67.7 us, 26 slots 73.9 us. A deeper ring
// puts more rows in flight than the HBM needs and makes each row's copy
// slower to land.
#ifndef DQ_RING_BYTES
#define DQ_RING_BYTES (100 * 1024)
#endif

// Ring kernel launch: one CTA per SM (fewer for few rows), NC row groups of
// G = tpr / 32 warps, as many as the kernel's largest block holds (at most 15
// with G > 1: one named barrier each), and NS row slots of about
// DQ_RING_BYTES in all (NC <= NS <= rows of a CTA).
template <typename InT, int MODE, int OUT, int SMK, int VPT, bool kRagged, bool kSS>
dq_status launch_dq_ring(dq::RowQuantArgs a, int device, int sms, cudaStream_t stream) {
  void (*kfn)(const dq::RowQuantArgs) = dq::dynamic_quant_ring_kernel<InT, MODE, OUT, SMK, VPT, kRagged, kSS>;
  const void* k = reinterpret_cast<const void*>(kfn);
  if (!allow_smem_bytes(k, device, kRingSmemBudget)) return kNotLaunchable;
  const int max_threads = kernel_max_threads(k, device);
  const int G = a.tpr / 32;
  const int64_t grid = a.rows < sms ? a.rows : sms;
  const int64_t per_cta = (a.rows + grid - 1) / grid;
  int64_t nc = max_threads / a.tpr;
  if (G > 1 && nc > 15) nc = 15;
  if (nc > per_cta) nc = per_cta;
  const size_t smooth_row = static_cast<size_t>(a.cols) * (SMK == dq::kSmF32 ? 4 : 2);
  size_t smooth_bytes = kSS ? smooth_row : 0;
  a.moe_stage = 0;
  if (!kSS && SMK != dq::kSmNone && a.group_index != nullptr) {
    // MoE: two expert smooth rows staged per CTA, when a ring of one slot per
    // group still fits beside them
    const size_t with = dq::ring_smem_bytes(static_cast<int>(nc), a.stage_stride, 2 * smooth_row, a.num_groups);
    if (with <= kRingSmemBudget) {
      smooth_bytes = 2 * smooth_row;
      a.moe_stage = 1;
    }
  }
  const size_t fixed = dq::ring_smem_bytes(0, a.stage_stride, smooth_bytes, a.group_index ? a.num_groups : 0);
  if (fixed >= kRingSmemBudget) return kNotLaunchable;
  const int64_t ns_fit = static_cast<int64_t>((kRingSmemBudget - fixed) / (a.stage_stride + 16));
  int64_t ns = DQ_RING_BYTES / a.stage_stride;
  if (ns < nc) ns = nc;  // at least one slot per group
  if (ns > ns_fit) ns = ns_fit;
  if (ns > DQ_RING_MAX_SLOTS) ns = DQ_RING_MAX_SLOTS;
  if (ns > per_cta) ns = per_cta;
  if (nc > ns) nc = ns;
  if (nc < 1) return kNotLaunchable;
  a.groups = static_cast<int>(nc);
  a.stages = static_cast<int>(ns);
  const size_t smem = dq::ring_smem_bytes(a.stages, a.stage_stride, smooth_bytes, a.group_index ? a.num_groups : 0);
  const int block = a.tpr * a.groups;
  if (blocks_per_sm(k, block, smem, device) < 1) return kNotLaunchable;
  return launch_programmatic(kfn, a, static_cast<int>(grid), block, smem, stream);
}

// Few short rows: one warp per row, one warp per CTA (see
// dynamic_quant_warp_kernel).
template <typename InT, int MODE, int OUT, int SMK, int VPT, bool kRagged>
dq_status launch_dq_warp(const dq::RowQuantArgs& a, int sms, cudaStream_t stream) {
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  const int grid = static_cast<int>(a.rows < cap ? a.rows : cap);
  return launch_programmatic(dq::dynamic_quant_warp_kernel<InT, MODE, OUT, SMK, VPT, kRagged>, a, grid,
                             dq::kWarpRowThreads, 0, stream);
}

// The warp kernel serves rows of one warp (tpr == 32) when there are at most
// DQ_WARP_KERNEL_MAX_ROWS_PER_SM rows per SM: too few for the ring's per-CTA
// set-up and copy pipeline to pay off.
#ifndef DQ_WARP_KERNEL_MAX_ROWS_PER_SM
#define DQ_WARP_KERNEL_MAX_ROWS_PER_SM 2
#endif

template <typename InT, int MODE, int OUT, int SMK, int VPT>
dq_status launch_dq_ragged(dq::RowQuantArgs a, int device, int sms, cudaStream_t stream) {
  // exact tiling (the row is G * 32 * VPT vectors) needs no per-vector bounds
  // checks; a dense smooth table is staged in shared memory
  const bool exact = (a.cols >> 3) == static_cast<int64_t>(a.tpr) * VPT;
  if (a.tpr == 32 && a.rows <= static_cast<int64_t>(sms) * DQ_WARP_KERNEL_MAX_ROWS_PER_SM) {
    return exact ? launch_dq_warp<InT, MODE, OUT, SMK, VPT, false>(a, sms, stream)
                 : launch_dq_warp<InT, MODE, OUT, SMK, VPT, true>(a, sms, stream);
  }
  const bool staged = SMK != dq::kSmNone && a.group_index == nullptr;
  if (exact) {
    return staged ? launch_dq_ring<InT, MODE, OUT, SMK, VPT, false, SMK != dq::kSmNone>(a, device, sms, stream)
                  : launch_dq_ring<InT, MODE, OUT, SMK, VPT, false, false>(a, device, sms, stream);
  }
  return staged ? launch_dq_ring<InT, MODE, OUT, SMK, VPT, true, SMK != dq::kSmNone>(a, device, sms, stream)
                : launch_dq_ring<InT, MODE, OUT, SMK, VPT, true, false>(a, device, sms, stream);
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
      a.stage_stride = static_cast<uint32_t>((row_bytes + 127) / 128 * 128);
      a.tpr = gs.tpr;
      {
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
