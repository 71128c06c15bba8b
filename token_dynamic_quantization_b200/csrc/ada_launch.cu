// AdaLayerNormQuant launch selection (aclnnAdaLayerNormQuant): the affine
// table kernel, then the bulk-copy row kernel for the row width (or the
// generic kernel), as its programmatic dependent.
#include <cstdlib>

#include "ada_layernorm_quant_kernels.cuh"
#include "dq_launch.cuh"

namespace dq_host {
namespace {

struct GroupShape {
  int vpt;
  int tpr;
};

// Affine-table kernel, launched as a programmatic dependent of the previous
// work; the row kernel follows as its programmatic dependent (it may start
// before the table is finished and waits for it with griddepcontrol.wait).
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

}  // namespace

dq_status ada_bf16(const dq::AdaArgs& a, bool vec, cudaStream_t s) { return launch_ada<__nv_bfloat16>(a, vec, s); }
dq_status ada_f16(const dq::AdaArgs& a, bool vec, cudaStream_t s) { return launch_ada<__half>(a, vec, s); }

}  // namespace dq_host
