// AdaLayerNormQuant launch selection (aclnnAdaLayerNormQuant): the bulk-copy
// ring kernel for the row width, which folds its batches' affine table rows
// itself when they fit in shared memory; otherwise the affine table kernel,
// then the ring kernel (or the generic kernel) as its programmatic dependent.
#include <cstdlib>

#include "ada_layernorm_quant_kernels.cuh"
#include "ada_layernorm_quant_ring.cuh"
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

// Largest dynamic shared memory of one CTA on sm_100 (227 KB), less the
// ring kernel's static shared memory and a reserve; the part of it the staged
// affine table may take.
constexpr size_t kAdaRingSmemBudget = 232448 - 2048;
#ifndef DQ_ADA_TABLE_BUDGET
#define DQ_ADA_TABLE_BUDGET (64 * 1024)
#endif
#ifndef DQ_ADA_RING_MAX_SLOTS
#define DQ_ADA_RING_MAX_SLOTS 32
#endif
// Bytes of row slots per CTA (hidden 3072, 16 one-warp groups: 16 slots of
// 6 KB 38.6 us, 20 slots 38.9 us, 29 slots 41.8 us).
#ifndef DQ_ADA_RING_BYTES
#define DQ_ADA_RING_BYTES (100 * 1024)
#endif

// Ring kernel launch: one CTA per SM (fewer for few rows), NC row groups of G
// warps (as many as the kernel's largest block holds, at most 15 with G > 1), the
// table rows of the CTA's batches staged when they fit DQ_ADA_TABLE_BUDGET,
// NS row slots of about DQ_ADA_RING_BYTES in all.
template <typename InT, int VPT, bool kRagged, bool kStaged>
dq_status launch_ada_ring(dq::AdaArgs a, int device, int sms, int64_t table_batches, cudaStream_t stream) {
  void (*kfn)(const dq::AdaArgs) = dq::ada_layernorm_quant_ring_kernel<InT, VPT, kRagged, kStaged>;
  const void* k = reinterpret_cast<const void*>(kfn);
  if (!allow_smem_bytes(k, device, kAdaRingSmemBudget)) return kNotLaunchable;
  const int max_threads = kernel_max_threads(k, device);
  const int G = a.tpr / 32;
  const int64_t rows = a.batch * a.seq;
  const int64_t grid = rows < sms ? rows : sms;
  const int64_t per_cta = (rows + grid - 1) / grid;
  int64_t nc = max_threads / a.tpr;
  if (G > 1 && nc > 15) nc = 15;
  if (nc > per_cta) nc = per_cta;
  a.table_batches = kStaged ? static_cast<int>(table_batches) : 0;
  const size_t fixed = dq::ada_ring_smem_bytes(0, a.stage_stride, a.table_batches, a.hidden);
  if (fixed >= kAdaRingSmemBudget) return kNotLaunchable;
  const int64_t ns_fit = static_cast<int64_t>((kAdaRingSmemBudget - fixed) / (a.stage_stride + 16));
  int64_t ns = DQ_ADA_RING_BYTES / a.stage_stride;
  if (ns < nc) ns = nc;  // at least one slot per group
  if (ns > ns_fit) ns = ns_fit;
  if (ns > DQ_ADA_RING_MAX_SLOTS) ns = DQ_ADA_RING_MAX_SLOTS;
  if (ns > per_cta) ns = per_cta;
  if (nc > ns) nc = ns;
  if (nc < 1) return kNotLaunchable;
  a.groups = static_cast<int>(nc);
  a.stages = static_cast<int>(ns);
  const size_t smem = dq::ada_ring_smem_bytes(a.stages, a.stage_stride, a.table_batches, a.hidden);
  const int block = a.tpr * a.groups;
  if (blocks_per_sm(k, block, smem, device) < 1) return kNotLaunchable;
  if (!kStaged) {
    // the ring kernel reads the table through L1: the table kernel writes it
    const dq_status st = launch_ada_table(a, sms, stream);
    if (st != DQ_OK) return st;
  }
  return launch_programmatic(kfn, a, static_cast<int>(grid), block, smem, stream);
}

template <typename InT, int VPT>
dq_status launch_ada_ragged(dq::AdaArgs a, int device, int sms, cudaStream_t stream) {
  // exact tiling (the row is G * 32 * VPT vectors) needs no per-vector bounds
  // checks; the table rows of a CTA's batches are staged when they fit
  const bool exact = (a.hidden >> 3) == static_cast<int64_t>(a.tpr) * VPT;
  const int64_t rows = a.batch * a.seq;
  const int64_t grid = rows < sms ? rows : sms;
  const int64_t per_cta = (rows + grid - 1) / grid;
  int64_t nb = (per_cta - 1) / a.seq + 2;  // batches a range of per_cta rows can touch
  if (nb > a.batch) nb = a.batch;
  const bool staged = static_cast<size_t>(nb) * static_cast<size_t>(a.hidden) * 8 <= DQ_ADA_TABLE_BUDGET;
  if (exact) {
    return staged ? launch_ada_ring<InT, VPT, false, true>(a, device, sms, nb, stream)
                  : launch_ada_ring<InT, VPT, false, false>(a, device, sms, nb, stream);
  }
  return staged ? launch_ada_ring<InT, VPT, true, true>(a, device, sms, nb, stream)
                : launch_ada_ring<InT, VPT, true, false>(a, device, sms, nb, stream);
}

// AdaLayerNorm row-group shape: VPT in {2, 3, 4, 6, 8, 12}, fewest wasted
// lanes, then the fewest warps per row. The per-row work (three row
// reductions, the row statistics and constants) is repeated by every warp of
// a row, and one warp per row needs no cross-warp combine: hidden 3072 runs
// one warp of 12 vectors per lane.
GroupShape pick_ada_shape(int64_t nvec) {
  GroupShape best{0, 0};
  double best_eff = -1.0;
  static const int kVpts[6] = {2, 3, 4, 6, 8, 12};
  for (int vpt : kVpts) {
    const int64_t warps = (nvec + 32 * vpt - 1) / (32 * vpt);
    if (warps > 16) continue;
    const int64_t tpr = warps * 32;
    const double eff = static_cast<double>(nvec) / static_cast<double>(tpr * vpt);
    const bool better = eff > best_eff + 1e-9 || (eff > best_eff - 1e-9 && tpr <= best.tpr);
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
      a.stage_stride = static_cast<uint32_t>((a.hidden * 2 + 127) / 128 * 128);
      a.tpr = gs.tpr;
      {
        dq_status st;
        switch (gs.vpt) {
          case 2: st = launch_ada_ragged<InT, 2>(a, device, sms, stream); break;
          case 3: st = launch_ada_ragged<InT, 3>(a, device, sms, stream); break;
          case 4: st = launch_ada_ragged<InT, 4>(a, device, sms, stream); break;
          case 6: st = launch_ada_ragged<InT, 6>(a, device, sms, stream); break;
          case 8: st = launch_ada_ragged<InT, 8>(a, device, sms, stream); break;
          default: st = launch_ada_ragged<InT, 12>(a, device, sms, stream); break;
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
