// Dequantization launch selection (AntiQuantize, PER_TOKEN and PER_GROUP):
// the vectorised kernel over work items, or the generic kernel.
#include "dequant_kernels.cuh"
#include "dq_launch.cuh"

namespace dq_host {
namespace {

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

template <int LAYOUT>
dq_status dequant_layout(const dq::DequantArgs& a, int out_kind, bool four, bool has_offset, bool vec,
                         cudaStream_t stream) {
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

}  // namespace

dq_status dequant(const dq::DequantArgs& a, int layout, int out_kind, bool four, bool has_offset, bool vec,
                  cudaStream_t s) {
  switch (layout) {
    case dq::kPerToken: return dequant_layout<dq::kPerToken>(a, out_kind, four, has_offset, vec, s);
    case dq::kGroupAlongRow: return dequant_layout<dq::kGroupAlongRow>(a, out_kind, four, has_offset, vec, s);
    default: return dequant_layout<dq::kGroupDownColumn>(a, out_kind, four, has_offset, vec, s);
  }
}

}  // namespace dq_host
