// Fused AdaLayerNorm + symmetric INT8 dynamic quantization
// (aclnnAdaLayerNormQuant, "Formula" steps 1-5), sm_100a.
//
// The per-(batch, column) parameters of steps 1-3 fold into a table
//     A[b][c] = (w[c] * (1 + scale[b][c])) * smooth[c]
//     B[b][c] = ((bias[c] * (1 + scale[b][c])) + shift[b][c]) * smooth[c]
// (absent weight = 1, bias = 0, smooth = 1), so steps 1-3 become one FMA per
// element, y = n * A + B (ada_fold_values, the one evaluation of these formulas).
//   * The ring kernel (ada_layernorm_quant_ring.cuh) with the table staged in
//     shared memory folds the table rows of its batches itself: one launch
//     per call.
//   * Otherwise two launches: ada_affine_table_kernel writes the table
//     (batch x hidden x 8 bytes) into the caller's workspace, then the row
//     kernel, a programmatic dependent of it (the ring kernel reading the
//     table through L1, or ada_layernorm_quant_generic_kernel below). The
//     table kernel is itself a programmatic dependent of the work before it
//     and releases the row kernel only after that work has completed, so the
//     row kernel may start copying rows of x before it waits for the table.
//
// Arithmetic of the ring kernel:
//   * E(x), Var(x) from one row reduction: each thread sums d = x - K and d^2
//     over its share, with K the mean of the row's first 4 elements (the same
//     value in every thread; d is exact when x and K are within a factor 2,
//     as on rows whose mean is far above their spread). Partial sums are fp32,
//     the sums across warps double; E(x) = K + E(d), Var = E(d^2) - E(d)^2.
//     While E(d)^2 <= 3/4 E(d^2) that difference loses at most a factor 4 of
//     relative accuracy. Rows past the bound (first elements far from the
//     mean) take a centred second pass about RN(E(x)). E(x) is rounded to
//     fp32 once, as the formula's mean is.
//   * n = (x - E(x)) * rstd with rstd = RN(1 / sqrt(Var + eps)), as
//     fma(d, rstd, -(E(x) - K) * rstd), then y = n * A + B. Against a
//     sequential evaluation that rounds every printed operation separately
//     and divides by the square root, this moves y by a few ulps:
//     quant_scale stays within a relative 1e-6 and about one code in 10^6
//     moves by one.
//   * steps 4-5 are the DynamicQuant quantizer (exact IEEE semantics).
#pragma once

#include <type_traits>

#include "dq_args.cuh"
#include "dq_device.cuh"
#include "tma_pipeline.cuh"

namespace dq {

// ============================================================ affine table

constexpr int kTableBlock = 256;

// A[b][c], B[b][c] of the folded table (ParamT: the parameters' type).
template <typename ParamT>
__device__ __forceinline__ float param_at(const void* p, int64_t i) {
  if constexpr (sizeof(ParamT) == 4) {
    return __ldg(static_cast<const float*>(p) + i);
  } else if constexpr (std::is_same<ParamT, __half>::value) {
    return __half2float(__ldg(static_cast<const __half*>(p) + i));
  } else {
    return __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(p) + i));
  }
}
// A, B of one column from its parameter values: the batch's scale and shift,
// the column's weight, bias and smooth scale (1, 0 and 1 when absent)
__device__ __forceinline__ void ada_fold_values(float scale, float shift, float w, float bs, float sm, float& A,
                                                float& B) {
  const float onep = __fadd_rn(1.0f, scale);
  A = __fmul_rn(__fmul_rn(w, onep), sm);
  B = __fmul_rn(__fadd_rn(__fmul_rn(bs, onep), shift), sm);
}
template <typename ParamT>
__device__ __forceinline__ void ada_fold(const AdaArgs& a, int64_t b, int64_t c, float& A, float& B) {
  const int64_t idx = b * a.hidden + c;
  ada_fold_values(param_at<ParamT>(a.ada_scale, idx), param_at<ParamT>(a.ada_shift, idx),
                  a.weight ? param_at<ParamT>(a.weight, c) : 1.0f, a.bias ? param_at<ParamT>(a.bias, c) : 0.0f,
                  a.smooth ? param_at<ParamT>(a.smooth, c) : 1.0f, A, B);
}

__global__ void __launch_bounds__(kTableBlock) ada_affine_table_kernel(const AdaArgs a) {
  // launched as a programmatic dependent of the previous work in the stream:
  // wait for it, then let the row kernel start (it copies rows of x before
  // its own wait, which is safe once the work before this kernel is done)
  pdl_wait_primary();
  pdl_launch_dependents();
  const int64_t H = a.hidden;
  const int64_t total = a.batch * H;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = idx / H, c = idx - (idx / H) * H;
    float A, B;
    if (a.param_dtype == kF32) {
      ada_fold<float>(a, b, c, A, B);
    } else if (a.param_dtype == kF16) {
      ada_fold<__half>(a, b, c, A, B);
    } else {
      ada_fold<__nv_bfloat16>(a, b, c, A, B);
    }
    a.table[idx] = A;
    a.table[total + idx] = B;
  }
}

// ============================================================ generic kernel

constexpr int kAdaGenericBlock = 256;

template <typename InT>
__global__ void __launch_bounds__(kAdaGenericBlock)
ada_layernorm_quant_generic_kernel(const AdaArgs a) {
  __shared__ double red_d[kAdaGenericBlock / 32];
  __shared__ float red_f[kAdaGenericBlock / 32];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  constexpr int kWarps = kAdaGenericBlock / 32;
  const int64_t rows = a.batch * a.seq;
  const int64_t H = a.hidden;
  const float* At = a.table;
  const float* Bt = a.table + a.batch * H;

  auto block_sum = [&](double v) {
    v = warp_sum(v);
    if (lane == 0) red_d[warp] = v;
    __syncthreads();
    double s = 0.0;
    for (int i = 0; i < kWarps; ++i) s += red_d[i];
    __syncthreads();
    return s;
  };

  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int64_t b = r / a.seq;
    const int64_t base = r * H;
    double s1 = 0.0;
    for (int64_t c = threadIdx.x; c < H; c += kAdaGenericBlock) s1 += InTraits<InT>::widen1(a.x, base + c);
    const double mean_d = block_sum(s1) * a.inv_hidden;
    const float mean_f = __double2float_rn(mean_d);
    double s2 = 0.0;
    for (int64_t c = threadIdx.x; c < H; c += kAdaGenericBlock) {
      const double dd = static_cast<double>(InTraits<InT>::widen1(a.x, base + c)) - mean_d;
      s2 += dd * dd;
    }
    const float var_f = __double2float_rn(block_sum(s2) * a.inv_hidden);
    const float rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(var_f, a.epsilon)));

    auto value = [&](int64_t c) {
      const float nn = __fmul_rn(__fsub_rn(InTraits<InT>::widen1(a.x, base + c), mean_f), rstd);
      return __fmaf_rn(nn, At[b * H + c], Bt[b * H + c]);
    };
    float amax = 0.0f;
    for (int64_t c = threadIdx.x; c < H; c += kAdaGenericBlock) amax = fmaxf(amax, fabsf(value(c)));
    amax = warp_max(amax);
    if (lane == 0) red_f[warp] = amax;
    __syncthreads();
    amax = red_f[0];
    for (int i = 1; i < kWarps; ++i) amax = fmaxf(amax, red_f[i]);
    __syncthreads();
    const RowQuant q = make_sym<127>(amax);
    if (threadIdx.x == 0) a.quant_scale[r] = q.scale;
    for (int64_t c = threadIdx.x; c < H; c += kAdaGenericBlock) {
      a.out[base + c] = static_cast<int8_t>(q.zero_scale ? 0 : code_exact<false>(value(c), q, -127.0f, 127.0f));
    }
  }
}

}  // namespace dq
