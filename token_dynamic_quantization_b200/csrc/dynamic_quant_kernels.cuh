// Per-token dynamic quantization (aclnnDynamicQuantV2, "Formula" and
// "Description"), sm_100a: the pieces the kernels share (quantization
// constants, the MoE expert lookup and status word, smooth-scale loads) and
// the generic kernel, which takes any column count or alignment: one CTA per
// row (grid-strided), two passes over the row (the second one mostly hits L2).
// The vectorised kernels (the ring kernel for most shapes, one warp per row
// for few short rows) are in dynamic_quant_ring.cuh.
#pragma once

#include "dq_args.cuh"
#include "dq_device.cuh"
#include "tma_pipeline.cuh"

namespace dq {

template <int MODE, int OUT>
struct QuantConsts {
  static constexpr bool kFour = OUT == kOutInt4;
  static constexpr int kDivisor = MODE == kSym ? (kFour ? 7 : 127) : (kFour ? 15 : 255);
  static constexpr int kOffsetOptInt = MODE == kSym ? 0 : (kFour ? 7 : 127);
  static constexpr float kOffsetOpt = static_cast<float>(kOffsetOptInt);
  static constexpr float kLo = MODE == kSym ? (kFour ? -7.0f : -127.0f) : (kFour ? -8.0f : -128.0f);
  static constexpr float kHi = kFour ? 7.0f : 127.0f;
};

// Status word of a MoE call: written by exactly one thread per launch, so it
// needs no clearing between calls.
__device__ __forceinline__ void write_group_status(const RowQuantArgs& a) {
  if (a.group_index == nullptr || blockIdx.x != 0 || threadIdx.x != 0) return;
  uint32_t flags = 0;
  int32_t prev = 0;
  for (int e = 0; e < a.num_groups; ++e) {
    const int32_t g = a.group_index[e];
    if (g < prev) flags |= 0x2u;
    prev = g > prev ? g : prev;
  }
  if (a.rows > static_cast<int64_t>(a.group_index[a.num_groups - 1])) flags |= 0x1u;
  *a.status = flags;
}

// expert(r): smallest e with r < gi[e]; num_groups if none.
__device__ __forceinline__ int expert_of(const int32_t* gi, int n, int64_t r) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (r < static_cast<int64_t>(gi[mid])) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// ============================================================ shared pieces

// Smooth-scale storage kinds (template parameter of the vectorised kernels).
enum : int { kSmNone = 0, kSmF32 = 1, kSmF16 = 2, kSmBF16 = 3 };

// Smooth scales of one 8-column vector of `row` (16-byte aligned), widened to
// fp32. The table is small and shared by every row, so it is read through L1.
template <int SMK>
__device__ __forceinline__ void load_smooth8(const void* row, int vi, float (&s)[8]) {
  if (SMK == kSmF32) {
    const float4* p = static_cast<const float4*>(row) + 2 * vi;
    const float4 a = __ldg(p), b = __ldg(p + 1);
    s[0] = a.x; s[1] = a.y; s[2] = a.z; s[3] = a.w;
    s[4] = b.x; s[5] = b.y; s[6] = b.z; s[7] = b.w;
  } else if (SMK == kSmBF16) {
    InTraits<__nv_bfloat16>::widen8(__ldg(static_cast<const uint4*>(row) + vi), s);
  } else if (SMK == kSmF16) {
    InTraits<__half>::widen8(__ldg(static_cast<const uint4*>(row) + vi), s);
  }
}

// input = x (* smooth) for one 8-element vector held in `raw`.
template <typename InT, int SMK>
__device__ __forceinline__ void input8(const uint4& raw, const void* smooth_row, int vi, float (&v)[8]) {
  InTraits<InT>::widen8(raw, v);
  if (SMK != kSmNone) {
    float sm[8];
    load_smooth8<SMK>(smooth_row, vi, sm);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float2 pr = __fmul2_rn(make_float2(v[2 * p], v[2 * p + 1]), make_float2(sm[2 * p], sm[2 * p + 1]));
      v[2 * p] = pr.x;
      v[2 * p + 1] = pr.y;
    }
  }
}

// ============================================================ generic kernel

constexpr int kGenericBlock = 256;

template <typename InT, int MODE, int OUT>
__global__ void __launch_bounds__(kGenericBlock)
dynamic_quant_generic_kernel(const RowQuantArgs a) {
  using C = QuantConsts<MODE, OUT>;
  constexpr bool kA = MODE == kAsym;
  __shared__ float red[kGenericBlock / 32][2];
  write_group_status(a);
  const bool moe = a.group_index != nullptr;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  constexpr int kWarps = kGenericBlock / 32;

  for (int64_t r = blockIdx.x; r < a.rows; r += gridDim.x) {
    int64_t srow = 0;
    bool row_valid = true;
    if (moe) {
      const int e = expert_of(a.group_index, a.num_groups, r);
      row_valid = e < a.num_groups;
      srow = e;
    }
    const int64_t base = r * a.cols;
    auto input = [&](int64_t c) {
      float v = InTraits<InT>::widen1(a.x, base + c);
      if (a.smooth != nullptr) v = __fmul_rn(v, load_param(a.smooth, a.smooth_dtype, srow * a.cols + c));
      return v;
    };
    float m0 = kA ? -INFINITY : 0.0f;
    float m1 = INFINITY;
    if (row_valid) {
      for (int64_t c = threadIdx.x; c < a.cols; c += kGenericBlock) {
        const float v = input(c);
        if (kA) {
          m0 = fmaxf(m0, v);
          m1 = fminf(m1, v);
        } else {
          m0 = fmaxf(m0, fabsf(v));
        }
      }
    }
    m0 = warp_max(m0);
    if (kA) m1 = warp_min(m1);
    if (lane == 0) {
      red[warp][0] = m0;
      red[warp][1] = m1;
    }
    __syncthreads();
    m0 = red[0][0];
    m1 = red[0][1];
    for (int w = 1; w < kWarps; ++w) {
      m0 = fmaxf(m0, red[w][0]);
      if (kA) m1 = fminf(m1, red[w][1]);
    }
    __syncthreads();  // red[] is rewritten by the next row

    RowQuant q = kA ? make_asym<C::kDivisor, C::kOffsetOptInt>(m0, m1) : make_sym<C::kDivisor>(m0);
    if (!row_valid) {
      q.scale = 0.0f;
      q.offset = 0.0f;
    }
    if (threadIdx.x == 0) {
      a.scale[r] = q.scale;
      if (kA) a.offset[r] = q.offset;
    }
    auto code = [&](int64_t c) -> int {
      if (!row_valid) return 0;
      if (q.zero_scale) return static_cast<int>(C::kOffsetOpt);
      return code_exact<kA>(input(c), q, C::kLo, C::kHi);
    };
    if (OUT == kOutInt8) {
      int8_t* yr = static_cast<int8_t*>(a.y) + base;
      for (int64_t c = threadIdx.x; c < a.cols; c += kGenericBlock) yr[c] = static_cast<int8_t>(code(c));
    } else {
      uint8_t* yr = static_cast<uint8_t*>(a.y) + (base >> 1);
      for (int64_t j = threadIdx.x; j < (a.cols >> 1); j += kGenericBlock) {
        const uint32_t lo = static_cast<uint32_t>(code(2 * j)) & 0xFu;
        const uint32_t hi = static_cast<uint32_t>(code(2 * j + 1)) & 0xFu;
        yr[j] = static_cast<uint8_t>(lo | (hi << 4));
      }
    }
  }
}

}  // namespace dq
