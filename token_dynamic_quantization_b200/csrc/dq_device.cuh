// Device helpers shared by the sm_100a quantization kernels.
//
// The quantization arithmetic follows the formulas of aclnnDynamicQuantV2
// ("Formula") bit for bit: IEEE binary32, one rounding per operation,
// round-half-to-even. Division by the row scale is the costly part, so it is
// done as a multiply by the correctly rounded reciprocal plus a proof-carrying
// guard band: whenever the product lies too close to a rounding tie for the
// two to be guaranteed to round alike, the element is redone with the true
// IEEE division. The bounds are derived next to each quantizer below.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace dq {

// Element type tags (mirror the dq_dtype values of the C ABI).
enum : int { kF32 = 0, kF16 = 1, kBF16 = 2 };

// ---------------------------------------------------------------- widening

template <typename T>
struct InTraits;

template <>
struct InTraits<__half> {
  // 8 fp16 values (one 16-byte vector) -> 8 floats, exact.
  static __device__ __forceinline__ void widen8(const uint4& raw, float (&v)[8]) {
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ float widen1(const void* p, int64_t i) {
    return __half2float(static_cast<const __half*>(p)[i]);
  }
};

template <>
struct InTraits<__nv_bfloat16> {
  // bf16 is the upper half of a binary32 pattern: a shift/mask widens it.
  static __device__ __forceinline__ void widen8(const uint4& raw, float (&v)[8]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  static __device__ __forceinline__ float widen1(const void* p, int64_t i) {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  }
};

// Runtime-typed scalar load (used for small side tensors: smooth scales,
// AdaLayerNorm parameters), widened to fp32 exactly.
__device__ __forceinline__ float load_param(const void* p, int dtype, int64_t i) {
  if (dtype == kF32) return static_cast<const float*>(p)[i];
  if (dtype == kF16) return __half2float(static_cast<const __half*>(p)[i]);
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

// ---------------------------------------------------------------- reductions

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Barrier over the `nthreads` threads of one row group (named barrier `id`,
// 1..15; id 0 is __syncthreads). nthreads is a multiple of 32.
__device__ __forceinline__ void group_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- quantizers

// Symmetric code of one element: RNE(fl(v / scale)), given rcp = RN(1/scale)
// and a normal, non-zero scale.
//
// Bound: with q = v/scale exact, fl(v/scale) = q(1+d1) and
// t = fl(v * rcp) = q(1+d2)(1+d3), |di| <= u = 2^-24, so
// |t - fl(v/scale)| <= 3.0001 u |q|. Here |v| <= absmax and
// scale >= (absmax/D)(1-u) give |q| <= D(1+2u), D in {127, 7}: the distance is
// at most 3.0001 * 127.0001 * 2^-24 < 2.3e-5 < 2^-15. If t is farther than
// kSymGuard = 2^-14 from every half-integer, fl(v/scale) lies strictly on the
// same side of the same half-integer, so both round to the same integer.
// Otherwise the element is recomputed with the IEEE division.
constexpr float kSymGuard = 6.103515625e-05f;  // 2^-14

// Asymmetric code: RNE(fl(fl(v / scale) + offset)), given rcp = RN(1/scale).
// Fast value t = fl(v * rcp + offset) (one fused rounding).
// Bound: with q = v/scale and w = q + offset exact,
// t = (w + q d2)(1 + d3) and z = fl(fl(q) + offset) = (w + q d1)(1 + d4), so
// |t - z| <= 2u|q| + 2u|w| + O(u^2). Elements lie in [min, max], hence
// w is within [offset_opt - scale_opt, offset_opt] up to rounding noise, so
// |w| <= 129 and |q| <= |offset| + 129; the distance is below
// 2u(|offset| + 260). The guard 4u(|offset| + 260) = 2^-22 (|offset| + 260)
// keeps a factor 2 of margin. Rows whose guard exceeds 1/4 use the IEEE path
// for every element.
__device__ __forceinline__ float asym_half_minus_guard(float offset) {
  const float guard = 2.384185791015625e-07f * (fabsf(offset) + 260.0f);  // 2^-22 (|off|+260)
  return guard > 0.25f ? -1.0f : 0.5f - guard;
}

// Per-row quantization constants.
struct RowQuant {
  float scale;        // written to scale[r]
  float offset;       // asymmetric only
  float rcp;          // RN(1/scale) when the fast path is valid
  float half_minus_guard;  // |t - rint(t)| above this => exact recompute; -1 => always
  bool zero_scale;    // scale == 0: constant codes
};

// symmetric: scale = absmax / D (IEEE division)
__device__ __forceinline__ RowQuant make_sym(float absmax, float divisor) {
  RowQuant q;
  q.scale = __fdiv_rn(absmax, divisor);
  q.offset = 0.0f;
  q.zero_scale = (q.scale == 0.0f);
  // A subnormal scale has too little precision for the bound above.
  const bool fast = q.scale >= 1.17549435e-38f;
  q.rcp = fast ? __frcp_rn(q.scale) : 0.0f;
  q.half_minus_guard = fast ? 0.5f - kSymGuard : -1.0f;
  return q;
}

// asymmetric: scale = (max - min) / scale_opt; offset = offset_opt - max / scale
__device__ __forceinline__ RowQuant make_asym(float mx, float mn, float scale_opt, float offset_opt) {
  RowQuant q;
  q.scale = __fdiv_rn(__fsub_rn(mx, mn), scale_opt);
  q.zero_scale = (q.scale == 0.0f);
  if (q.zero_scale) {
    q.offset = offset_opt;
    q.rcp = 0.0f;
    q.half_minus_guard = -1.0f;
    return q;
  }
  q.offset = __fsub_rn(offset_opt, __fdiv_rn(mx, q.scale));
  const bool fast = q.scale >= 1.17549435e-38f && isfinite(q.offset);
  q.rcp = fast ? __frcp_rn(q.scale) : 0.0f;
  q.half_minus_guard = fast ? asym_half_minus_guard(q.offset) : -1.0f;
  return q;
}

// One symmetric code, rounded integer value as float (in [lo, hi]).
__device__ __forceinline__ float sym_code(float v, const RowQuant& q, float lo, float hi) {
  const float t = __fmul_rn(v, q.rcp);
  const float rt = rintf(t);
  if (fabsf(__fsub_rn(t, rt)) <= q.half_minus_guard) return rt;  // proven equal to the exact path
  const float exact = rintf(__fdiv_rn(v, q.scale));
  return fminf(fmaxf(exact, lo), hi);
}

__device__ __forceinline__ float asym_code(float v, const RowQuant& q, float lo, float hi) {
  const float t = __fmaf_rn(v, q.rcp, q.offset);
  const float rt = rintf(t);
  if (fabsf(__fsub_rn(t, rt)) <= q.half_minus_guard) return fminf(fmaxf(rt, lo), hi);
  const float exact = rintf(__fadd_rn(__fdiv_rn(v, q.scale), q.offset));
  return fminf(fmaxf(exact, lo), hi);
}

// ---------------------------------------------------------------- packing

// 8 int8 codes (as integral floats) -> 8 bytes.
__device__ __forceinline__ uint2 pack_int8x8(const float (&c)[8]) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = static_cast<uint32_t>(__float2int_rn(c[i])) & 0xFFu;
  uint2 r;
  r.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
  r.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
  return r;
}

// 8 int4 codes -> one 32-bit word, element k in bits 4k..4k+3.
__device__ __forceinline__ uint32_t pack_int4x8(const float (&c)[8]) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) w |= (static_cast<uint32_t>(__float2int_rn(c[i])) & 0xFu) << (4 * i);
  return w;
}

}  // namespace dq
