// Device helpers shared by the sm_100a quantization kernels.
//
// The quantization arithmetic follows the formulas of aclnnDynamicQuantV2
// ("Formula") bit for bit: IEEE binary32, one rounding per operation,
// round-half-to-even. The division by the row scale uses a two-term
// reciprocal y + y_lo of s (y = RN(1/s); the residual 1 - s*y is exact, and
// y_lo = RN((1 - s*y) * y), as in multiplication by a constant written as a
// sum of two floats: N. Brisebarre, J.-M. Muller, S. K. Raina, IEEE Trans.
// Computers 53(8), 2004). q0 = RN(v*y + RN(v*y_lo)) is then within one ulp of
// v/s, and one correction step of Markstein's method (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990), q = RN(q0 + RN(v - s*q0)*y),
// gives the correctly rounded RN(v/s) whenever nothing underflows. The rows
// that could break that precondition in a way that matters are sent to the
// IEEE division instead (see RowQuant).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "dq_args.cuh"

namespace dq {

// Compile-time flag carried through generic lambdas.
template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};

// ---------------------------------------------------------------- launch overlap

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream is still
// running. launch_dependents lets the next such kernel start early;
// wait_primary blocks until the previous kernel has completed and its memory
// is visible (a no-op for an ordinary launch), so no global memory may be
// touched before it.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- loads

// 16 bytes of data read once: read-only path, not kept in L1.
__device__ __forceinline__ uint4 ld_stream_16(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

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

// Warp-wide max / min of a float in one instruction (sm_100a redux.sync on
// f32). Max and min are exact, so the result does not depend on the order;
// NaN lanes are ignored like fmaxf/fminf do (NaN inputs are outside the
// contract anyway).
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float warp_min(float v) {
  float r;
  asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
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

// ---------------------------------------------------------------- tree reductions

// Three-input max / min (sm_100a). max and min are exact in any order, so the
// row reductions use shallow trees instead of one serial chain.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float min3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// max |v| of 8 values (depth 3)
__device__ __forceinline__ float absmax8(const float (&v)[8]) {
  const float a = fmaxf(fabsf(v[0]), fabsf(v[1])), b = fmaxf(fabsf(v[2]), fabsf(v[3]));
  const float c = fmaxf(fabsf(v[4]), fabsf(v[5])), d = fmaxf(fabsf(v[6]), fabsf(v[7]));
  return fmaxf(fmaxf(a, b), fmaxf(c, d));
}
__device__ __forceinline__ float max8(const float (&v)[8]) {
  return fmaxf(max3(v[0], v[1], v[2]), max3(v[3], v[4], max3(v[5], v[6], v[7])));
}
__device__ __forceinline__ float min8(const float (&v)[8]) {
  return fminf(min3(v[0], v[1], v[2]), min3(v[3], v[4], min3(v[5], v[6], v[7])));
}
// combine N partials with a tree
template <int N, bool kMax>
__device__ __forceinline__ float tree(float (&p)[N]) {
#pragma unroll
  for (int w = 1; w < N; w *= 2) {
#pragma unroll
    for (int i = 0; i + w < N; i += 2 * w) p[i] = kMax ? fmaxf(p[i], p[i + w]) : fminf(p[i], p[i + w]);
  }
  return p[0];
}

// ---------------------------------------------------------------- packed reductions

// Row max / absmax / min on the raw 16-bit values, two per instruction
// (comparisons are exact, so this equals the fp32 reduction of the widened
// values). Used when no smooth scales are applied.
template <typename T>
struct Packed;

template <>
struct Packed<__half> {
  using T2 = __half2;
  static __device__ __forceinline__ T2 from_bits(uint32_t b) { return *reinterpret_cast<const T2*>(&b); }
  static __device__ __forceinline__ T2 lowest() { return from_bits(0xFC00FC00u); }  // -inf, -inf
  static __device__ __forceinline__ T2 highest() { return from_bits(0x7C007C00u); }  // +inf, +inf
  static __device__ __forceinline__ T2 zero() { return from_bits(0u); }
  static __device__ __forceinline__ T2 vmax(T2 a, T2 b) { return __hmax2(a, b); }
  static __device__ __forceinline__ T2 vmin(T2 a, T2 b) { return __hmin2(a, b); }
  static __device__ __forceinline__ float hi_lo_max(T2 a) { return fmaxf(__low2float(a), __high2float(a)); }
  static __device__ __forceinline__ float hi_lo_min(T2 a) { return fminf(__low2float(a), __high2float(a)); }
};

template <>
struct Packed<__nv_bfloat16> {
  using T2 = __nv_bfloat162;
  static __device__ __forceinline__ T2 from_bits(uint32_t b) { return *reinterpret_cast<const T2*>(&b); }
  static __device__ __forceinline__ T2 lowest() { return from_bits(0xFF80FF80u); }
  static __device__ __forceinline__ T2 highest() { return from_bits(0x7F807F80u); }
  static __device__ __forceinline__ T2 zero() { return from_bits(0u); }
  static __device__ __forceinline__ T2 vmax(T2 a, T2 b) { return __hmax2(a, b); }
  static __device__ __forceinline__ T2 vmin(T2 a, T2 b) { return __hmin2(a, b); }
  static __device__ __forceinline__ float hi_lo_max(T2 a) { return fmaxf(__low2float(a), __high2float(a)); }
  static __device__ __forceinline__ float hi_lo_min(T2 a) { return fminf(__low2float(a), __high2float(a)); }
};

// ---------------------------------------------------------------- quantizers

// Per-row quantization constants.
//   exact_row: use the IEEE division for every element of the row. Set when
//     scale is outside [2^-40, 2^100] or the offset is not finite. Otherwise an
//     element whose remainder or v*y_lo can underflow has |v| < 2^-100 or a
//     quotient below 2^-100, hence a quotient below 2^-60 in magnitude: it
//     rounds to code 0 (symmetric), or it cannot move fl(q + offset) across a
//     rounding midpoint that decides a code (asymmetric: a decisive z needs
//     |offset| > 1/4, whose neighbouring midpoints are at least 2^-27 away),
//     so the computed quotient is exact wherever it is used.
//   clamp: saturate before rounding (asymmetric rows with |offset| >= 2^20,
//     where rounding noise of the offset can push the row's extremes past the
//     code range; below 2^20 every code provably lies in range).
struct RowQuant {
  float scale;   // written to scale[r]
  float offset;  // asymmetric only
  float rcp;     // RN(1 / scale) (IEEE reciprocal)
  float rcp_lo;  // RN((1 - scale * rcp) * rcp): 1 / scale ~ rcp + rcp_lo
  bool zero_scale;
  bool exact_row;
  bool clamp;
};

constexpr float kMarksteinMinScale = 0x1p-40f;  // scales outside [2^-40, 2^100] use the IEEE division
constexpr float kMarksteinMaxScale = 0x1p100f;

// The two-term reciprocal of `scale` used by quant8. The residual
// 1 - scale * rcp of a correctly rounded reciprocal is exact in binary32, so
// rcp + rcp_lo carries 1 / scale to about 2^-47 relative.
__device__ __forceinline__ void set_reciprocal(RowQuant& q) {
  q.rcp = __frcp_rn(q.scale);
  q.rcp_lo = __fmul_rn(__fmaf_rn(-q.scale, q.rcp, 1.0f), q.rcp);
}

// RN(v / scale) from the row's two-term reciprocal and one Markstein
// correction (the method of quant8, for one value).
__device__ __forceinline__ float div_split(float v, const RowQuant& q) {
  const float q0 = __fmaf_rn(v, q.rcp, __fmul_rn(v, q.rcp_lo));
  return __fmaf_rn(__fmaf_rn(-q.scale, q0, v), q.rcp, q0);
}

// Two-term reciprocals of the quantizers' constant divisors: y = RN(1/D) and
// lo = RN((1 - D*y) * y), as exact binary32 literals.
template <int D>
struct ConstRecip;
template <>
struct ConstRecip<7> {
  static constexpr float y = 0x1.24924ap-3f, lo = -0x1.b6db7p-28f;
};
template <>
struct ConstRecip<15> {
  static constexpr float y = 0x1.111112p-4f, lo = -0x1.ddddep-29f;
};
template <>
struct ConstRecip<127> {
  static constexpr float y = 0x1.020408p-7f, lo = 0x1.020408p-35f;
};
template <>
struct ConstRecip<255> {
  static constexpr float y = 0x1.010102p-8f, lo = -0x1.fdfep-33f;
};

// RN(a / D) for D in {7, 15, 127, 255} with three FMA-pipe operations and no
// branch: exact for every finite binary32 a (checked exhaustively on the host
// against the IEEE division).
template <int D>
__device__ __forceinline__ float div_const(float a) {
  const float q0 = __fmaf_rn(a, ConstRecip<D>::y, __fmul_rn(a, ConstRecip<D>::lo));
  return __fmaf_rn(__fmaf_rn(-static_cast<float>(D), q0, a), ConstRecip<D>::y, q0);
}

// symmetric: scale = absmax / D
template <int D>
__device__ __forceinline__ RowQuant make_sym(float absmax) {
  RowQuant q;
  q.scale = div_const<D>(absmax);
  q.offset = 0.0f;
  q.zero_scale = (q.scale == 0.0f);
  q.exact_row = !q.zero_scale && !(q.scale >= kMarksteinMinScale && q.scale <= kMarksteinMaxScale);
  q.rcp = 0.0f;
  q.rcp_lo = 0.0f;
  if (!q.zero_scale && !q.exact_row) set_reciprocal(q);
  q.clamp = false;
  return q;
}

// asymmetric: scale = (max - min) / D; offset = OFF - max / scale
template <int D, int OFF>
__device__ __forceinline__ RowQuant make_asym(float mx, float mn) {
  RowQuant q;
  q.scale = div_const<D>(__fsub_rn(mx, mn));
  q.zero_scale = (q.scale == 0.0f);
  q.clamp = false;
  q.rcp = 0.0f;
  q.rcp_lo = 0.0f;
  if (q.zero_scale) {
    q.offset = static_cast<float>(OFF);
    q.exact_row = false;
    return q;
  }
  const bool in_range = q.scale >= kMarksteinMinScale && q.scale <= kMarksteinMaxScale;
  float mq;
  if (in_range) {
    set_reciprocal(q);
    // the split division is exact for |max| >= 2^-100 (and for 0)
    mq = (fabsf(mx) >= 0x1p-100f || mx == 0.0f) ? div_split(mx, q) : __fdiv_rn(mx, q.scale);
  } else {
    mq = __fdiv_rn(mx, q.scale);
  }
  q.offset = __fsub_rn(static_cast<float>(OFF), mq);
  q.exact_row = !in_range || !isfinite(q.offset);
  if (q.exact_row) {
    q.rcp = 0.0f;
    q.rcp_lo = 0.0f;
  }
  q.clamp = !(fabsf(q.offset) < 1048576.0f);  // 2^20
  return q;
}

// ---------------------------------------------------------------- rounding

// Adding 1.5 * 2^23 to a binary32 t with |t| < 2^22 lands in [2^23, 2^24),
// where the spacing is exactly 1, so the RN sum is M + RNE(t) (M is even, so
// ties still go to even). Subtracting M back is exact. The low bits of the
// sum's pattern hold RNE(t) in two's complement (0x4B400000 + RNE(t)), so a
// code's byte or nibble can be taken from the pattern directly. This keeps
// the rounding on the FMA pipe instead of the conversion unit.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// Codes of 8 elements (magic-sum patterns, see kRoundMagic) on a row whose
// RowQuant has neither zero_scale nor exact_row set:
//   q = RN(v / scale) from the two-term reciprocal and one Markstein
//   correction (4 FMA-pipe operations per element pair),
//   z = RN(q + offset) (asymmetric), optional saturation, then RNE via the
//   magic add. Branch-free; every element gets the formulas' exact result.
template <bool kAsym, bool kClamp>
__device__ __forceinline__ void quant8(const float (&v)[8], const RowQuant& q, float lo, float hi,
                                       uint32_t (&bits)[8]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 vv = make_float2(v[2 * p], v[2 * p + 1]);
    const float2 q0 = __ffma2_rn(vv, f2(q.rcp), __fmul2_rn(vv, f2(q.rcp_lo)));  // faithful v / scale
    const float2 r0 = __ffma2_rn(f2(-q.scale), q0, vv);                         // exact remainder
    float2 z = __ffma2_rn(r0, f2(q.rcp), q0);                                    // RN(v / scale)
    if (kAsym) z = __fadd2_rn(z, f2(q.offset));
    if (kClamp) {
      z.x = fminf(fmaxf(z.x, lo), hi);
      z.y = fminf(fmaxf(z.y, lo), hi);
    }
    const float2 sum = __fadd2_rn(z, f2(kRoundMagic));
    bits[2 * p] = __float_as_uint(sum.x);
    bits[2 * p + 1] = __float_as_uint(sum.y);
  }
}

// The formulas' own arithmetic for 8 elements with the IEEE division (then
// + offset), RNE and saturation to [lo, hi]: the path of exact_row rows.
template <bool kAsym>
__device__ __forceinline__ void quant8_exact(const float (&v)[8], const RowQuant& q, float lo, float hi,
                                          uint32_t (&bits)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float z = __fdiv_rn(v[j], q.scale);
    if (kAsym) z = __fadd_rn(z, q.offset);
    z = fminf(fmaxf(rintf(z), lo), hi);
    bits[j] = __float_as_uint(__fadd_rn(z, kRoundMagic));
  }
}

// Scalar version (generic kernels): the code as an int.
template <bool kAsym>
__device__ __forceinline__ int code_exact(float v, const RowQuant& q, float lo, float hi) {
  float z = __fdiv_rn(v, q.scale);
  if (kAsym) z = __fadd_rn(z, q.offset);
  return __float2int_rn(fminf(fmaxf(rintf(z), lo), hi));
}

// ---------------------------------------------------------------- packing

// 8 codes (low bytes of the patterns) -> 8 int8 bytes.
__device__ __forceinline__ uint2 pack8_int8(const uint32_t (&b)[8]) {
  uint2 r;
  r.x = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  r.y = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
  return r;
}

// 8 codes (low nibbles of the patterns) -> one word, element k in bits 4k..4k+3.
__device__ __forceinline__ uint32_t pack8_int4(const uint32_t (&b)[8]) {
  const uint2 bytes = pack8_int8(b);
  uint32_t lo = bytes.x & 0x0F0F0F0Fu;
  uint32_t hi = bytes.y & 0x0F0F0F0Fu;
  lo |= lo >> 4;  // byte0 = c0 | c1 << 4, byte2 = c2 | c3 << 4
  hi |= hi >> 4;
  return __byte_perm(lo, hi, 0x6420);
}

}  // namespace dq
