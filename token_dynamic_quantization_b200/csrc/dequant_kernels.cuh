// Dequantization (AntiQuantize, PER_TOKEN and PER_GROUP policies), sm_100a.
//
// One scale and one optional offset per row of an [m, n] code matrix
// (PER_TOKEN), or per group of groupSize elements along a row or down a
// column (PER_GROUP). The page's formula images were lost; the operation is
// the inverse of the aclnnDynamicQuantV2 quantizer (codes = round(x / scale +
// offset)):
//   out[i,j] = (code[i,j] - offset[e]) * scale[e]   (e: the element's table entry)
// in binary32, one rounding per operation, then rounded to nearest even into
// the output type.
//
// The work is 1 (int8) or 0.5 (int4) byte in and 2 or 4 bytes out per element,
// so the kernel is HBM-bound. A warp takes one chunk of a row at a time; each
// lane streams 16-byte vectors of codes (16 int8 or 32 int4 codes).
// A code becomes a float without the conversion unit: XOR with the sign bit
// makes it an unsigned byte u = code + 128 (u = code + 8 for nibbles), a byte
// permute places u in the low byte of the pattern of 1.5 * 2^23, and one
// subtraction of 1.5 * 2^23 + 128 (or + 8) leaves the code exactly. Then
// (v - offset) * scale as packed f32x2 operations and one packed conversion
// (cvt.rn.{bf16x2,f16x2}.f32) per pair of outputs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "dq_args.cuh"
#include "dq_device.cuh"

namespace dq {

// Output element storage and pair narrowing (round to nearest even).
template <int OUT>
struct OutTraits;
template <>
struct OutTraits<kOutF32> {
  static constexpr int kBytes = 4;
};
template <>
struct OutTraits<kOutF16> {
  static constexpr int kBytes = 2;
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  static __device__ __forceinline__ void store1(void* p, int64_t i, float v) {
    static_cast<__half*>(p)[i] = __float2half_rn(v);
  }
};
template <>
struct OutTraits<kOutBF16> {
  static constexpr int kBytes = 2;
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  static __device__ __forceinline__ void store1(void* p, int64_t i, float v) {
    static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  }
};

// 1.5 * 2^23 + bias as a binary32 value: the pattern 0x4B400000 | u reads as
// 1.5 * 2^23 + u, so subtracting this gives u - bias exactly.
constexpr float kCodeMagic8 = 12583040.0f;  // 1.5 * 2^23 + 128
constexpr float kCodeMagic4 = 12582920.0f;  // 1.5 * 2^23 + 8

// Value of byte j (0..3) of `u` placed in the low byte of 1.5 * 2^23's pattern.
__device__ __forceinline__ float byte_as_float(uint32_t u, int j, float magic) {
  return __uint_as_float(__byte_perm(u, 0x4B400000u, 0x7650u | static_cast<uint32_t>(j))) - magic;
}

// The 16 (int8) or 32 (int4) codes of one 16-byte vector as floats, in element order.
template <bool kFour>
__device__ __forceinline__ void codes_of(const uint4& w, float (&v)[kFour ? 32 : 16]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (!kFour) {
      const uint32_t u = ws[i] ^ 0x80808080u;  // signed byte -> code + 128
#pragma unroll
      for (int j = 0; j < 4; ++j) v[4 * i + j] = byte_as_float(u, j, kCodeMagic8);
    } else {
      const uint32_t u = ws[i] ^ 0x88888888u;  // signed nibble -> code + 8
      const uint32_t lo = u & 0x0F0F0F0Fu;        // elements 8i + 0, 2, 4, 6
      const uint32_t hi = (u >> 4) & 0x0F0F0F0Fu;  // elements 8i + 1, 3, 5, 7
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * i + 2 * j] = byte_as_float(lo, j, kCodeMagic4);
        v[8 * i + 2 * j + 1] = byte_as_float(hi, j, kCodeMagic4);
      }
    }
  }
}

// (v - offset) * scale over the vector, as packed pairs.
template <int N, bool kOff>
__device__ __forceinline__ void apply_row_constants(float (&v)[N], float scale, float offset) {
#pragma unroll
  for (int p = 0; p < N / 2; ++p) {
    float2 t = make_float2(v[2 * p], v[2 * p + 1]);
    if (kOff) t = __fadd2_rn(t, f2(-offset));
    t = __fmul2_rn(t, f2(scale));
    v[2 * p] = t.x;
    v[2 * p + 1] = t.y;
  }
}

// (v - offset[e]) * scale[e] with per-element tables.
template <int N, bool kOff>
__device__ __forceinline__ void apply_element_constants(float (&v)[N], const float (&scale)[N], const float (&off)[N]) {
#pragma unroll
  for (int p = 0; p < N / 2; ++p) {
    float2 t = make_float2(v[2 * p], v[2 * p + 1]);
    if (kOff) t = __fadd2_rn(t, make_float2(-off[2 * p], -off[2 * p + 1]));
    t = __fmul2_rn(t, make_float2(scale[2 * p], scale[2 * p + 1]));
    v[2 * p] = t.x;
    v[2 * p + 1] = t.y;
  }
}

// N consecutive table values from element `first` (16-byte aligned), widened.
template <int N>
__device__ __forceinline__ void load_table(const void* table, int dtype, int64_t first, float (&t)[N]) {
  if (dtype == kF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(table) + first);
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
      const float4 f = __ldg(p + q);
      t[4 * q] = f.x;
      t[4 * q + 1] = f.y;
      t[4 * q + 2] = f.z;
      t[4 * q + 3] = f.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(table) + first);
#pragma unroll
    for (int q = 0; q < N / 8; ++q) {
      float h[8];
      if (dtype == kF16) {
        InTraits<__half>::widen8(__ldg(p + q), h);
      } else {
        InTraits<__nv_bfloat16>::widen8(__ldg(p + q), h);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) t[8 * q + e] = h[e];
    }
  }
}

template <int OUT, int N>
__device__ __forceinline__ void store_vector(void* out_row, int vi, const float (&v)[N]) {
  if constexpr (OUT == kOutF32) {
    float4* o = reinterpret_cast<float4*>(out_row) + static_cast<int64_t>(vi) * (N / 4);
#pragma unroll
    for (int q = 0; q < N / 4; ++q) __stcs(o + q, make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]));
  } else {
    uint4* o = reinterpret_cast<uint4*>(out_row) + static_cast<int64_t>(vi) * (N / 8);
#pragma unroll
    for (int q = 0; q < N / 8; ++q) {
      uint4 w;
      w.x = OutTraits<OUT>::pack(v[8 * q + 0], v[8 * q + 1]);
      w.y = OutTraits<OUT>::pack(v[8 * q + 2], v[8 * q + 3]);
      w.z = OutTraits<OUT>::pack(v[8 * q + 4], v[8 * q + 5]);
      w.w = OutTraits<OUT>::pack(v[8 * q + 6], v[8 * q + 7]);
      __stcs(o + q, w);
    }
  }
}

constexpr int kDequantBlock = 256;
// 16-byte code vectors per lane and work item, per scale layout (measured:
// per-token rows stream best with one vector per lane and item, grouped
// tables with two, which amortize the table lookups).
#ifndef DQ_DEQUANT_UNROLL_TOKEN
#define DQ_DEQUANT_UNROLL_TOKEN 1
#endif
#ifndef DQ_DEQUANT_UNROLL_GROUP
#define DQ_DEQUANT_UNROLL_GROUP 2
#endif
template <int LAYOUT>
__host__ __device__ constexpr int dequant_unroll() {
  return LAYOUT == kPerToken ? DQ_DEQUANT_UNROLL_TOKEN : DQ_DEQUANT_UNROLL_GROUP;
}

// Rows whose code bytes are a whole number of 16-byte vectors, 16-byte
// aligned codes and output rows. A work item is one chunk of a row: 32 lanes
// x dequant_unroll vectors (512 or 1024 int8 codes). Items are many
// and small, and the grid covers them all (a grid-stride loop only beyond
// the grid limit), so the block scheduler balances the tail.
template <int OUT, bool kFour, bool kOff, int LAYOUT>
__global__ void __launch_bounds__(kDequantBlock) dequant_vec_kernel(const DequantArgs a) {
  constexpr int N = kFour ? 32 : 16;  // codes per 16-byte vector
  constexpr int kWarps = kDequantBlock / 32;
  constexpr int kDequantUnroll = dequant_unroll<LAYOUT>();
  pdl_launch_dependents();
  pdl_wait_primary();  // launched as a programmatic dependent: inputs are visible from here on
  const int lane = threadIdx.x & 31;
  const int nvec = static_cast<int>(a.cols / N);
  const int64_t chunks = (nvec + 32 * kDequantUnroll - 1) / (32 * kDequantUnroll);  // per row
  const int64_t items = a.rows * chunks;
  const int64_t row_code_bytes = kFour ? a.cols / 2 : a.cols;
  const int64_t row_out_bytes = a.cols * OutTraits<OUT>::kBytes;
  for (int64_t item = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); item < items;
       item += static_cast<int64_t>(gridDim.x) * kWarps) {
    const int64_t r = item / chunks;
    const int v0 = static_cast<int>(item - r * chunks) * (32 * kDequantUnroll) + lane;
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.y) + r * row_code_bytes);
    void* dst = static_cast<uint8_t*>(a.out) + r * row_out_bytes;
    uint4 w[kDequantUnroll];
#pragma unroll
    for (int u = 0; u < kDequantUnroll; ++u) {
      const int vi = v0 + 32 * u;
      w[u] = vi < nvec ? __ldcs(src + vi) : make_uint4(0, 0, 0, 0);
    }
    // the row's constants after the code loads are in flight (measured:
    // loading them first delays the stream)
    float scale = 0.0f, offset = 0.0f;
    if (LAYOUT == kPerToken) {
      scale = load_param(a.scale, a.scale_dtype, r);
      offset = kOff ? load_param(a.offset, a.scale_dtype, r) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kDequantUnroll; ++u) {
      const int vi = v0 + 32 * u;
      if (vi < nvec) {
        float v[N];
        codes_of<kFour>(w[u], v);
        if (LAYOUT == kPerToken) {
          apply_row_constants<N, kOff>(v, scale, offset);
        } else if (LAYOUT == kGroupAlongRow) {
          // a vector lies inside one group (the group size is a multiple of 32)
          const int64_t entry = r * a.table_cols + static_cast<int64_t>(vi) * N / a.group_size;
          apply_row_constants<N, kOff>(v, load_param(a.scale, a.scale_dtype, entry),
                                       kOff ? load_param(a.offset, a.scale_dtype, entry) : 0.0f);
        } else {
          const int64_t first = (r / a.group_size) * a.table_cols + static_cast<int64_t>(vi) * N;
          float sc[N], of[N];
          load_table<N>(a.scale, a.scale_dtype, first, sc);
          if (kOff) load_table<N>(a.offset, a.scale_dtype, first, of);
          apply_element_constants<N, kOff>(v, sc, of);
        }
        store_vector<OUT, N>(dst, vi, v);
      }
    }
  }
}

// Any shape and alignment: one element per thread step, grid-strided rows.
template <int OUT, bool kFour, bool kOff, int LAYOUT>
__global__ void __launch_bounds__(kDequantBlock) dequant_generic_kernel(const DequantArgs a) {
  pdl_launch_dependents();
  pdl_wait_primary();
  for (int64_t r = blockIdx.x; r < a.rows; r += gridDim.x) {
    for (int64_t c = threadIdx.x; c < a.cols; c += kDequantBlock) {
      const int64_t entry = LAYOUT == kPerToken        ? r
                            : LAYOUT == kGroupAlongRow ? r * a.table_cols + c / a.group_size
                                                       : (r / a.group_size) * a.table_cols + c;
      const float scale = load_param(a.scale, a.scale_dtype, entry);
      const float offset = kOff ? load_param(a.offset, a.scale_dtype, entry) : 0.0f;
      const int64_t i = r * a.cols + c;
      int code;
      if (kFour) {
        const uint8_t byte = static_cast<const uint8_t*>(a.y)[i >> 1];
        const int nib = (i & 1) ? (byte >> 4) : (byte & 0xF);
        code = nib >= 8 ? nib - 16 : nib;
      } else {
        code = static_cast<const int8_t*>(a.y)[i];
      }
      float v = static_cast<float>(code);
      if (kOff) v = __fsub_rn(v, offset);
      v = __fmul_rn(v, scale);
      if constexpr (OUT == kOutF32) {
        static_cast<float*>(a.out)[i] = v;
      } else {
        OutTraits<OUT>::store1(a.out, i, v);
      }
    }
  }
}

}  // namespace dq
