// Per-token dynamic quantization kernels (aclnnDynamicQuantV2, "Formula" and
// "Description"), sm_100a.
//
// The operation is HBM-bound: each row is read once (2 B/element) and its
// codes written once (1 or 0.5 B/element). Design:
//   * vector kernel: a persistent grid; each CTA holds `groups` row groups of
//     `tpr` threads, and each group walks a contiguous range of rows. A thread
//     owns VPT 16-byte vectors (8 elements each) of the row, so the whole row
//     sits in registers; the next row's vectors are loaded while the current
//     one is reduced and quantized (one row of prefetch per group). Smooth
//     scales for the thread's columns live in registers and are reloaded only
//     when the MoE expert changes. Reductions: warp shuffles, then the
//     group's warps through shared memory behind a named barrier.
//   * generic kernel: any cols / alignment; one CTA per row (grid-strided),
//     two passes over the row (the second one mostly hits L2).
#pragma once

#include "dq_device.cuh"

namespace dq {

enum : int { kSym = 0, kAsym = 1 };
enum : int { kOutInt8 = 0, kOutInt4 = 1 };  // kOutInt4: INT4X2 and INT32 share bytes

struct RowQuantArgs {
  const void* x;
  int64_t rows;
  int64_t cols;
  const void* smooth;          // nullptr, [cols] or [num_groups, cols]
  int smooth_dtype;
  const int32_t* group_index;  // nullptr or [num_groups] cumulative end rows
  int num_groups;
  void* y;
  float* scale;
  float* offset;               // asymmetric only
  uint32_t* status;            // workspace status word (with a group index)
  int tpr;                     // threads per row group (vector kernel)
  int groups;                  // row groups per CTA (vector kernel)
};

template <int MODE, int OUT>
struct QuantConsts {
  static constexpr bool kFour = OUT == kOutInt4;
  static constexpr float kDivisor = MODE == kSym ? (kFour ? 7.0f : 127.0f) : (kFour ? 15.0f : 255.0f);
  static constexpr float kOffsetOpt = MODE == kSym ? 0.0f : (kFour ? 7.0f : 127.0f);
  static constexpr float kLo = MODE == kSym ? (kFour ? -7.0f : -127.0f) : (kFour ? -8.0f : -128.0f);
  static constexpr float kHi = MODE == kSym ? (kFour ? 7.0f : 127.0f) : (kFour ? 7.0f : 127.0f);
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

// ============================================================ vector kernel

constexpr int kMaxBlock = 512;

template <typename InT, int MODE, int OUT, int VPT>
__global__ void __launch_bounds__(kMaxBlock)
dynamic_quant_vec_kernel(const RowQuantArgs a) {
  using C = QuantConsts<MODE, OUT>;
  __shared__ float red[2][kMaxBlock / 32][2];
  extern __shared__ int32_t gi_smem[];

  write_group_status(a);
  const bool moe = a.group_index != nullptr;
  if (moe) {
    for (int i = threadIdx.x; i < a.num_groups; i += blockDim.x) gi_smem[i] = a.group_index[i];
    __syncthreads();
  }

  const int tpr = a.tpr;
  const int g = threadIdx.x / tpr;
  const int lane_g = threadIdx.x - g * tpr;
  const int warp = threadIdx.x >> 5;
  const int warp_g0 = (g * tpr) >> 5;  // first warp of this group
  const int nwarps_g = tpr >> 5;
  const int lane = threadIdx.x & 31;

  const int64_t workers = static_cast<int64_t>(gridDim.x) * a.groups;
  const int64_t worker = static_cast<int64_t>(blockIdx.x) * a.groups + g;
  const int64_t r_begin = worker * a.rows / workers;
  const int64_t r_end = (worker + 1) * a.rows / workers;
  if (r_begin >= r_end) return;  // whole group idle (its barrier is group-local)

  const int64_t nvec = a.cols >> 3;
  const uint4* __restrict__ xv = static_cast<const uint4*>(a.x);

  // smooth scales of this thread's columns
  float sm[VPT][8];
  const bool has_smooth = a.smooth != nullptr;
  int cur_expert = -1;
  int64_t expert_end = -1;  // rows < expert_end belong to cur_expert
  auto load_smooth = [&](int e) {
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int64_t vi = lane_g + static_cast<int64_t>(k) * tpr;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sm[k][j] = vi < nvec ? load_param(a.smooth, a.smooth_dtype, e * a.cols + vi * 8 + j) : 1.0f;
      }
    }
  };
  if (has_smooth && !moe) load_smooth(0);

  uint4 cur[VPT], nxt[VPT];
  auto load_row = [&](int64_t r, uint4 (&buf)[VPT]) {
    const uint4* p = xv + r * nvec;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int64_t vi = lane_g + static_cast<int64_t>(k) * tpr;
      if (vi < nvec) buf[k] = __ldcs(p + vi);
    }
  };
  load_row(r_begin, cur);

  int parity = 0;
  for (int64_t r = r_begin; r < r_end; ++r) {
    if (r + 1 < r_end) load_row(r + 1, nxt);

    bool row_valid = true;
    if (moe) {
      if (r >= expert_end) {
        const int e = expert_of(gi_smem, a.num_groups, r);
        if (e >= a.num_groups) {
          row_valid = false;
          expert_end = INT64_MAX;
          cur_expert = a.num_groups;
        } else {
          expert_end = gi_smem[e];
          if (e != cur_expert) {
            load_smooth(e);
            cur_expert = e;
          }
        }
      }
      row_valid = cur_expert < a.num_groups;
    }

    // widen (+ smooth multiply), reduce
    float v[VPT][8];
    float m0 = MODE == kSym ? 0.0f : -INFINITY;  // absmax or max
    float m1 = INFINITY;                         // min (asymmetric)
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int64_t vi = lane_g + static_cast<int64_t>(k) * tpr;
      InTraits<InT>::widen8(cur[k], v[k]);
      if (has_smooth) {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[k][j] = __fmul_rn(v[k][j], sm[k][j]);
      }
      if (vi < nvec) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (MODE == kSym) {
            m0 = fmaxf(m0, fabsf(v[k][j]));
          } else {
            m0 = fmaxf(m0, v[k][j]);
            m1 = fminf(m1, v[k][j]);
          }
        }
      }
    }
    m0 = warp_max(m0);
    if (MODE == kAsym) m1 = warp_min(m1);
    if (nwarps_g > 1) {
      if (lane == 0) {
        red[parity][warp][0] = m0;
        red[parity][warp][1] = m1;
      }
      group_barrier(1 + g, tpr);
      m0 = red[parity][warp_g0][0];
      m1 = red[parity][warp_g0][1];
      for (int w = 1; w < nwarps_g; ++w) {
        m0 = fmaxf(m0, red[parity][warp_g0 + w][0]);
        if (MODE == kAsym) m1 = fminf(m1, red[parity][warp_g0 + w][1]);
      }
      parity ^= 1;
    }

    RowQuant q = MODE == kSym ? make_sym(m0, C::kDivisor) : make_asym(m0, m1, C::kDivisor, C::kOffsetOpt);
    if (!row_valid) {
      q.scale = 0.0f;
      q.offset = 0.0f;
    }
    if (lane_g == 0) {
      __stcs(a.scale + r, q.scale);
      if (MODE == kAsym) __stcs(a.offset + r, q.offset);
    }

#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int64_t vi = lane_g + static_cast<int64_t>(k) * tpr;
      if (vi >= nvec) continue;
      float c[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!row_valid) {
          c[j] = 0.0f;
        } else if (q.zero_scale) {
          c[j] = C::kOffsetOpt;
        } else if (MODE == kSym) {
          c[j] = sym_code(v[k][j], q, C::kLo, C::kHi);
        } else {
          c[j] = asym_code(v[k][j], q, C::kLo, C::kHi);
        }
      }
      if (OUT == kOutInt8) {
        uint2* yp = reinterpret_cast<uint2*>(static_cast<int8_t*>(a.y) + r * a.cols) + vi;
        __stcs(yp, pack_int8x8(c));
      } else {
        uint32_t* yp = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(a.y) + r * (a.cols >> 1)) + vi;
        __stcs(reinterpret_cast<unsigned int*>(yp), pack_int4x8(c));
      }
    }

#pragma unroll
    for (int k = 0; k < VPT; ++k) cur[k] = nxt[k];
  }
}

// ============================================================ generic kernel

constexpr int kGenericBlock = 256;

template <typename InT, int MODE, int OUT>
__global__ void __launch_bounds__(kGenericBlock)
dynamic_quant_generic_kernel(const RowQuantArgs a) {
  using C = QuantConsts<MODE, OUT>;
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
    float m0 = MODE == kSym ? 0.0f : -INFINITY;
    float m1 = INFINITY;
    if (row_valid) {
      for (int64_t c = threadIdx.x; c < a.cols; c += kGenericBlock) {
        const float v = input(c);
        if (MODE == kSym) {
          m0 = fmaxf(m0, fabsf(v));
        } else {
          m0 = fmaxf(m0, v);
          m1 = fminf(m1, v);
        }
      }
    }
    m0 = warp_max(m0);
    if (MODE == kAsym) m1 = warp_min(m1);
    if (lane == 0) {
      red[warp][0] = m0;
      red[warp][1] = m1;
    }
    __syncthreads();
    m0 = red[0][0];
    m1 = red[0][1];
    for (int w = 1; w < kWarps; ++w) {
      m0 = fmaxf(m0, red[w][0]);
      if (MODE == kAsym) m1 = fminf(m1, red[w][1]);
    }
    __syncthreads();  // red[] is rewritten by the next row

    RowQuant q = MODE == kSym ? make_sym(m0, C::kDivisor) : make_asym(m0, m1, C::kDivisor, C::kOffsetOpt);
    if (!row_valid) {
      q.scale = 0.0f;
      q.offset = 0.0f;
    }
    if (threadIdx.x == 0) {
      a.scale[r] = q.scale;
      if (MODE == kAsym) a.offset[r] = q.offset;
    }
    auto code = [&](int64_t c) -> int {
      if (!row_valid) return 0;
      if (q.zero_scale) return static_cast<int>(C::kOffsetOpt);
      const float v = input(c);
      return __float2int_rn(MODE == kSym ? sym_code(v, q, C::kLo, C::kHi) : asym_code(v, q, C::kLo, C::kHi));
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
