// Per-token dynamic quantization kernels (aclnnDynamicQuantV2, "Formula" and
// "Description"), sm_100a.
//
// The operation moves 2 B/element in and 1 or 0.5 B/element out, so it is
// bounded by HBM bandwidth if each element costs only a handful of
// instructions. Two kernels:
//   * bulk-copy kernel (rows whose bytes, smooth-scale rows and code rows are
//     suitably aligned): a row group of one or more warps per row, persistent
//     grid. Each group keeps a ring of shared-memory row buffers filled with
//     cp.async.bulk (TMA) copies of its next rows, reduces the row (one-
//     instruction warp reductions, then a shared-memory combine across the
//     group's warps), derives the row constants, then quantizes the row with an exact FMA division
//     (two-term reciprocal, one Markstein correction; branch-free) and packs
//     codes with byte permutes.
//   * generic kernel: any cols / alignment; one CTA per row (grid-strided),
//     two passes over the row (the second one mostly hits L2).
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

// Shared memory of the bulk-copy kernel: [groups][stages] row buffers, then
// [groups][stages] mbarriers, then the MoE group index.
__host__ __device__ inline size_t dq_smem_bytes(int groups, int stages, uint32_t stride, int num_groups) {
  return static_cast<size_t>(groups) * stages * stride + static_cast<size_t>(groups) * stages * 8 +
         static_cast<size_t>(num_groups) * 4;
}

// ============================================================ bulk-copy kernel

// Smooth-scale storage kinds (template parameter of the bulk-copy kernel).
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

// Rows whose RowQuant has exact_row set (scale below 2^-40, or a non-finite
// offset): every element of the row with the IEEE division. Out of line and
// reached only for such rows.
template <typename InT, int MODE, int OUT, int SMK>
__device__ __noinline__ void quantize_row_exact(const uint4* srow, const void* smooth_row, RowQuant q, int lane_g,
                                                int tpr, int nvec, uint8_t* yrow) {
  using C = QuantConsts<MODE, OUT>;
  for (int vi = lane_g; vi < nvec; vi += tpr) {
    float v[8];
    input8<InT, SMK>(srow[vi], smooth_row, vi, v);
    uint32_t bits[8];
    quant8_exact<MODE == kAsym>(v, q, C::kLo, C::kHi, bits);
    if (OUT == kOutInt8) {
      reinterpret_cast<uint2*>(yrow)[vi] = pack8_int8(bits);
    } else {
      reinterpret_cast<unsigned int*>(yrow)[vi] = pack8_int4(bits);
    }
  }
}

// Row groups of tpr = 32 * G threads, `groups` row groups per CTA. Each group
// owns a ring of `stages` shared-memory row buffers that its first lane keeps
// filled with cp.async.bulk (TMA) copies of the group's next rows. Warp w of a
// group owns the contiguous chunk of 32 * VPT 16-byte vectors starting at
// w * 32 * VPT; lane l of it owns vectors chunk + l + 32 * k (k < VPT), so
// consecutive lanes touch consecutive 16-byte vectors (conflict-free shared
// loads, coalesced stores) and every per-k offset is a compile-time constant.
// kRagged: the row is not exactly G * 32 * VPT vectors, so vectors past the
// row end are skipped.
//   pass 1: copy the thread's vectors from the stage into registers (raw
//     16-bit values) and reduce (packed 16-bit pairs without smooth scales;
//     fp32 products with them, kept in registers for pass 2 when VPT <= 4);
//     the group reduces through warp shuffles and, for G > 1, shared memory
//     behind its named barrier. That barrier also tells the leader that the
//     stage has been read by every thread, so the stage is refilled right
//     away: while a group quantizes one row, its next `stages` rows are in
//     flight.
//   pass 2: from registers only: widen (* smooth) unless kept, exact FMA
//     division, magic rounding, byte-permute packing, one 8-byte (int8) or
//     4-byte (int4) store per vector.
constexpr int kWarpKernelMaxThreads = 512;
#ifndef DQ_MAX_REGS
#define DQ_MAX_REGS 128  // registers per thread: 2 CTAs of 256 threads per SM
#endif

template <typename InT, int MODE, int OUT, int SMK, int VPT, bool kRagged>
__global__ void __maxnreg__(DQ_MAX_REGS)
dynamic_quant_tma_kernel(const RowQuantArgs a) {
  using C = QuantConsts<MODE, OUT>;
  using P = Packed<InT>;
  constexpr bool kA = MODE == kAsym;
#ifndef DQ_KEEP_MAX_VPT
#define DQ_KEEP_MAX_VPT 8
#endif
  constexpr bool kKeep = SMK != kSmNone && VPT <= DQ_KEEP_MAX_VPT;  // fp32 products stay in registers
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[2][2][kWarpKernelMaxThreads / 32];  // [parity][max, min][warp]

  const int tpr = a.tpr;
  const int g = threadIdx.x / tpr;
  const int lane_g = threadIdx.x - g * tpr;
  const int warp = threadIdx.x >> 5;
  const int warp_g0 = (g * tpr) >> 5;
  const int nwarps_g = tpr >> 5;
  const int lane = threadIdx.x & 31;
  const int vbase = (lane_g >> 5) * (32 * VPT) + lane;  // this thread's vector k is vbase + 32 * k
  const int S = a.stages;
  const int NG = a.groups;
  const uint32_t stride = a.stage_stride;
  const size_t ring_bytes = static_cast<size_t>(NG) * S * stride;
  uint8_t* ring = smem + static_cast<size_t>(g) * S * stride;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ring_bytes) + g * S;
  int32_t* gi_s = reinterpret_cast<int32_t*>(smem + ring_bytes + static_cast<size_t>(NG) * S * 8);

  const bool moe = a.group_index != nullptr;
  if (threadIdx.x == 0) {
    uint64_t* all = reinterpret_cast<uint64_t*>(smem + ring_bytes);
    for (int i = 0; i < NG * S; ++i) mbar_init(all + i, 1);
    fence_mbarrier_init();
  }
  // launched as a programmatic dependent: the set-up above overlaps the tail
  // of the previous kernel; every global memory access comes after the wait
  pdl_launch_dependents();
  pdl_wait_primary();
  if (moe) {
    for (int i = threadIdx.x; i < a.num_groups; i += blockDim.x) gi_s[i] = a.group_index[i];
  }
  __syncthreads();
  write_group_status(a);

  const int64_t workers = static_cast<int64_t>(gridDim.x) * NG;
  const int64_t worker = static_cast<int64_t>(blockIdx.x) * NG + g;
  const int64_t r_begin = worker * a.rows / workers;
  const int64_t r_end = (worker + 1) * a.rows / workers;
  const int n = static_cast<int>(r_end - r_begin);  // rows of this group (< 2^31 by validation)
  if (n <= 0) return;  // whole group idle (its barriers are group-local)

  const int nvec = static_cast<int>(a.cols >> 3);
  const uint32_t row_bytes = static_cast<uint32_t>(a.cols) * 2u;
  const bool leader = lane_g == 0;
  const uint64_t policy = leader ? l2_evict_first_policy() : 0;
  const uint8_t* x_next = static_cast<const uint8_t*>(a.x) + r_begin * static_cast<int64_t>(row_bytes);
  int issued = 0;
  auto issue_into = [&](int st) {  // leader only
    mbar_arrive_expect_tx(bars + st, row_bytes);
    bulk_copy_g2s(ring + static_cast<size_t>(st) * stride, x_next, row_bytes, bars + st, policy);
    x_next += row_bytes;
    ++issued;
  };
  if (leader) {
    for (int st = 0; st < S && st < n; ++st) issue_into(st);
  }

  const size_t smooth_row_bytes = static_cast<size_t>(a.cols) * (SMK == kSmF32 ? 4 : 2);
  const uint8_t* smooth_row = static_cast<const uint8_t*>(a.smooth);
  int cur_expert = moe ? -1 : 0;
  int64_t expert_end = moe ? -1 : INT64_MAX;
  const int64_t y_row_bytes = OUT == kOutInt8 ? a.cols : (a.cols >> 1);
  uint8_t* yrow = static_cast<uint8_t*>(a.y) + r_begin * y_row_bytes;
  auto in_row = [&](int k) { return !kRagged || vbase + 32 * k < nvec; };

  int st = 0;
  uint32_t phase = 0;
  int parity = 0;
  for (int i = 0; i < n; ++i, yrow += y_row_bytes) {
    const int64_t r = r_begin + i;
    const bool arrived = mbar_wait_parity(bars + st, phase);
    const uint4* srow = reinterpret_cast<const uint4*>(ring + static_cast<size_t>(st) * stride);

    bool row_valid = true;
    if (moe) {
      if (r >= expert_end) {
        const int e = expert_of(gi_s, a.num_groups, r);
        cur_expert = e;
        expert_end = e < a.num_groups ? static_cast<int64_t>(gi_s[e]) : INT64_MAX;
        smooth_row = static_cast<const uint8_t*>(a.smooth) + static_cast<size_t>(e < a.num_groups ? e : 0) *
                                                                 smooth_row_bytes;
      }
      row_valid = cur_expert < a.num_groups;
    }

    // ---- pass 1: this thread's vectors into registers, reduce
    uint4 raw[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) raw[k] = in_row(k) ? srow[vbase + 32 * k] : make_uint4(0, 0, 0, 0);
    float m0, m1;
    constexpr int NACC = VPT < 4 ? VPT : 4;  // independent accumulators: short dependency chains
    float prod[kKeep ? VPT : 1][8];
    if (SMK != kSmNone) {
      float amx[NACC], amn[NACC];
#pragma unroll
      for (int j = 0; j < NACC; ++j) {
        amx[j] = kA ? -INFINITY : 0.0f;
        amn[j] = INFINITY;
      }
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (in_row(k)) {
          float v[8];
          input8<InT, SMK>(raw[k], smooth_row, vbase + 32 * k, v);
          if (kKeep) {
#pragma unroll
            for (int j = 0; j < 8; ++j) prod[kKeep ? k : 0][j] = v[j];
          }
          if (kA) {
            amx[k % NACC] = fmaxf(amx[k % NACC], max8(v));
            amn[k % NACC] = fminf(amn[k % NACC], min8(v));
          } else {
            amx[k % NACC] = fmaxf(amx[k % NACC], absmax8(v));
          }
        }
      }
      m0 = tree<NACC, true>(amx);
      m1 = kA ? tree<NACC, false>(amn) : INFINITY;
    } else {
      typename P::T2 hmax[NACC], hmin[NACC];
#pragma unroll
      for (int j = 0; j < NACC; ++j) {
        hmax[j] = kA ? P::lowest() : P::zero();
        hmin[j] = P::highest();
      }
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (in_row(k)) {
          const uint32_t w[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
          if (kA) {
            hmax[k % NACC] = P::vmax(hmax[k % NACC], P::vmax(P::vmax(P::from_bits(w[0]), P::from_bits(w[1])),
                                                              P::vmax(P::from_bits(w[2]), P::from_bits(w[3]))));
            hmin[k % NACC] = P::vmin(hmin[k % NACC], P::vmin(P::vmin(P::from_bits(w[0]), P::from_bits(w[1])),
                                                              P::vmin(P::from_bits(w[2]), P::from_bits(w[3]))));
          } else {
            hmax[k % NACC] = P::vmax(hmax[k % NACC],
                                     P::vmax(P::vmax(P::from_bits(w[0] & 0x7FFF7FFFu), P::from_bits(w[1] & 0x7FFF7FFFu)),
                                             P::vmax(P::from_bits(w[2] & 0x7FFF7FFFu), P::from_bits(w[3] & 0x7FFF7FFFu))));
          }
        }
      }
#pragma unroll
      for (int w = 1; w < NACC; w *= 2) {
#pragma unroll
        for (int i = 0; i + w < NACC; i += 2 * w) {
          hmax[i] = P::vmax(hmax[i], hmax[i + w]);
          if (kA) hmin[i] = P::vmin(hmin[i], hmin[i + w]);
        }
      }
      m0 = P::hi_lo_max(hmax[0]);
      m1 = kA ? P::hi_lo_min(hmin[0]) : INFINITY;
    }
    m0 = warp_max(m0);
    if (kA) m1 = warp_min(m1);
    bool failed;
    if (nwarps_g > 1) {
      if (lane == 0) {
        red[parity][0][warp] = m0;
        if (kA) red[parity][1][warp] = m1;
      }
      failed = group_barrier_or(1 + g, tpr, !arrived);
      // lane j takes warp j's partial; one more warp reduction combines them
      const bool has = lane < nwarps_g;
      m0 = warp_max(has ? red[parity][0][warp_g0 + lane] : (kA ? -INFINITY : 0.0f));
      if (kA) m1 = warp_min(has ? red[parity][1][warp_g0 + lane] : INFINITY);
      parity ^= 1;
    } else {
      failed = __any_sync(0xffffffffu, !arrived);
    }
    if (failed) {
      // A row copy never completed (not a data-dependent condition): mark this
      // and the group's remaining rows with NaN scales, drain, and stop.
      for (int64_t rr = r + lane_g; rr < r_end; rr += tpr) a.scale[rr] = __int_as_float(0x7fc00000);
      if (leader) {
        int s2 = st;
        uint32_t ph = phase;
        for (int j = i + 1; j < issued; ++j) {
          s2 = s2 + 1 == S ? 0 : s2 + 1;
          if (s2 == 0) ph ^= 1u;
          mbar_wait_parity(bars + s2, ph);
        }
      }
      return;
    }

    RowQuant q = kA ? make_asym<C::kDivisor, C::kOffsetOptInt>(m0, m1) : make_sym<C::kDivisor>(m0);
    const bool exact = q.exact_row && row_valid && !q.zero_scale;
    if (exact) {
      // rare: the stage is still needed by the out-of-line exact path
      quantize_row_exact<InT, MODE, OUT, SMK>(srow, smooth_row, q, lane_g, tpr, nvec, yrow);
      if (nwarps_g > 1) group_barrier(1 + g, tpr); else __syncwarp();
    }
    // Every thread of the group has its share of the row in registers (and the
    // exact path, if taken, is done): refill this stage with the group's next row.
    if (leader && issued < n) {
      fence_proxy_async_smem();
      issue_into(st);
    }
    st = st + 1 == S ? 0 : st + 1;
    if (st == 0) phase ^= 1u;
    if (!row_valid) {
      q.scale = 0.0f;
      q.offset = 0.0f;
    }
    if (leader) {
      __stcs(a.scale + r, q.scale);
      if (kA) __stcs(a.offset + r, q.offset);
    }
    if (exact) continue;

    // ---- pass 2: quantize from registers and store
    auto store8 = [&](int k, const uint32_t (&bits)[8]) {
      const int vi = vbase + 32 * k;
      if (OUT == kOutInt8) {
        __stcs(reinterpret_cast<uint2*>(yrow) + vi, pack8_int8(bits));
      } else {
        __stcs(reinterpret_cast<unsigned int*>(yrow) + vi, pack8_int4(bits));
      }
    };
    if (!row_valid || q.zero_scale) {
      // every code of the row is the same: 0, or offset_opt for a constant
      // asymmetric row (rows past the last group get 0)
      const uint32_t cb = __float_as_uint(__fadd_rn(row_valid ? C::kOffsetOpt : 0.0f, kRoundMagic));
      uint32_t bits[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) bits[j] = cb;
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (in_row(k)) store8(k, bits);
      }
      continue;
    }
    auto pass2 = [&](auto clamp_tag) {
      constexpr bool kClamp = decltype(clamp_tag)::value;
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (!in_row(k)) continue;
        float v[8];
        if (kKeep) {
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = prod[kKeep ? k : 0][j];
        } else {
          input8<InT, SMK>(raw[k], smooth_row, vbase + 32 * k, v);
        }
        uint32_t bits[8];
        quant8<kA, kClamp>(v, q, C::kLo, C::kHi, bits);
        store8(k, bits);
      }
    };
    if (kA && q.clamp) {
      pass2(BoolTag<true>{});
    } else {
      pass2(BoolTag<false>{});
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
