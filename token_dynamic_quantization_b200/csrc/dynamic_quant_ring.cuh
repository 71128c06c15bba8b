// Per-token dynamic quantization, ring kernel (aclnnDynamicQuantV2, "Formula"
// and "Description"), sm_100a.
//
// One persistent CTA per SM owns a contiguous range of rows and one ring of
// NS shared-memory row slots; local row j lives in slot j % NS.
//   * Before griddepcontrol.wait (while the kernel before finishes), thread
//     0 prefetches about 48 KB of the CTA's first rows into L2
//     (cp.async.bulk.prefetch; 8192 x 4096 bf16: 17.4 us against 18.3 us
//     per launch).
//   * After the wait, thread 0 issues cp.async.bulk (TMA) copies of the CTA's
//     first rows, each completing its slot's `full` mbarrier (transaction
//     count): ceil(NC / 2) of them at once, the rest of the ring after the
//     CTA's set-up. Copies in flight together share the memory system, so
//     all NS issued at once land at about the same time, late; a few issued
//     first land early and the row groups start on them while the rest are
//     on their way (8192 x 4096 bf16: 18.6 us against 20.4 us per launch).
//   * The warps form NC row groups of G warps; group c takes the CTA's rows
//     c, c + NC, c + 2NC, ... A group reads its row once from the slot into
//     registers (pass 1: widen, multiply by the smooth scales, reduce). Once
//     all of its warps are past that point (the group's barrier, which also
//     exchanges their partial reductions), its first lane refills the slot
//     with the row NS further on. The group then combines the partial
//     reductions, derives the row constants and quantizes from registers
//     (pass 2).
// Because the slots are shared by the whole CTA, copies run ahead of every
// group by up to NS rows, independently of which group is slowest, and no
// warp is set aside for issuing copies.
//
// Dense smooth-scale tables are staged once per CTA in shared memory. MoE
// tables (one row per expert): the rows of the experts of the CTA's first
// and last rows are staged too when they are at most two (a CTA's contiguous
// rows rarely span more; 32768 x 7168 bf16, 64 experts: 116 us against
// 130 us reading them through L1), and any row of another expert reads
// its smooth row through L1.
//
// Failure handling: every wait is bounded in time (tma_pipeline.cuh) and also
// gives up when a shared abort flag is set. A group whose row copy never
// completes writes NaN scales for its remaining rows, sets the flag and
// stops; the other groups stop at their next row that has not landed; before
// the CTA exits, thread 0 waits (bounded) for every slot's last copy. No
// thread waits forever.
#pragma once

#include "dq_args.cuh"
#include "dq_device.cuh"
#include "ring_prefetch.cuh"
#include "dynamic_quant_kernels.cuh"
#include "tma_pipeline.cuh"

namespace dq {

// Shared memory of the ring kernel, in this order: NS row slots of `stride`
// bytes; full[NS] mbarriers; per slot the fill round of its last issued copy
// (and a spare word); a 16-byte abort word; the staged smooth table
// (`smooth_bytes`, a multiple of 16); the MoE group index.
__host__ __device__ inline size_t ring_smem_bytes(int slots, uint32_t stride, size_t smooth_bytes, int num_groups) {
  return static_cast<size_t>(slots) * stride + static_cast<size_t>(slots) * 16 + 16 + smooth_bytes +
         static_cast<size_t>(num_groups) * 4;
}

// Smooth scales of vector vi from the staged shared-memory copy. An fp32
// table is staged as two planes (elements 0-3 and 4-7 of every 8-column
// vector), so that 32 lanes reading consecutive vectors read consecutive
// 16-byte words: no bank conflicts. `nvec` is the number of vectors.
template <int SMK>
__device__ __forceinline__ void load_smooth8_smem(const uint8_t* s, int vi, int nvec, float (&v)[8]) {
  if (SMK == kSmF32) {
    const float4* p = reinterpret_cast<const float4*>(s);
    const float4 a = p[vi], b = p[nvec + vi];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else if (SMK == kSmBF16) {
    InTraits<__nv_bfloat16>::widen8(reinterpret_cast<const uint4*>(s)[vi], v);
  } else if (SMK == kSmF16) {
    InTraits<__half>::widen8(reinterpret_cast<const uint4*>(s)[vi], v);
  }
}

#ifndef DQ_RING_MAX_REGS
#define DQ_RING_MAX_REGS 128
#endif

// kSmemSmooth: the smooth table (dense, no group index) is staged in shared
// memory; otherwise smooth rows are read with __ldg, or, for MoE inputs with
// a.moe_stage set, from the up to two expert rows staged in shared memory
// (the staged region holds 2 rows then).
template <typename InT, int MODE, int OUT, int SMK, int VPT, bool kRagged, bool kSmemSmooth>
__global__ void __maxnreg__(DQ_RING_MAX_REGS) dynamic_quant_ring_kernel(const RowQuantArgs a) {
  using C = QuantConsts<MODE, OUT>;
  using P = Packed<InT>;
  constexpr bool kA = MODE == kAsym;
  constexpr bool kSmooth = SMK != kSmNone;
  constexpr int kSmoothElem = SMK == kSmF32 ? 4 : 2;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[2][2][kRingMaxThreads / 32];  // [parity][max, min][warp]

  const int NS = a.stages;
  const uint32_t stride = a.stage_stride;
  const int tpr = a.tpr;
  const int G = tpr >> 5;
  const int NC = a.groups;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(NS) * stride);
  // fill round of the slot's last issued copy (-1: none). An mbarrier only
  // exposes the parity of its current phase, so a group that reaches round k
  // of a slot first waits until round k has been issued, and only then for
  // the phase's parity: it can never mistake a pending round k - 1 for k.
  volatile int32_t* issued_round = reinterpret_cast<volatile int32_t*>(full + NS);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(issued_round + 2 * NS);
  uint8_t* smooth_s = reinterpret_cast<uint8_t*>(const_cast<int32_t*>(issued_round) + 2 * NS) + 16;
  const size_t smooth_row_bytes = static_cast<size_t>(a.cols) * kSmoothElem;
  const bool moe_stage = !kSmemSmooth && kSmooth && a.group_index != nullptr && a.moe_stage != 0;
  const size_t smooth_bytes = kSmemSmooth ? smooth_row_bytes : (moe_stage ? 2 * smooth_row_bytes : 0);
  int32_t* gi_s = reinterpret_cast<int32_t*>(smooth_s + smooth_bytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool moe = a.group_index != nullptr;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.x) * a.rows / gridDim.x;
  const int n = static_cast<int>((static_cast<int64_t>(blockIdx.x) + 1) * a.rows / gridDim.x - r_begin);
  const uint32_t row_bytes = static_cast<uint32_t>(a.cols) * 2u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      issued_round[s] = -1;
    }
    *abort_flag = 0u;
    fence_mbarrier_init();
  }
  // launched as a programmatic dependent: the set-up above overlaps the tail
  // of the previous kernel, and so does an L2 prefetch of the CTA's first
  // rows (a hint: it returns no data); every global load and store comes
  // after the wait
  const uint8_t* x_cta = static_cast<const uint8_t*>(a.x) + r_begin * static_cast<int64_t>(row_bytes);
  if (threadIdx.x == 0) {
    const int npf = ring_prefetch_rows(row_bytes, NS, n);
    for (int j = 0; j < npf; ++j) bulk_prefetch_l2(x_cta + static_cast<int64_t>(j) * row_bytes, row_bytes);
  }
  pdl_launch_dependents();
  pdl_wait_primary();

  // local row j of the CTA into slot s (= j % NS), completing full[s]
  const uint64_t policy = l2_evict_first_policy();
  auto issue = [&](int s, int j, int round) {  // round = j / NS
    __threadfence_block();
    issued_round[s] = round;
#ifdef DQ_TEST_SKIP_COPY_ROW
    // test builds only: leave one row's copy out, so that its consumer's
    // bounded wait runs out and the failure path runs
    if (r_begin + j == static_cast<int64_t>(DQ_TEST_SKIP_COPY_ROW)) return;
#endif
    mbar_arrive_expect_tx(full + s, row_bytes);
    bulk_copy_g2s(smem + static_cast<size_t>(s) * stride, x_cta + static_cast<int64_t>(j) * row_bytes, row_bytes,
                  full + s, policy);
  };
  // the first ceil(NC / 2) rows before anything else, the rest of the ring
  // once the smooth table is staged
  const int first_fill = (NC + 1) / 2;
  if (threadIdx.x == 0) {
    for (int j = 0; j < first_fill && j < n; ++j) issue(j, j, 0);
  }
  if (moe) {
    for (int i = threadIdx.x; i < a.num_groups; i += blockDim.x) gi_s[i] = a.group_index[i];
  }
  // smooth rows staged: the dense table, or the experts e_lo .. e_lo +
  // n_staged - 1 of the CTA's first and last rows
  int e_lo = 0, n_staged = kSmemSmooth ? 1 : 0;
  if (moe_stage) {
    __syncthreads();  // the group index is in shared memory
    if (n > 0) {
      e_lo = expert_of(gi_s, a.num_groups, r_begin);
      int e_hi = expert_of(gi_s, a.num_groups, r_begin + n - 1);
      if (e_hi >= a.num_groups) e_hi = a.num_groups - 1;  // rows past the last group use no smooth row
      if (e_lo < a.num_groups && e_hi >= e_lo && e_hi - e_lo <= 1) n_staged = e_hi - e_lo + 1;
    }
  }
  if (kSmemSmooth || moe_stage) {
    const int words = static_cast<int>(smooth_row_bytes / 16);
    const int nv = static_cast<int>(a.cols >> 3);
    for (int t = 0; t < n_staged; ++t) {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.smooth) +
                                                        static_cast<size_t>(e_lo + t) * smooth_row_bytes);
      uint4* dst = reinterpret_cast<uint4*>(smooth_s + static_cast<size_t>(t) * smooth_row_bytes);
      for (int i = threadIdx.x; i < words; i += blockDim.x) {
        // fp32: word i is half (i & 1) of vector i / 2 -> plane (i & 1)
        const int d = SMK == kSmF32 ? (i & 1) * nv + (i >> 1) : i;
        dst[d] = __ldg(src + i);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int j = first_fill; j < NS && j < n; ++j) issue(j, j, 0);
  }
  write_group_status(a);
  if (n <= 0) return;

  // ------------------------------------------------------------ row groups
  const int c = warp / G;              // group
  const int wg = warp - c * G;         // warp within the group
  const int lane_g = wg * 32 + lane;   // thread within the group
  const int warp_g0 = c * G;           // first warp of the group
  const int nvec = static_cast<int>(a.cols >> 3);
  const int vbase = wg * (32 * VPT) + lane;  // this thread's vector k is vbase + 32 * k
  auto in_row = [&](int k) { return !kRagged || vbase + 32 * k < nvec; };

  const uint8_t* smooth_row = static_cast<const uint8_t*>(a.smooth);
  const uint8_t* smooth_row_s = smooth_s;  // the row's staged smooth scales (when row_staged)
  bool row_staged = kSmemSmooth;
  int cur_expert = moe ? -1 : 0;
  int64_t expert_end = moe ? -1 : INT64_MAX;
  const int64_t y_row_bytes = OUT == kOutInt8 ? a.cols : (a.cols >> 1);
  const int64_t y_step = y_row_bytes * NC;
  uint8_t* yrow = static_cast<uint8_t*>(a.y) + (r_begin + c) * y_row_bytes;

  int s = c;           // slot of local row j (NC <= NS)
  int round = 0;       // its fill round, j / NS
  int parity = 0;      // red[] buffer
  for (int j = c; j < n && c < NC; j += NC, yrow += y_step) {
    const int64_t r = r_begin + j;
    const bool ok = wait_round(issued_round + s, round, abort_flag) &&
                    mbar_wait_parity_or_abort(full + s, static_cast<uint32_t>(round) & 1u, abort_flag);
    const uint4* srow = reinterpret_cast<const uint4*>(smem + static_cast<size_t>(s) * stride);

    bool row_valid = true;
    if (moe) {
      if (r >= expert_end) {
        const int e = expert_of(gi_s, a.num_groups, r);
        cur_expert = e;
        expert_end = e < a.num_groups ? static_cast<int64_t>(gi_s[e]) : INT64_MAX;
        smooth_row = static_cast<const uint8_t*>(a.smooth) +
                     static_cast<size_t>(e < a.num_groups ? e : 0) * smooth_row_bytes;
        row_staged = moe_stage && e >= e_lo && e < e_lo + n_staged;
        smooth_row_s = smooth_s + static_cast<size_t>(row_staged ? e - e_lo : 0) * smooth_row_bytes;
      }
      row_valid = cur_expert < a.num_groups;
    }

    // ---- pass 1: the thread's vectors into registers, reduce
    uint4 raw[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) raw[k] = in_row(k) ? srow[vbase + 32 * k] : make_uint4(0, 0, 0, 0);
    float m0, m1;
    constexpr int NACC = VPT < 4 ? VPT : 4;
    float prod[kSmooth ? VPT : 1][8];
    if (kSmooth) {
      float amx[NACC], amn[NACC];
#pragma unroll
      for (int t = 0; t < NACC; ++t) {
        amx[t] = kA ? -INFINITY : 0.0f;
        amn[t] = INFINITY;
      }
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (in_row(k)) {
          float v[8], sm[8];
          InTraits<InT>::widen8(raw[k], v);
          if (kSmemSmooth || row_staged) {
            load_smooth8_smem<SMK>(smooth_row_s, vbase + 32 * k, nvec, sm);
          } else {
            load_smooth8<SMK>(smooth_row, vbase + 32 * k, sm);
          }
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float2 pr = __fmul2_rn(make_float2(v[2 * p], v[2 * p + 1]), make_float2(sm[2 * p], sm[2 * p + 1]));
            prod[kSmooth ? k : 0][2 * p] = pr.x;
            prod[kSmooth ? k : 0][2 * p + 1] = pr.y;
          }
          if (kA) {
            amx[k % NACC] = fmaxf(amx[k % NACC], max8(prod[kSmooth ? k : 0]));
            amn[k % NACC] = fminf(amn[k % NACC], min8(prod[kSmooth ? k : 0]));
          } else {
            amx[k % NACC] = fmaxf(amx[k % NACC], absmax8(prod[kSmooth ? k : 0]));
          }
        }
      }
      m0 = tree<NACC, true>(amx);
      m1 = kA ? tree<NACC, false>(amn) : INFINITY;
    } else {
      typename P::T2 hmax[NACC], hmin[NACC];
#pragma unroll
      for (int t = 0; t < NACC; ++t) {
        hmax[t] = kA ? P::lowest() : P::zero();
        hmin[t] = P::highest();
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
    // every lane's shared loads of the slot are complete (their values fed the
    // warp reduction); once the whole group is past this point (its barrier
    // below, or this warp alone), the group's first lane refills the slot
    // with the row NS further on
    bool failed;
    if (G > 1) {
      if (lane == 0) {
        red[parity][0][warp] = m0;
        if (kA) red[parity][1][warp] = m1;
      }
      failed = group_barrier_or(1 + c, tpr, !ok);
    } else {
      failed = __any_sync(0xffffffffu, !ok);
    }
    if (lane_g == 0 && !failed && j + NS < n) {
      fence_proxy_async_smem();
      issue(s, j + NS, round + 1);
    }
    s += NC;  // slot and fill round of local row j + NC (NC <= NS)
    if (s >= NS) {
      s -= NS;
      ++round;
    }
    if (G > 1) {
      // lane i takes warp i's partial; one more warp reduction combines them
      const bool has = lane < G;
      m0 = warp_max(has ? red[parity][0][warp_g0 + lane] : (kA ? -INFINITY : 0.0f));
      if (kA) m1 = warp_min(has ? red[parity][1][warp_g0 + lane] : INFINITY);
      parity ^= 1;
    }
    if (failed) {
      // A row copy never completed (not a data-dependent condition): mark this
      // and the group's remaining rows with NaN scales and stop; the abort
      // flag stops the other groups at their next row that has not landed.
      *abort_flag = 1u;
      for (int jj = j + lane_g * NC; jj < n; jj += tpr * NC) a.scale[r_begin + jj] = __int_as_float(0x7fc00000);
      break;
    }

    RowQuant q = kA ? make_asym<C::kDivisor, C::kOffsetOptInt>(m0, m1) : make_sym<C::kDivisor>(m0);
    if (!row_valid) {
      q.scale = 0.0f;
      q.offset = 0.0f;
    }
    if (lane_g == 0) {
      __stcs(a.scale + r, q.scale);
      if (kA) __stcs(a.offset + r, q.offset);
    }

    // ---- pass 2: quantize from registers and store
    auto store8 = [&](int k, const uint32_t (&bits)[8]) {
      const int vi = vbase + 32 * k;
      if (OUT == kOutInt8) {
        __stcs(reinterpret_cast<uint2*>(yrow) + vi, pack8_int8(bits));
      } else {
        __stcs(reinterpret_cast<unsigned int*>(yrow) + vi, pack8_int4(bits));
      }
    };
    auto value8 = [&](int k, float (&v)[8]) {
      if (kSmooth) {
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = prod[kSmooth ? k : 0][t];
      } else {
        InTraits<InT>::widen8(raw[k], v);
      }
    };
    if (!row_valid || q.zero_scale) {
      // every code of the row is the same: 0, or offset_opt for a constant
      // asymmetric row (rows past the last group get 0)
      const uint32_t cb = __float_as_uint(__fadd_rn(row_valid ? C::kOffsetOpt : 0.0f, kRoundMagic));
      uint32_t bits[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) bits[t] = cb;
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (in_row(k)) store8(k, bits);
      }
      continue;
    }
    if (q.exact_row) {
      // rare (scale outside [2^-40, 2^100] or a non-finite offset): the IEEE
      // division for every element
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (!in_row(k)) continue;
        float v[8];
        value8(k, v);
        uint32_t bits[8];
        quant8_exact<kA>(v, q, C::kLo, C::kHi, bits);
        store8(k, bits);
      }
      continue;
    }
    auto pass2 = [&](auto clamp_tag) {
      constexpr bool kClamp = decltype(clamp_tag)::value;
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (!in_row(k)) continue;
        float v[8];
        value8(k, v);
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
  // After a failed wait, copies issued for rows that nobody consumed may still
  // be landing: wait (bounded) for every slot's last copy before the CTA's
  // shared memory is released. On the normal path every copy was consumed.
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag != 0u) {
    for (int t = 0; t < NS; ++t) {
      if (issued_round[t] >= 0) mbar_wait_parity(full + t, static_cast<uint32_t>(issued_round[t]) & 1u);
    }
  }
}

}  // namespace dq

namespace dq {

// ============================================================ small inputs

// Few short rows (e.g. 64 rows of 1024 fp16): the ring's per-CTA set-up is not
// amortized, so one warp per row loads its row straight into registers with
// 16-byte read-only loads (lane l holds vectors l + 32k, k < VPT: coalesced),
// reduces it with one warp instruction, derives the row constants and stores
// the codes; no shared memory, no barrier, no wait. Rows are spread one warp
// per CTA over as many SMs as there are rows (grid-strided beyond that).
constexpr int kWarpRowThreads = 32;

template <typename InT, int MODE, int OUT, int SMK, int VPT, bool kRagged>
__global__ void __launch_bounds__(kWarpRowThreads) dynamic_quant_warp_kernel(const RowQuantArgs a) {
  using C = QuantConsts<MODE, OUT>;
  using P = Packed<InT>;
  constexpr bool kA = MODE == kAsym;
  constexpr bool kSmooth = SMK != kSmNone;
  constexpr int kSmoothElem = SMK == kSmF32 ? 4 : 2;
  const int lane = threadIdx.x;
  const int nvec = static_cast<int>(a.cols >> 3);
  auto in_row = [&](int k) { return !kRagged || lane + 32 * k < nvec; };
  // the CTA's first row into L2 while the kernel before finishes (see
  // ring_prefetch.cuh; 64 x 1024 fp16: 2.15 us against 2.33 us per call)
  if (lane == 0 && static_cast<int64_t>(blockIdx.x) < a.rows) {
    bulk_prefetch_l2(static_cast<const uint8_t*>(a.x) + static_cast<int64_t>(blockIdx.x) * a.cols * 2,
                     static_cast<uint32_t>(a.cols * 2));
  }
  pdl_launch_dependents();
  pdl_wait_primary();
  write_group_status(a);
  const bool moe = a.group_index != nullptr;
  const int64_t y_row_bytes = OUT == kOutInt8 ? a.cols : (a.cols >> 1);
  for (int64_t r = blockIdx.x; r < a.rows; r += gridDim.x) {
    const uint4* xrow = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.x) + r * a.cols * 2);
    uint4 raw[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) raw[k] = in_row(k) ? ld_stream_16(xrow + lane + 32 * k) : make_uint4(0, 0, 0, 0);
    bool row_valid = true;
    const uint8_t* smooth_row = static_cast<const uint8_t*>(a.smooth);
    if (moe) {
      const int e = expert_of(a.group_index, a.num_groups, r);
      row_valid = e < a.num_groups;
      smooth_row += static_cast<size_t>(row_valid ? e : 0) * static_cast<size_t>(a.cols) * kSmoothElem;
    }
    float m0, m1;
    float prod[kSmooth ? VPT : 1][8];
    if (kSmooth) {
      float amx = kA ? -INFINITY : 0.0f, amn = INFINITY;
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (in_row(k)) {
          float v[8], sm[8];
          InTraits<InT>::widen8(raw[k], v);
          load_smooth8<SMK>(smooth_row, lane + 32 * k, sm);
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float2 pr = __fmul2_rn(make_float2(v[2 * p], v[2 * p + 1]), make_float2(sm[2 * p], sm[2 * p + 1]));
            prod[kSmooth ? k : 0][2 * p] = pr.x;
            prod[kSmooth ? k : 0][2 * p + 1] = pr.y;
          }
          if (kA) {
            amx = fmaxf(amx, max8(prod[kSmooth ? k : 0]));
            amn = fminf(amn, min8(prod[kSmooth ? k : 0]));
          } else {
            amx = fmaxf(amx, absmax8(prod[kSmooth ? k : 0]));
          }
        }
      }
      m0 = amx;
      m1 = amn;
    } else {
      typename P::T2 hmax = kA ? P::lowest() : P::zero(), hmin = P::highest();
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (in_row(k)) {
          const uint32_t w[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            if (kA) {
              hmax = P::vmax(hmax, P::from_bits(w[t]));
              hmin = P::vmin(hmin, P::from_bits(w[t]));
            } else {
              hmax = P::vmax(hmax, P::from_bits(w[t] & 0x7FFF7FFFu));
            }
          }
        }
      }
      m0 = P::hi_lo_max(hmax);
      m1 = kA ? P::hi_lo_min(hmin) : INFINITY;
    }
    m0 = warp_max(m0);
    if (kA) m1 = warp_min(m1);
    RowQuant q = kA ? make_asym<C::kDivisor, C::kOffsetOptInt>(m0, m1) : make_sym<C::kDivisor>(m0);
    if (!row_valid) {
      q.scale = 0.0f;
      q.offset = 0.0f;
    }
    if (lane == 0) {
      a.scale[r] = q.scale;
      if (kA) a.offset[r] = q.offset;
    }
    uint8_t* yrow = static_cast<uint8_t*>(a.y) + r * y_row_bytes;
    auto store8 = [&](int k, const uint32_t (&bits)[8]) {
      const int vi = lane + 32 * k;
      if (OUT == kOutInt8) {
        reinterpret_cast<uint2*>(yrow)[vi] = pack8_int8(bits);
      } else {
        reinterpret_cast<unsigned int*>(yrow)[vi] = pack8_int4(bits);
      }
    };
    auto value8 = [&](int k, float (&v)[8]) {
      if (kSmooth) {
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = prod[kSmooth ? k : 0][t];
      } else {
        InTraits<InT>::widen8(raw[k], v);
      }
    };
    if (!row_valid || q.zero_scale) {
      const uint32_t cb = __float_as_uint(__fadd_rn(row_valid ? C::kOffsetOpt : 0.0f, kRoundMagic));
      uint32_t bits[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) bits[t] = cb;
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (in_row(k)) store8(k, bits);
      }
      continue;
    }
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      if (!in_row(k)) continue;
      float v[8];
      value8(k, v);
      uint32_t bits[8];
      if (q.exact_row) {
        quant8_exact<kA>(v, q, C::kLo, C::kHi, bits);
      } else if (kA && q.clamp) {
        quant8<kA, true>(v, q, C::kLo, C::kHi, bits);
      } else {
        quant8<kA, false>(v, q, C::kLo, C::kHi, bits);
      }
      store8(k, bits);
    }
  }
}

}  // namespace dq
