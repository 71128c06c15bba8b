// Fused AdaLayerNorm + symmetric INT8 dynamic quantization
// (aclnnAdaLayerNormQuant, "Formula" steps 1-5), sm_100a.
//
// Two launches per call:
//   1. ada_affine_table_kernel folds the per-(batch, column) parameters of
//      steps 1-3 into a table in the caller's workspace,
//        A[b][c] = (w[c] * (1 + scale[b][c])) * smooth[c]
//        B[b][c] = ((bias[c] * (1 + scale[b][c])) + shift[b][c]) * smooth[c]
//      (absent weight = 1, bias = 0, smooth = 1), so steps 1-3 become one FMA
//      per element, y = n * A + B. The table is batch x hidden x 8 bytes and
//      is read through L1/L2 by the main kernel.
//   2. ada_layernorm_quant_tma_kernel streams rows through the bulk-copy (TMA)
//      ring (tma_pipeline.cuh) and keeps each thread's share of the row in
//      registers between its passes. It is launched as a programmatic
//      dependent of the table kernel: it sets up its ring and starts copying
//      rows while the table is still being written, and waits for the table
//      (griddepcontrol.wait) just before first reading it. The table kernel
//      is itself a programmatic dependent of the work before it and releases
//      the row kernel only after that work has completed.
//
// Arithmetic:
//   * E(x), Var(x) from one row reduction: each thread sums d = x - K and d^2
//     over its share, with K the mean of the row's first 8 elements (the same
//     value in every thread; d is exact when x and K are within a factor 2,
//     as on rows whose mean is far above their spread). Partial sums are fp32,
//     the sums across warps double; E(x) = K + E(d), Var = E(d^2) - E(d)^2.
//     While E(d)^2 <= 3/4 E(d^2) that difference loses at most a factor 4 of
//     relative accuracy. Rows past the bound (first elements far from the
//     mean) take a centred second pass about RN(E(x)). E(x) is rounded to
//     fp32 once, as the formula's mean is.
//   * n = (x - E(x)) * rstd with rstd = RN(1 / RN(sqrt(Var + eps))), as
//     fma(d, rstd, -(E(x) - K) * rstd), then y = n * A + B. Against a
//     sequential evaluation that rounds every printed operation separately
//     and divides by the square root, this moves y by a few ulps:
//     quant_scale stays within a relative 1e-6 and about one code in 10^6
//     moves by one.
//   * steps 4-5 are the DynamicQuant quantizer (exact IEEE semantics).
#pragma once

#include "dq_args.cuh"
#include "dq_device.cuh"
#include "tma_pipeline.cuh"

namespace dq {

__host__ __device__ inline size_t ada_smem_bytes(int groups, int stages, uint32_t stride) {
  return static_cast<size_t>(groups) * stages * stride + static_cast<size_t>(groups) * stages * 8;
}

// ============================================================ affine table

constexpr int kTableBlock = 256;

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
    const int64_t c = idx % H;
    const float onep = __fadd_rn(1.0f, load_param(a.ada_scale, a.param_dtype, idx));
    const float w = a.weight ? load_param(a.weight, a.param_dtype, c) : 1.0f;
    const float bs = a.bias ? load_param(a.bias, a.param_dtype, c) : 0.0f;
    const float sm = a.smooth ? load_param(a.smooth, a.param_dtype, c) : 1.0f;
    const float sh = load_param(a.ada_shift, a.param_dtype, idx);
    a.table[idx] = __fmul_rn(__fmul_rn(w, onep), sm);
    a.table[total + idx] = __fmul_rn(__fadd_rn(__fmul_rn(bs, onep), sh), sm);
  }
}

// Rows whose quant_scale is below 2^-40 (RowQuant::exact_row): every element
// of this thread's share with the IEEE division, out of line. y is recomputed
// from the row still resident in shared memory with the main loop's
// arithmetic (widen, - mean, * rstd, * A + B).
template <typename InT>
__device__ __noinline__ void ada_quantize_row_exact(const uint4* srow, const float4* A4, const float4* B4,
                                                    float mean_f, float rstd, RowQuant q, int lane_g, int tpr,
                                                    int nvec, int8_t* orow) {
  for (int vi = lane_g; vi < nvec; vi += tpr) {
    float v[8];
    InTraits<InT>::widen8(srow[vi], v);
    const float4 a0 = A4[2 * vi], a1 = A4[2 * vi + 1], b0 = B4[2 * vi], b1 = B4[2 * vi + 1];
    const float Av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float Bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[j] = __fmaf_rn(__fmul_rn(__fadd_rn(v[j], -mean_f), rstd), Av[j], Bv[j]);
    }
    uint32_t bits[8];
    quant8_exact<false>(v, q, -127.0f, 127.0f, bits);
    reinterpret_cast<uint2*>(orow)[vi] = pack8_int8(bits);
  }
}

// ============================================================ bulk-copy kernel

#ifndef DQ_ADA_MAX_BLOCK
#define DQ_ADA_MAX_BLOCK 512
#endif
constexpr int kAdaMaxBlock = DQ_ADA_MAX_BLOCK;
#ifndef DQ_ADA_MAX_REGS
#define DQ_ADA_MAX_REGS 128  // the row share stays in registers across four passes
#endif

// Warp w of a row group owns the contiguous chunk of 32 * VPT vectors starting
// at w * 32 * VPT; lane l owns vectors chunk + l + 32 * k (k < VPT), so every
// per-k offset is a compile-time constant. kRagged: the row is not exactly
// G * 32 * VPT vectors, so vectors past the row end are skipped.
template <typename InT, int VPT, bool kRagged>
__global__ void __maxnreg__(DQ_ADA_MAX_REGS)
ada_layernorm_quant_tma_kernel(const AdaArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ double red_d[2][3][kAdaMaxBlock / 32];  // [parity][sum|sq|centred sq][warp]
  __shared__ float red_f[2][kAdaMaxBlock / 32];       // [parity][warp] absmax

  const int tpr = a.tpr;
  const int S = a.stages;
  const int g = threadIdx.x / tpr;
  const int lane_g = threadIdx.x - g * tpr;
  const int warp = threadIdx.x >> 5;
  const int warp_g0 = (g * tpr) >> 5;
  const int nwarps_g = tpr >> 5;
  const int lane = threadIdx.x & 31;
  const int vbase = (lane_g >> 5) * (32 * VPT) + lane;  // this thread's vector k is vbase + 32 * k
  const uint32_t stride = a.stage_stride;
  const size_t ring_bytes = static_cast<size_t>(a.groups) * S * stride;
  uint8_t* ring = smem + static_cast<size_t>(g) * S * stride;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ring_bytes) + g * S;

  if (threadIdx.x == 0) {
    uint64_t* all = reinterpret_cast<uint64_t*>(smem + ring_bytes);
    for (int i = 0; i < a.groups * S; ++i) mbar_init(all + i, 1);
    fence_mbarrier_init();
  }
  __syncthreads();

  const int64_t rows = a.batch * a.seq;
  const int64_t workers = static_cast<int64_t>(gridDim.x) * a.groups;
  const int64_t worker = static_cast<int64_t>(blockIdx.x) * a.groups + g;
  const int64_t r_begin = worker * rows / workers;
  const int64_t r_end = (worker + 1) * rows / workers;
  const int64_t n = r_end - r_begin;
  if (n <= 0) {
    pdl_wait_primary();
    return;
  }

  const int64_t H = a.hidden;
  const int nvec = static_cast<int>(H >> 3);
  const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
  const bool leader = lane_g == 0;
  const uint64_t policy = leader ? l2_evict_first_policy() : 0;
  const uint8_t* x_next = static_cast<const uint8_t*>(a.x) + r_begin * static_cast<int64_t>(row_bytes);
  int64_t issued = 0;
  int p_stage = 0;
  auto issue_next = [&]() {
    mbar_arrive_expect_tx(bars + p_stage, row_bytes);
    bulk_copy_g2s(ring + static_cast<size_t>(p_stage) * stride, x_next, row_bytes, bars + p_stage, policy);
    x_next += row_bytes;
    ++issued;
    p_stage = p_stage + 1 == S ? 0 : p_stage + 1;
  };
  if (leader) {
    while (issued < n && issued < S - 1) issue_next();
  }
  auto in_row = [&](int k) { return !kRagged || vbase + 32 * k < nvec; };

  pdl_wait_primary();  // the affine table is complete and visible from here on

  // batch of the current row, tracked without division
  int64_t b = r_begin / a.seq;
  int64_t b_end = (b + 1) * a.seq;
  const float4* A4 = reinterpret_cast<const float4*>(a.table + b * H) + 2 * vbase;
  const float4* B4 = reinterpret_cast<const float4*>(a.table + a.batch * H + b * H) + 2 * vbase;
  const int64_t table_b_stride4 = H / 4;
  int8_t* orow = a.out + r_begin * H;

  int c_stage = 0;
  uint32_t phase = 0;
  int parity = 0;
  for (int64_t r = r_begin; r < r_end; ++r, orow += H) {
    if (r >= b_end) {
      ++b;
      b_end += a.seq;
      A4 += table_b_stride4;
      B4 += table_b_stride4;
    }
    const bool arrived = mbar_wait_parity(bars + c_stage, phase);
    const uint4* srow = reinterpret_cast<const uint4*>(ring + static_cast<size_t>(c_stage) * stride);

    // ---- pass 1: load, widen, shift by K, both moments of d = x - K
    // K is the mean of the row's first 8 elements, the same value in every
    // thread. E(d) and E(d^2) come out of one reduction; Var = E(d^2) - E(d)^2
    // loses at most a factor 4 of relative accuracy while E(d)^2 <= 3/4 E(d^2),
    // and rows past that bound take a centred second pass.
    constexpr int NACC = VPT < 4 ? VPT : 4;  // independent accumulators: short dependency chains
    float K;
    {
      float f[8];
      InTraits<InT>::widen8(srow[0], f);
      K = __fmul_rn(__fadd_rn(__fadd_rn(__fadd_rn(f[0], f[1]), __fadd_rn(f[2], f[3])),
                              __fadd_rn(__fadd_rn(f[4], f[5]), __fadd_rn(f[6], f[7]))),
                    0.125f);
    }
    float v[VPT][8];
    float2 acc[NACC], acq[NACC];
#pragma unroll
    for (int j = 0; j < NACC; ++j) acc[j] = acq[j] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const bool active = in_row(k);
      InTraits<InT>::widen8(active ? srow[vbase + 32 * k] : make_uint4(0, 0, 0, 0), v[k]);
      float2 d[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        d[p] = __fadd2_rn(make_float2(v[k][2 * p], v[k][2 * p + 1]), f2(-K));
        if (kRagged && !active) d[p] = make_float2(0.0f, 0.0f);
        v[k][2 * p] = d[p].x;
        v[k][2 * p + 1] = d[p].y;
        acq[(k + p) % NACC] = __ffma2_rn(d[p], d[p], acq[(k + p) % NACC]);
      }
      acc[k % NACC] = __fadd2_rn(acc[k % NACC], __fadd2_rn(__fadd2_rn(d[0], d[1]), __fadd2_rn(d[2], d[3])));
    }
#pragma unroll
    for (int j = 1; j < NACC; ++j) {
      acc[0] = __fadd2_rn(acc[0], acc[j]);
      acq[0] = __fadd2_rn(acq[0], acq[j]);
    }
    // butterflies: every lane ends with the same bits (each step adds the
    // same two operands on both lanes of a pair)
    float s1 = __fadd_rn(acc[0].x, acc[0].y), s2 = __fadd_rn(acq[0].x, acq[0].y);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s1 = __fadd_rn(s1, __shfl_xor_sync(0xffffffffu, s1, o));
      s2 = __fadd_rn(s2, __shfl_xor_sync(0xffffffffu, s2, o));
    }
    double sum = s1, sq = s2;
    bool failed;
    if (nwarps_g > 1) {
      if (lane == 0) {
        red_d[parity][0][warp] = sum;
        red_d[parity][1][warp] = sq;
      }
      failed = group_barrier_or(1 + g, tpr, !arrived);
      sum = 0.0;
      sq = 0.0;
      for (int w = 0; w < nwarps_g; ++w) {
        sum += red_d[parity][0][warp_g0 + w];
        sq += red_d[parity][1][warp_g0 + w];
      }
    } else {
      failed = __any_sync(0xffffffffu, !arrived);
      __syncwarp();
    }
    if (failed) {
      for (int64_t rr = r + lane_g; rr < r_end; rr += tpr) a.quant_scale[rr] = __int_as_float(0x7fc00000);
      if (leader) {
        int st = c_stage;
        uint32_t ph = phase;
        for (int64_t j = r - r_begin + 1; j < issued; ++j) {
          st = st + 1 == S ? 0 : st + 1;
          if (st == 0) ph ^= 1u;
          mbar_wait_parity(bars + st, ph);
        }
      }
      return;
    }
    // refill the stage of the previous row (S - 1 copies stay in flight; the
    // current row's stage is kept for the out-of-line exact path)
    if (leader && issued < n) {
      fence_proxy_async_smem();
      issue_next();
    }
    c_stage = c_stage + 1 == S ? 0 : c_stage + 1;
    if (c_stage == 0) phase ^= 1u;
    const double m1 = sum * a.inv_hidden;  // E(d)
    const double m2 = sq * a.inv_hidden;   // E(d^2)
    const double mean_d = static_cast<double>(K) + m1;
    const float mean_f = __double2float_rn(mean_d);
    const float c_f = __fsub_rn(mean_f, K);  // mean_f - K (exact when K and mean_f are within a factor 2)
    double var_d;
    if (m1 * m1 <= 0.75 * m2) {
      var_d = m2 - m1 * m1;
    } else {
      // ---- centred second pass (rows whose first elements sit far from the mean)
#pragma unroll
      for (int j = 0; j < NACC; ++j) acq[j] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        const bool active = in_row(k);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float2 e = __fadd2_rn(make_float2(v[k][2 * p], v[k][2 * p + 1]), f2(-c_f));
          if (kRagged && !active) e = make_float2(0.0f, 0.0f);
          acq[(k + p) % NACC] = __ffma2_rn(e, e, acq[(k + p) % NACC]);
        }
      }
#pragma unroll
      for (int j = 1; j < NACC; ++j) acq[0] = __fadd2_rn(acq[0], acq[j]);
      double sc = warp_sum(static_cast<double>(acq[0].x) + static_cast<double>(acq[0].y));
      if (nwarps_g > 1) {
        if (lane == 0) red_d[parity][2][warp] = sc;
        group_barrier(1 + g, tpr);
        sc = 0.0;
        for (int w = 0; w < nwarps_g; ++w) sc += red_d[parity][2][warp_g0 + w];
      }
      const double dm = m1 - static_cast<double>(c_f);
      var_d = sc * a.inv_hidden - dm * dm;
    }
    var_d = var_d > 0.0 ? var_d : 0.0;
    const float var_f = __double2float_rn(var_d);
    const float rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(var_f, a.epsilon)));
    // n = (x - mean_f) * rstd = fma(d, rstd, -(mean_f - K) * rstd)
    const float nb = -__fmul_rn(c_f, rstd);
    // ---- pass 3: y = n * A + B, absmax
    float amx[NACC];
#pragma unroll
    for (int j = 0; j < NACC; ++j) amx[j] = 0.0f;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      if (in_row(k)) {
        const float4 a0 = __ldg(A4 + 64 * k), a1 = __ldg(A4 + 64 * k + 1);
        const float4 b0 = __ldg(B4 + 64 * k), b1 = __ldg(B4 + 64 * k + 1);
        const float Av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float Bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 nn = __ffma2_rn(make_float2(v[k][2 * p], v[k][2 * p + 1]), f2(rstd), f2(nb));
          const float2 y =
              __ffma2_rn(nn, make_float2(Av[2 * p], Av[2 * p + 1]), make_float2(Bv[2 * p], Bv[2 * p + 1]));
          v[k][2 * p] = y.x;
          v[k][2 * p + 1] = y.y;
        }
        amx[k % NACC] = fmaxf(amx[k % NACC], absmax8(v[k]));
      }
    }
    float amax = warp_max(tree<NACC, true>(amx));
    if (nwarps_g > 1) {
      if (lane == 0) red_f[parity][warp] = amax;
      group_barrier(1 + g, tpr);
      // lane j takes warp j's partial; one more warp reduction combines them
      amax = warp_max(lane < nwarps_g ? red_f[parity][warp_g0 + lane] : 0.0f);
      parity ^= 1;
    }

    // ---- steps 4-5
    const RowQuant q = make_sym<127>(amax);
    if (lane_g == 0) __stcs(a.quant_scale + r, q.scale);
    if (q.exact_row) {
      ada_quantize_row_exact<InT>(srow, A4 - 2 * vbase, B4 - 2 * vbase, mean_f, rstd, q, lane_g, tpr, nvec, orow);
      continue;
    }
    uint2* ov = reinterpret_cast<uint2*>(orow) + vbase;
    if (q.zero_scale) {
      const uint2 zeros = make_uint2(0u, 0u);
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (in_row(k)) __stcs(ov + 32 * k, zeros);
      }
      continue;
    }
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      if (!in_row(k)) continue;
      uint32_t bits[8];
      quant8<false, false>(v[k], q, -127.0f, 127.0f, bits);
      __stcs(ov + 32 * k, pack8_int8(bits));
    }
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
