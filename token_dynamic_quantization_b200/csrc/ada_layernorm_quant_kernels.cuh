// Fused AdaLayerNorm + symmetric INT8 dynamic quantization
// (aclnnAdaLayerNormQuant, "Formula" steps 1-5), sm_100a.
//
// One HBM read of x and one write of the codes per row; everything between
// stays in registers. The statistics are exact-as-possible rather than
// Welford: the row is resident, so a two-pass mean / centred variance costs
// no extra traffic. Per-thread partial sums are fp32, the cross-thread sums
// double; the variance is corrected to the double mean:
//   sum (v - m_d)^2 = sum (v - m_f)^2 - H (m_d - m_f)^2,
// so E(x) and Var(x) agree with a double-precision evaluation rounded to
// fp32 except for the last bit in rare rows. x - E(x) is multiplied by the
// correctly rounded 1/sqrt(Var + eps) instead of divided by the square root
// (the only other departure from a sequential fp32 evaluation); steps 2-3 are
// one IEEE operation each in the order the formula prints them, and steps 4-5
// are the exact DynamicQuant quantizer.
#pragma once

#include "dq_device.cuh"

namespace dq {

struct AdaArgs {
  const void* x;
  int64_t batch, seq, hidden;
  const void* ada_scale;  // [batch, hidden]
  const void* ada_shift;  // [batch, hidden]
  const void* weight;     // [hidden] or nullptr
  const void* bias;       // [hidden] or nullptr
  const void* smooth;     // [hidden] or nullptr
  int param_dtype;
  float epsilon;
  int8_t* out;
  float* quant_scale;
  int tpr;
  int groups;
};

// ============================================================ vector kernel

constexpr int kAdaMaxBlock = 512;

template <typename InT>
__global__ void __launch_bounds__(kAdaMaxBlock)
ada_layernorm_quant_vec_kernel(const AdaArgs a) {
  __shared__ double red_d[2][2][kAdaMaxBlock / 32];  // [parity][sum|sq][warp]
  __shared__ float red_f[2][kAdaMaxBlock / 32];       // [parity][warp] absmax

  const int tpr = a.tpr;
  const int g = threadIdx.x / tpr;
  const int lane_g = threadIdx.x - g * tpr;
  const int warp = threadIdx.x >> 5;
  const int warp_g0 = (g * tpr) >> 5;
  const int nwarps_g = tpr >> 5;
  const int lane = threadIdx.x & 31;

  const int64_t rows = a.batch * a.seq;
  const int64_t workers = static_cast<int64_t>(gridDim.x) * a.groups;
  const int64_t worker = static_cast<int64_t>(blockIdx.x) * a.groups + g;
  const int64_t r_begin = worker * rows / workers;
  const int64_t r_end = (worker + 1) * rows / workers;
  if (r_begin >= r_end) return;

  const int64_t nvec = a.hidden >> 3;
  const bool active = lane_g < nvec;  // one 8-element vector per thread
  const int64_t col0 = static_cast<int64_t>(lane_g) * 8;
  const double hd = static_cast<double>(a.hidden);

  // per-column parameters (fp32, exact widening)
  float w[8], bs[8], sm[8], onep[8], sh[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    w[j] = (active && a.weight) ? load_param(a.weight, a.param_dtype, col0 + j) : 1.0f;
    bs[j] = (active && a.bias) ? load_param(a.bias, a.param_dtype, col0 + j) : 0.0f;
    sm[j] = (active && a.smooth) ? load_param(a.smooth, a.param_dtype, col0 + j) : 1.0f;
  }
  int64_t cur_b = -1;

  const uint4* __restrict__ xv = static_cast<const uint4*>(a.x);
  uint4 buf0 = make_uint4(0, 0, 0, 0), buf1 = buf0, buf2 = buf0;
  if (active) buf0 = __ldcs(xv + r_begin * nvec + lane_g);
  if (active && r_begin + 1 < r_end) buf1 = __ldcs(xv + (r_begin + 1) * nvec + lane_g);

  int parity = 0;
  for (int64_t r = r_begin; r < r_end; ++r) {
    if (active && r + 2 < r_end) buf2 = __ldcs(xv + (r + 2) * nvec + lane_g);

    const int64_t b = r / a.seq;
    if (b != cur_b) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        onep[j] = active ? __fadd_rn(1.0f, load_param(a.ada_scale, a.param_dtype, b * a.hidden + col0 + j)) : 1.0f;
        sh[j] = active ? load_param(a.ada_shift, a.param_dtype, b * a.hidden + col0 + j) : 0.0f;
      }
      cur_b = b;
    }

    float v[8];
    InTraits<InT>::widen8(buf0, v);
    // ---- E(x)
    float s1 = 0.0f;
    if (active) {
#pragma unroll
      for (int j = 0; j < 8; ++j) s1 = __fadd_rn(s1, v[j]);
    }
    double sum = warp_sum(static_cast<double>(s1));
    if (nwarps_g > 1) {
      if (lane == 0) red_d[parity][0][warp] = sum;
      group_barrier(1 + g, tpr);
      sum = 0.0;
      for (int i = 0; i < nwarps_g; ++i) sum += red_d[parity][0][warp_g0 + i];
    }
    const double mean_d = sum / hd;
    const float mean_f = __double2float_rn(mean_d);
    // ---- Var(x), biased, about the double mean
    float d[8];
    float s2 = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      d[j] = __fsub_rn(v[j], mean_f);
      if (active) s2 = __fmaf_rn(d[j], d[j], s2);
    }
    double sq = warp_sum(static_cast<double>(s2));
    if (nwarps_g > 1) {
      if (lane == 0) red_d[parity][1][warp] = sq;
      group_barrier(1 + g, tpr);
      sq = 0.0;
      for (int i = 0; i < nwarps_g; ++i) sq += red_d[parity][1][warp_g0 + i];
    }
    const double dm = mean_d - static_cast<double>(mean_f);
    double var_d = sq / hd - dm * dm;
    var_d = var_d > 0.0 ? var_d : 0.0;
    const float var_f = __double2float_rn(var_d);
    const float rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(var_f, a.epsilon)));

    // ---- steps 1-3, then absmax
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float t = __fmul_rn(d[j], rstd);
      t = __fmul_rn(t, w[j]);
      t = __fadd_rn(t, bs[j]);
      t = __fmul_rn(t, onep[j]);
      t = __fadd_rn(t, sh[j]);
      t = __fmul_rn(t, sm[j]);
      v[j] = t;
      if (active) amax = fmaxf(amax, fabsf(t));
    }
    amax = warp_max(amax);
    if (nwarps_g > 1) {
      if (lane == 0) red_f[parity][warp] = amax;
      group_barrier(1 + g, tpr);
      amax = red_f[parity][warp_g0];
      for (int i = 1; i < nwarps_g; ++i) amax = fmaxf(amax, red_f[parity][warp_g0 + i]);
    }
    parity ^= 1;

    // ---- steps 4-5
    const RowQuant q = make_sym(amax, 127.0f);
    if (lane_g == 0) __stcs(a.quant_scale + r, q.scale);
    if (active) {
      float c[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) c[j] = q.zero_scale ? 0.0f : sym_code(v[j], q, -127.0f, 127.0f);
      uint2* op = reinterpret_cast<uint2*>(a.out + r * a.hidden) + lane_g;
      __stcs(op, pack_int8x8(c));
    }

    buf0 = buf1;
    buf1 = buf2;
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
    const double mean_d = block_sum(s1) / static_cast<double>(H);
    const float mean_f = __double2float_rn(mean_d);
    double s2 = 0.0;
    for (int64_t c = threadIdx.x; c < H; c += kAdaGenericBlock) {
      const double dd = static_cast<double>(InTraits<InT>::widen1(a.x, base + c)) - mean_d;
      s2 += dd * dd;
    }
    const float var_f = __double2float_rn(block_sum(s2) / static_cast<double>(H));
    const float rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(var_f, a.epsilon)));

    auto value = [&](int64_t c) {
      float t = __fmul_rn(__fsub_rn(InTraits<InT>::widen1(a.x, base + c), mean_f), rstd);
      if (a.weight) t = __fmul_rn(t, load_param(a.weight, a.param_dtype, c));
      if (a.bias) t = __fadd_rn(t, load_param(a.bias, a.param_dtype, c));
      t = __fmul_rn(t, __fadd_rn(1.0f, load_param(a.ada_scale, a.param_dtype, b * H + c)));
      t = __fadd_rn(t, load_param(a.ada_shift, a.param_dtype, b * H + c));
      if (a.smooth) t = __fmul_rn(t, load_param(a.smooth, a.param_dtype, c));
      return t;
    };
    float amax = 0.0f;
    for (int64_t c = threadIdx.x; c < H; c += kAdaGenericBlock) amax = fmaxf(amax, fabsf(value(c)));
    amax = warp_max(amax);
    if (lane == 0) red_f[warp] = amax;
    __syncthreads();
    amax = red_f[0];
    for (int i = 1; i < kWarps; ++i) amax = fmaxf(amax, red_f[i]);
    __syncthreads();
    const RowQuant q = make_sym(amax, 127.0f);
    if (threadIdx.x == 0) a.quant_scale[r] = q.scale;
    for (int64_t c = threadIdx.x; c < H; c += kAdaGenericBlock) {
      const float code = q.zero_scale ? 0.0f : sym_code(value(c), q, -127.0f, 127.0f);
      a.out[base + c] = static_cast<int8_t>(__float2int_rn(code));
    }
  }
}

}  // namespace dq
