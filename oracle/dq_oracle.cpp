// Plain single-threaded CPU oracle for per-token dynamic quantization.
//
// TEST INFRASTRUCTURE ONLY. This file is the independent reference that the
// CUDA path is checked against. Only the test suite, the smoke check and the
// benchmark's CPU-baseline leg may load it; the product path never does.
// It shares no code, header, table or helper with the CUDA library.
//
// What it computes, and where the pages define it:
//   * aclnnDynamicQuantV2, "Formula": symmetric quantization
//       scaleOut = row_max(abs(input)) / 127,  yOut = round(input / scaleOut)
//     and asymmetric quantization
//       scaleOut = (row_max(input) - row_min(input)) / scale_opt
//       offset   = offset_opt - row_max(input) / scaleOut
//       yOut     = round(input / scaleOut + offset)
//     where input = x * smoothScalesOptional when smooth scales are given,
//     and (scale_opt, offset_opt) = (255, 127) for INT8, (15, 7) for INT4/INT32.
//   * aclnnDynamicQuantV2, "Description": in the MoE case each expert has its
//     own smooth-scale row, selected through groupIndexOptional.
//   * aclnnDynamicQuantV2, "Constraints": INT4 output needs an even last dim,
//     INT32 output (eight int4 codes per int32) a last dim divisible by 8.
//   * aclnnAdaLayerNormQuant, "Formula" steps 1-5: LayerNorm with optional
//     weight/bias, y = LN * (1 + scale) + shift, optional smooth scales, then
//     symmetric INT8 dynamic quantization of y.
//
// Readings where the pages are silent (each one is listed in the design notes):
//   * arithmetic is IEEE-754 binary32 with round-to-nearest-even, one rounding
//     per written operation, no fused multiply-add (built with
//     -ffp-contract=off), true division (never x * (1/scale));
//   * "round" is round-half-to-even (std::nearbyint in FE_TONEAREST mode);
//   * codes saturate to the output range: symmetric INT8 [-127, 127],
//     symmetric INT4 [-7, 7], asymmetric INT8 [-128, 127], asymmetric INT4
//     [-8, 7] (saturation only removes rounding noise for finite inputs);
//   * symmetric quantization to INT4/INT32 divides by 7 (= offset_opt of the
//     4-bit type) rather than 127, since 127 cannot be held in four bits.
//     The pages fix no value here: parity unpinned for that case (the tests
//     pin the arithmetic given the divisor, not the divisor itself);
//   * a symmetric row whose absmax is 0 gets scale 0 and all codes 0; an
//     asymmetric row whose max equals its min gets scale 0, offset offset_opt
//     and all codes offset_opt (the row max maps to offset_opt, as the
//     asymmetric formula gives for any non-constant row);
//   * group_index holds, per expert, the cumulative END row (exclusive) of
//     that expert's rows; expert(r) = the smallest e with r < group_index[e];
//     a row at or past group_index[E-1] is an error here;
//   * packed INT4: element 2j goes to bits 0-3 and element 2j+1 to bits 4-7 of
//     byte j (two's-complement nibbles); INT32: element 8j+k goes to bits
//     4k..4k+3 of word j;
//   * AntiQuantize, PER_TOKEN policy (one scale and offset per row): the
//     formula was lost from the page; the dequantizer is read as the inverse
//     of the quantizer above, out = (code - offset) * scale in binary32, then
//     rounded once to the output type (round to nearest even). Only the
//     page's printed example (scale 1, offset 0: output = input) pins it
//     directly; the sign of the offset is parity unpinned by the pages (the
//     tests pin it against the quantizer, whose inverse it is read to be);
//   * AntiQuantize, PER_GROUP policy: every groupSize elements along the k
//     axis (kDim 1: along a row; kDim 0: down a column) share one scale and
//     offset of a [rows, ceil(cols/g)] or [ceil(rows/g), cols] table (the
//     page's shapes); the value is the PER_TOKEN reading with that element's
//     scale and offset (the page's formula images were lost here too);
//   * aclnnQuantBatchMatmulInplaceAdd, "计算公式" (T-T form): the quantized
//     product sum_k x1[m,k] x2[k,n] times (scale1 * scale2), plus y; read
//     with scale1 per row (per token, as the quantizer produces it) and
//     scale2 per output column (per channel), the product of the two scales
//     taken first as printed, then the multiply, then the optional add, each
//     rounded once in binary32 (the integer sum is exact);
//   * AdaLayerNormQuant: the mean and the biased variance (divide by H) are
//     accumulated in double over the fp32-widened row and rounded to float
//     once; epsilon is added inside the square root; x - E(x) is divided by
//     sqrt(Var(x) + epsilon) (a true division, as the formula prints it); every
//     later step is one fp32 operation rounded separately.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC.

#include "dq_oracle.h"

#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ---- widening of the storage types to binary32 (exact) -------------------

// IEEE-754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
float half_bits_to_float(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int exponent = (h >> 10) & 0x1F;
  const int fraction = h & 0x3FF;
  float magnitude;
  if (exponent == 0) {
    // subnormal (or zero): fraction * 2^-24
    magnitude = std::ldexp(static_cast<float>(fraction), -24);
  } else if (exponent == 31) {
    magnitude = fraction == 0 ? INFINITY : NAN;
  } else {
    // normal: (1024 + fraction) * 2^(exponent - 15 - 10)
    magnitude = std::ldexp(static_cast<float>(1024 + fraction), exponent - 25);
  }
  return sign ? -magnitude : magnitude;
}

// bfloat16 is the upper half of a binary32 bit pattern.
float bfloat16_bits_to_float(uint16_t b) {
  const uint32_t bits = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return f;
}

float load_element(const void* base, int dtype, int64_t index) {
  switch (dtype) {
    case ORACLE_F32:
      return static_cast<const float*>(base)[index];
    case ORACLE_F16:
      return half_bits_to_float(static_cast<const uint16_t*>(base)[index]);
    case ORACLE_BF16:
      return bfloat16_bits_to_float(static_cast<const uint16_t*>(base)[index]);
    default:
      return NAN;
  }
}

// ---- narrowing of binary32 to the 16-bit storage types (round to nearest even)

// A finite value v > 0 with 2^e <= v < 2^(e+1) is written with `fraction_bits`
// bits after the leading one: scaling by 2^(fraction_bits - e) makes the
// significand an integer in [2^fraction_bits, 2^(fraction_bits+1)) plus a
// fraction, which nearbyint rounds to nearest even (exact scaling by powers of
// two in double). Below the smallest normal exponent the spacing stays fixed
// (subnormals). Returns the rounded significand and updates e.
double round_significand(double v, int fraction_bits, int min_exponent, int* e) {
  int exp2;
  std::frexp(v, &exp2);  // v = m * 2^exp2, m in [0.5, 1)
  int ee = exp2 - 1;     // 2^ee <= v < 2^(ee+1)
  if (ee < min_exponent) ee = min_exponent;  // subnormal: fixed spacing 2^(min_exponent - fraction_bits)
  double q = std::nearbyint(std::ldexp(v, fraction_bits - ee));
  if (q >= std::ldexp(1.0, fraction_bits + 1)) {  // rounded up into the next binade
    q = std::ldexp(1.0, fraction_bits);
    ++ee;
  }
  *e = ee;
  return q;
}

uint16_t narrow_to_half(float f) {
  uint32_t x;
  std::memcpy(&x, &f, sizeof x);
  const uint16_t sign = static_cast<uint16_t>((x >> 16) & 0x8000u);
  if (std::isnan(f)) return static_cast<uint16_t>(sign | 0x7E00u);
  if (std::isinf(f)) return static_cast<uint16_t>(sign | 0x7C00u);
  const double v = std::fabs(static_cast<double>(f));
  if (v == 0.0) return sign;
  int e;
  const double q = round_significand(v, 10, -14, &e);  // binary16: 10 fraction bits, exponents -14..15
  if (e > 15) return static_cast<uint16_t>(sign | 0x7C00u);  // overflow: infinity
  const uint32_t sig = static_cast<uint32_t>(q);
  if (sig < 1024u) return static_cast<uint16_t>(sign | sig);  // subnormal (e == -14, no leading one)
  return static_cast<uint16_t>(sign | (static_cast<uint32_t>(e + 15) << 10) | (sig - 1024u));
}

uint16_t narrow_to_bfloat16(float f) {
  uint32_t x;
  std::memcpy(&x, &f, sizeof x);
  const uint16_t sign = static_cast<uint16_t>((x >> 16) & 0x8000u);
  if (std::isnan(f)) return static_cast<uint16_t>(sign | 0x7FC0u);
  if (std::isinf(f)) return static_cast<uint16_t>(sign | 0x7F80u);
  const double v = std::fabs(static_cast<double>(f));
  if (v == 0.0) return sign;
  int e;
  const double q = round_significand(v, 7, -126, &e);  // bfloat16: 7 fraction bits, exponents -126..127
  if (e > 127) return static_cast<uint16_t>(sign | 0x7F80u);
  const uint32_t sig = static_cast<uint32_t>(q);
  if (sig < 128u) return static_cast<uint16_t>(sign | sig);
  return static_cast<uint16_t>(sign | (static_cast<uint32_t>(e + 127) << 7) | (sig - 128u));
}

// Signed code c of a container (ORACLE_Y_*): int8, or 4-bit two's complement
// with element 2j in the low nibble of byte j (INT32 words hold the same bytes).
int load_code(const void* y, int y_dtype, int64_t index) {
  if (y_dtype == ORACLE_Y_INT8) return static_cast<const int8_t*>(y)[index];
  const uint8_t byte = static_cast<const uint8_t*>(y)[index / 2];
  const int nibble = (index % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
  return nibble >= 8 ? nibble - 16 : nibble;
}

bool is_float_dtype(int dtype) {
  return dtype == ORACLE_F32 || dtype == ORACLE_F16 || dtype == ORACLE_BF16;
}

// ---- the quantization constants (aclnnDynamicQuantV2, Formula note) ------

struct QuantRange {
  float divisor;   // symmetric: 127 or 7; asymmetric: scale_opt (255 or 15)
  float offset_opt;
  int lo, hi;      // saturation bounds of the code
};

QuantRange range_for(int mode, int y_dtype) {
  const bool four_bit = (y_dtype == ORACLE_Y_INT4X2 || y_dtype == ORACLE_Y_INT32);
  if (mode == ORACLE_SYMMETRIC) {
    return four_bit ? QuantRange{7.0f, 0.0f, -7, 7} : QuantRange{127.0f, 0.0f, -127, 127};
  }
  return four_bit ? QuantRange{15.0f, 7.0f, -8, 7} : QuantRange{255.0f, 127.0f, -128, 127};
}

int saturate(float rounded, const QuantRange& r) {
  if (rounded < static_cast<float>(r.lo)) return r.lo;
  if (rounded > static_cast<float>(r.hi)) return r.hi;
  return static_cast<int>(rounded);
}

// Quantize one row `v` (already smooth-multiplied) into integer codes, and
// return its scale (and offset for the asymmetric mode).
void quantize_row(const std::vector<float>& v, int mode, const QuantRange& r,
                  std::vector<int>& codes, float* scale_out, float* offset_out) {
  const size_t n = v.size();
  codes.assign(n, 0);
  if (mode == ORACLE_SYMMETRIC) {
    float amax = 0.0f;
    for (size_t c = 0; c < n; ++c) {
      const float a = std::fabs(v[c]);
      if (a > amax) amax = a;
    }
    const float scale = amax / r.divisor;
    *scale_out = scale;
    if (scale == 0.0f) return;  // all-zero row: codes stay 0
    for (size_t c = 0; c < n; ++c) {
      const float quotient = v[c] / scale;
      codes[c] = saturate(std::nearbyint(quotient), r);
    }
    return;
  }
  // asymmetric
  float mx = v.empty() ? 0.0f : v[0];
  float mn = mx;
  for (size_t c = 0; c < n; ++c) {
    if (v[c] > mx) mx = v[c];
    if (v[c] < mn) mn = v[c];
  }
  const float range = mx - mn;
  const float scale = range / r.divisor;
  *scale_out = scale;
  if (scale == 0.0f) {
    // constant row: every element equals the row max, which maps to offset_opt
    *offset_out = r.offset_opt;
    for (size_t c = 0; c < n; ++c) codes[c] = static_cast<int>(r.offset_opt);
    return;
  }
  const float max_over_scale = mx / scale;
  const float offset = r.offset_opt - max_over_scale;
  *offset_out = offset;
  for (size_t c = 0; c < n; ++c) {
    const float quotient = v[c] / scale;
    const float shifted = quotient + offset;
    codes[c] = saturate(std::nearbyint(shifted), r);
  }
}

void store_codes(const std::vector<int>& codes, int y_dtype, void* y, int64_t row, int64_t cols) {
  if (y_dtype == ORACLE_Y_INT8) {
    int8_t* out = static_cast<int8_t*>(y) + row * cols;
    for (int64_t c = 0; c < cols; ++c) out[c] = static_cast<int8_t>(codes[c]);
  } else if (y_dtype == ORACLE_Y_INT4X2) {
    uint8_t* out = static_cast<uint8_t*>(y) + row * (cols / 2);
    for (int64_t j = 0; j < cols / 2; ++j) {
      const unsigned lo = static_cast<unsigned>(codes[2 * j]) & 0xFu;
      const unsigned hi = static_cast<unsigned>(codes[2 * j + 1]) & 0xFu;
      out[j] = static_cast<uint8_t>(lo | (hi << 4));
    }
  } else {  // ORACLE_Y_INT32
    uint32_t* out = static_cast<uint32_t*>(y) + row * (cols / 8);
    for (int64_t j = 0; j < cols / 8; ++j) {
      uint32_t word = 0;
      for (int k = 0; k < 8; ++k) {
        word |= (static_cast<uint32_t>(codes[8 * j + k]) & 0xFu) << (4 * k);
      }
      out[j] = word;
    }
  }
}

// expert(r): the smallest e with r < group_index[e] (cumulative end rows).
int expert_of_row(const int32_t* group_index, int32_t num_groups, int64_t row) {
  for (int32_t e = 0; e < num_groups; ++e) {
    if (row < static_cast<int64_t>(group_index[e])) return e;
  }
  return -1;
}

}  // namespace

extern "C" {

int oracle_dynamic_quant(const void* x, int x_dtype, int64_t rows, int64_t cols,
                         const void* smooth, int smooth_dtype,
                         const int32_t* group_index, int32_t num_groups,
                         int mode, int y_dtype,
                         void* y, float* scale, float* offset) {
  std::fesetround(FE_TONEAREST);
  if (rows < 0 || cols < 1) return ORACLE_ERR_SHAPE;
  if (!is_float_dtype(x_dtype)) return ORACLE_ERR_DTYPE;
  if (mode != ORACLE_SYMMETRIC && mode != ORACLE_ASYMMETRIC) return ORACLE_ERR_ARGUMENT;
  if (y_dtype != ORACLE_Y_INT8 && y_dtype != ORACLE_Y_INT4X2 && y_dtype != ORACLE_Y_INT32)
    return ORACLE_ERR_DTYPE;
  if (y_dtype == ORACLE_Y_INT4X2 && cols % 2 != 0) return ORACLE_ERR_SHAPE;
  if (y_dtype == ORACLE_Y_INT32 && cols % 8 != 0) return ORACLE_ERR_SHAPE;
  if (smooth != nullptr && !is_float_dtype(smooth_dtype)) return ORACLE_ERR_DTYPE;
  if ((group_index != nullptr) != (num_groups > 0)) return ORACLE_ERR_ARGUMENT;
  if (group_index != nullptr && smooth == nullptr) return ORACLE_ERR_ARGUMENT;
  if (mode == ORACLE_ASYMMETRIC && offset == nullptr) return ORACLE_ERR_ARGUMENT;
  if (group_index != nullptr) {
    int32_t previous = 0;
    for (int32_t e = 0; e < num_groups; ++e) {
      if (group_index[e] < previous) return ORACLE_ERR_GROUP_INDEX;
      previous = group_index[e];
    }
  }

  const QuantRange r = range_for(mode, y_dtype);
  std::vector<float> v(static_cast<size_t>(cols));
  std::vector<int> codes;
  for (int64_t row = 0; row < rows; ++row) {
    int64_t smooth_row = 0;
    if (group_index != nullptr) {
      const int e = expert_of_row(group_index, num_groups, row);
      if (e < 0) return ORACLE_ERR_GROUP_INDEX;
      smooth_row = e;
    }
    for (int64_t c = 0; c < cols; ++c) {
      float value = load_element(x, x_dtype, row * cols + c);
      if (smooth != nullptr) {
        value = value * load_element(smooth, smooth_dtype, smooth_row * cols + c);
      }
      v[static_cast<size_t>(c)] = value;
    }
    float row_scale = 0.0f;
    float row_offset = 0.0f;
    quantize_row(v, mode, r, codes, &row_scale, &row_offset);
    scale[row] = row_scale;
    if (mode == ORACLE_ASYMMETRIC) offset[row] = row_offset;
    store_codes(codes, y_dtype, y, row, cols);
  }
  return ORACLE_OK;
}

int oracle_ada_layernorm_pre(const void* x, int x_dtype, int64_t batch, int64_t seq, int64_t hidden,
                             const void* ada_scale, const void* ada_shift,
                             const void* weight, const void* bias, const void* smooth,
                             int param_dtype, float epsilon,
                             float* y, float* mean_out, float* std_out) {
  std::fesetround(FE_TONEAREST);
  if (batch < 0 || seq < 0 || hidden < 1) return ORACLE_ERR_SHAPE;
  if (!is_float_dtype(x_dtype) || !is_float_dtype(param_dtype)) return ORACLE_ERR_DTYPE;
  if (ada_scale == nullptr || ada_shift == nullptr) return ORACLE_ERR_ARGUMENT;

  std::vector<float> v(static_cast<size_t>(hidden));
  for (int64_t b = 0; b < batch; ++b) {
    for (int64_t s = 0; s < seq; ++s) {
      const int64_t row = b * seq + s;
      for (int64_t c = 0; c < hidden; ++c) {
        v[static_cast<size_t>(c)] = load_element(x, x_dtype, row * hidden + c);
      }
      // Step 1, E(x) and Var(x): two passes in double, each rounded to float once.
      double sum = 0.0;
      for (int64_t c = 0; c < hidden; ++c) sum += static_cast<double>(v[c]);
      const double mean_d = sum / static_cast<double>(hidden);
      double squares = 0.0;
      for (int64_t c = 0; c < hidden; ++c) {
        const double d = static_cast<double>(v[c]) - mean_d;
        squares += d * d;
      }
      const float mean = static_cast<float>(mean_d);
      const float var = static_cast<float>(squares / static_cast<double>(hidden));
      // sqrt(Var(x) + epsilon), then a true division per element, as printed.
      const float denom = std::sqrt(var + epsilon);
      if (mean_out != nullptr) mean_out[row] = mean;
      if (std_out != nullptr) std_out[row] = denom;
      for (int64_t c = 0; c < hidden; ++c) {
        const float centred = v[c] - mean;
        float ln = centred / denom;
        if (weight != nullptr) ln = ln * load_element(weight, param_dtype, c);
        if (bias != nullptr) ln = ln + load_element(bias, param_dtype, c);
        // Step 2: y = LayerNorm(x) * (1 + scale) + shift, scale/shift per batch.
        const float one_plus = 1.0f + load_element(ada_scale, param_dtype, b * hidden + c);
        float out = ln * one_plus;
        out = out + load_element(ada_shift, param_dtype, b * hidden + c);
        // Step 3: optional smooth scales.
        if (smooth != nullptr) out = out * load_element(smooth, param_dtype, c);
        y[row * hidden + c] = out;
      }
    }
  }
  return ORACLE_OK;
}

int oracle_ada_layernorm_quant(const void* x, int x_dtype, int64_t batch, int64_t seq, int64_t hidden,
                               const void* ada_scale, const void* ada_shift,
                               const void* weight, const void* bias, const void* smooth,
                               int param_dtype, float epsilon,
                               int8_t* out, float* quant_scale) {
  const int64_t rows = batch * seq;
  std::vector<float> y(static_cast<size_t>(rows > 0 ? rows * hidden : 0));
  int status = oracle_ada_layernorm_pre(x, x_dtype, batch, seq, hidden, ada_scale, ada_shift,
                                        weight, bias, smooth, param_dtype, epsilon, y.data(),
                                        nullptr, nullptr);
  if (status != ORACLE_OK) return status;
  // Steps 4-5: symmetric INT8 dynamic quantization of y.
  return oracle_dynamic_quant(y.data(), ORACLE_F32, rows, hidden, nullptr, ORACLE_F32, nullptr, 0,
                              ORACLE_SYMMETRIC, ORACLE_Y_INT8, out, quant_scale, nullptr);
}

int oracle_dequant_per_token(const void* y, int y_dtype, int64_t rows, int64_t cols,
                             const void* scale, const void* offset, int scale_dtype,
                             int out_dtype, void* out) {
  if (rows < 0 || cols < 1) return ORACLE_ERR_SHAPE;
  if (y_dtype != ORACLE_Y_INT8 && y_dtype != ORACLE_Y_INT4X2 && y_dtype != ORACLE_Y_INT32) return ORACLE_ERR_DTYPE;
  if (y_dtype == ORACLE_Y_INT4X2 && cols % 2 != 0) return ORACLE_ERR_SHAPE;
  if (y_dtype == ORACLE_Y_INT32 && cols % 8 != 0) return ORACLE_ERR_SHAPE;
  if (!is_float_dtype(scale_dtype) || !is_float_dtype(out_dtype)) return ORACLE_ERR_DTYPE;
  if (rows > 0 && (y == nullptr || scale == nullptr || out == nullptr)) return ORACLE_ERR_ARGUMENT;
  for (int64_t r = 0; r < rows; ++r) {
    const float s = load_element(scale, scale_dtype, r);
    const float o = offset != nullptr ? load_element(offset, scale_dtype, r) : 0.0f;
    for (int64_t c = 0; c < cols; ++c) {
      const int64_t i = r * cols + c;
      float v = static_cast<float>(load_code(y, y_dtype, i));
      if (offset != nullptr) v = v - o;
      v = v * s;
      if (out_dtype == ORACLE_F32) {
        static_cast<float*>(out)[i] = v;
      } else if (out_dtype == ORACLE_F16) {
        static_cast<uint16_t*>(out)[i] = narrow_to_half(v);
      } else {
        static_cast<uint16_t*>(out)[i] = narrow_to_bfloat16(v);
      }
    }
  }
  return ORACLE_OK;
}

int oracle_dequant_per_group(const void* y, int y_dtype, int64_t rows, int64_t cols,
                             const void* scale, const void* offset, int scale_dtype,
                             int64_t group_size, int k_dim, int out_dtype, void* out) {
  if (rows < 0 || cols < 1) return ORACLE_ERR_SHAPE;
  if (y_dtype != ORACLE_Y_INT8 && y_dtype != ORACLE_Y_INT4X2 && y_dtype != ORACLE_Y_INT32) return ORACLE_ERR_DTYPE;
  if (y_dtype == ORACLE_Y_INT4X2 && cols % 2 != 0) return ORACLE_ERR_SHAPE;
  if (y_dtype == ORACLE_Y_INT32 && cols % 8 != 0) return ORACLE_ERR_SHAPE;
  if (!is_float_dtype(scale_dtype) || !is_float_dtype(out_dtype)) return ORACLE_ERR_DTYPE;
  if (group_size <= 0 || group_size % 32 != 0 || (k_dim != 0 && k_dim != 1)) return ORACLE_ERR_ARGUMENT;
  if (rows > 0 && (y == nullptr || scale == nullptr || out == nullptr)) return ORACLE_ERR_ARGUMENT;
  const int64_t groups_per_row = (cols + group_size - 1) / group_size;  // k_dim 1: table width
  for (int64_t i = 0; i < rows; ++i) {
    for (int64_t j = 0; j < cols; ++j) {
      const int64_t entry = k_dim == 1 ? i * groups_per_row + j / group_size : (i / group_size) * cols + j;
      const float s = load_element(scale, scale_dtype, entry);
      const int64_t e = i * cols + j;
      float v = static_cast<float>(load_code(y, y_dtype, e));
      if (offset != nullptr) v = v - load_element(offset, scale_dtype, entry);
      v = v * s;
      if (out_dtype == ORACLE_F32) {
        static_cast<float*>(out)[e] = v;
      } else if (out_dtype == ORACLE_F16) {
        static_cast<uint16_t*>(out)[e] = narrow_to_half(v);
      } else {
        static_cast<uint16_t*>(out)[e] = narrow_to_bfloat16(v);
      }
    }
  }
  return ORACLE_OK;
}

int oracle_w8a8_gemm(const int8_t* a, const int8_t* b, int64_t m, int64_t n, int64_t k,
                     const float* a_scale, const float* b_scale, int out_dtype, int accumulate, void* out) {
  if (m < 0 || n < 0 || k < 1) return ORACLE_ERR_SHAPE;
  if (k >= (int64_t(1) << 17)) return ORACLE_ERR_SHAPE;  // |acc| <= k * 2^14 < 2^31 for any int8 codes
  if (!is_float_dtype(out_dtype)) return ORACLE_ERR_DTYPE;
  if (accumulate && out_dtype != ORACLE_F32) return ORACLE_ERR_ARGUMENT;
  if (m > 0 && n > 0 && (a == nullptr || b == nullptr || a_scale == nullptr || b_scale == nullptr || out == nullptr))
    return ORACLE_ERR_ARGUMENT;
  for (int64_t i = 0; i < m; ++i) {
    for (int64_t j = 0; j < n; ++j) {
      int64_t acc = 0;
      for (int64_t kk = 0; kk < k; ++kk) acc += static_cast<int64_t>(a[i * k + kk]) * static_cast<int64_t>(b[j * k + kk]);
      const float scales = a_scale[i] * b_scale[j];
      float t = static_cast<float>(static_cast<int32_t>(acc)) * scales;
      const int64_t e = i * n + j;
      if (out_dtype == ORACLE_F32) {
        float* o = static_cast<float*>(out);
        o[e] = accumulate ? t + o[e] : t;
      } else if (out_dtype == ORACLE_F16) {
        static_cast<uint16_t*>(out)[e] = narrow_to_half(t);
      } else {
        static_cast<uint16_t*>(out)[e] = narrow_to_bfloat16(t);
      }
    }
  }
  return ORACLE_OK;
}

uint16_t oracle_float_to_half_bits(float f) { return narrow_to_half(f); }
uint16_t oracle_float_to_bfloat16_bits(float f) { return narrow_to_bfloat16(f); }

}  // extern "C"
