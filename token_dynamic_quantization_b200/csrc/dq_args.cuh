// Argument blocks of the library's kernels and the enums they carry: the
// host side (dq_api.cu) fills them after validation, the kernels read them.
#pragma once

#include <stdint.h>

namespace dq {

// Largest CTA of the ring kernels: one producer warp and up to 31 consumer warps.
constexpr int kRingMaxThreads = 1024;

// Element type tags (mirror the dq_dtype values of the C ABI).
enum : int { kF32 = 0, kF16 = 1, kBF16 = 2 };

// ---- DynamicQuant (aclnnDynamicQuantV2)
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
  int tpr;                     // threads per row group (bulk-copy kernel)
  int groups;                  // row groups per CTA (bulk-copy kernel)
  int stages;                  // ring depth per group (bulk-copy kernel)
  uint32_t stage_stride;       // bytes between stages (multiple of 128)
  int moe_stage;               // ring kernel, MoE: stage up to 2 expert smooth rows per CTA
};

// ---- AdaLayerNormQuant (aclnnAdaLayerNormQuant)
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
  double inv_hidden;      // 1 / hidden, rounded once in double
  float* table;           // workspace: A [batch][hidden], then B [batch][hidden]
  int8_t* out;
  float* quant_scale;
  int tpr;
  int groups;
  int stages;
  uint32_t stage_stride;
  int table_batches;      // ring kernel: batches of the table staged in shared memory per CTA (0: read from L2)
};

// ---- dequantization (AntiQuantize)
struct DequantArgs {
  const void* y;       // codes
  int64_t rows, cols;
  const void* scale;   // scale table of scale_dtype (layout below)
  const void* offset;  // table of the same shape and dtype, or nullptr
  int scale_dtype;     // kF32 / kF16 / kBF16
  void* out;           // [rows, cols] of the output type
  int64_t group_size;  // group layouts only
  int64_t table_cols;  // row length of the scale table
};

enum : int { kOutF32 = 0, kOutF16 = 1, kOutBF16 = 2 };

// Scale-table layouts (AntiQuantize policies): PER_TOKEN [rows]; PER_GROUP
// with k along a row (kDim 1) [rows, ceil(cols/g)], entry (i, j / g); PER_GROUP
// with k down a column (kDim 0) [ceil(rows/g), cols], entry (i / g, j).
enum : int { kPerToken = 0, kGroupAlongRow = 1, kGroupDownColumn = 2 };

}  // namespace dq
