// DynamicQuant dispatch for bf16 input, sym mode (aclnnDynamicQuantV2, "Formula").
#include "quant_launch.cuh"

DQ_DEFINE_QUANT_DISPATCH(quant_bf16_sym, __nv_bfloat16, dq::kSym)
