// DynamicQuant dispatch for bf16 input, asym mode (aclnnDynamicQuantV2, "Formula").
#include "quant_launch.cuh"

DQ_DEFINE_QUANT_DISPATCH(quant_bf16_asym, __nv_bfloat16, dq::kAsym)
