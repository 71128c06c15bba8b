// DynamicQuant dispatch for f16 input, sym mode (aclnnDynamicQuantV2, "Formula").
#include "quant_launch.cuh"

DQ_DEFINE_QUANT_DISPATCH(quant_f16_sym, __half, dq::kSym)
