// tc_kernels.cu — tcgen05 tensor-core kernels (bf16/fp16 inputs, fp32 state).
#include "tc_launch.h"

namespace la {

bool tc_supported(la_dtype, int, int) { return false; }
bool tc_noncausal_supported(la_dtype, int) { return false; }
la_status tc_causal(const TcCausalArgs &, cudaStream_t) { return LA_ERR_UNSUPPORTED; }
la_status tc_noncausal(const TcNoncausalArgs &, cudaStream_t) { return LA_ERR_UNSUPPORTED; }

}  // namespace la
