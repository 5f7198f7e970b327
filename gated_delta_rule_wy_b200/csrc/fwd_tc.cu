// fwd_tc.cu -- tcgen05/TMEM chunkwise forward for bf16 inputs (sm_100a).
#include "gdr2_common.cuh"
#include "gdr2_launch.h"

namespace gdr2 {

bool forward_tc_supported(const FwdArgs &) { return false; }

cudaError_t launch_forward_tc(const FwdArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdr2
