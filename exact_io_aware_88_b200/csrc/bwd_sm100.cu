// bwd_sm100.cu -- attention backward on sm_100a (placeholder until the kernels land).
#include <cuda_runtime.h>

#include "launch.h"

namespace fa {

cudaError_t launch_bwd_sm100(const BwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace fa
