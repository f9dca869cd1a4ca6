// bf16_causal.cu -- tcgen05 tensor-core path for causal phi attention.
#include <cuda_runtime.h>

#include "la_internal.h"

namespace la {

cudaError_t launch_bf16_causal(const LaunchArgs&) { return cudaErrorNotSupported; }

}  // namespace la
