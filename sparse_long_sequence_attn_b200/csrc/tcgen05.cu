// Kernel family TCGEN05 (placeholder until the tensor-core kernel lands).
#include <cuda_runtime.h>

#include "params.h"

namespace longnet {
bool tcgen05_supports(const Problem&) { return false; }
int launch_tcgen05(const Problem&, cudaStream_t) { return LONGNET_ERR_UNSUPPORTED; }
}  // namespace longnet
