// Kernel family SMALLSEG (placeholder until the memory-bound kernel lands).
#include <cuda_runtime.h>

#include "params.h"

namespace longnet {
bool smallseg_supports(const Problem&) { return false; }
int launch_smallseg(const Problem&, cudaStream_t) { return LONGNET_ERR_UNSUPPORTED; }
}  // namespace longnet
