// tcgen05 tensor-core path (sm_100a). Shapes without a tensor-core kernel are
// reported unsupported and run on the CUDA-core path under TM_PATH_AUTO.
#include "tm_internal.h"

namespace tmem {

bool tc_supported(const Problem &) { return false; }
size_t tc_scratch_bytes(const Problem &) { return 0; }
cudaError_t tc_launch(const Problem &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace tmem
