// fa_bwd.cu -- attention backward (placeholder until the kernels land).
#include <cuda_runtime.h>
#include "fa_internal.h"
namespace fa {
cudaError_t launch_bwd(const BwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace fa
