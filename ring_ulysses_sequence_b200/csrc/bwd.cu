// Ring attention backward (placeholder until the tensor-core kernels land).
#include "internal.h"

namespace rm {

cudaError_t launch_bwd(const AttnShape&, const void*, const void*, const void*, const void*,
                       const float*, const void*, float*, float*, float*, float*,
                       const LaunchCtx&) {
    return cudaErrorNotSupported;
}

}  // namespace rm
