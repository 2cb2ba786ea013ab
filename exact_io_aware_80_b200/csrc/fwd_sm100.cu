// fwd_sm100.cu -- placeholder until the tcgen05 forward lands.
#include "kernels.h"

namespace fa {
bool fwd_sm100_supported(const AttnArgs&) { return false; }
cudaError_t launch_fwd_sm100(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace fa
