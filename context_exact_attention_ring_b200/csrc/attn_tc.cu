// Tensor-core ring attention (placeholder until the tcgen05 kernel lands).
#include "kernels.h"

namespace ra {
cudaError_t launch_attn_tc(const Plan&, const TcArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace ra
