// s2_bwd.cu -- S²-Attn backward (placeholder until the tcgen05 backward lands).
#include <cuda_runtime.h>

#include "s2_kernels.h"

namespace s2 {
int launch_bwd(const BwdArgs&) { return (int)cudaErrorNotSupported; }
}  // namespace s2
