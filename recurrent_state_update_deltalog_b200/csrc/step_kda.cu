// Kernel instantiations for the KDA operator (all supported d_k x d_v shapes,
// fp32 and bf16 inputs; deferred step, eager baseline, materialisation).
#include "launch.cuh"

namespace dl {
DL_INSTANTIATE_OP(OP_KDA)
}  // namespace dl
