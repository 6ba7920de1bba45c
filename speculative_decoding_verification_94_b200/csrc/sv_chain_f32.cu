// sv_chain_f32.cu -- the persistent chain kernel for fp32 target logits.
#include "sv_chain_launch.cuh"

namespace sv {
cudaError_t launch_chain_f32(const ChainArgs& a) { return launch_chain_dtype<F32>(a); }
}  // namespace sv
