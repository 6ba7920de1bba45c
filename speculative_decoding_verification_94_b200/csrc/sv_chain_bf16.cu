// sv_chain_bf16.cu -- the persistent chain kernel for bf16 target logits.
#include "sv_chain_launch.cuh"

namespace sv {
size_t chain_ws_bytes(int B, int k, int V, int K) { return chain_ws_layout(B, k, V, K).bytes; }
cudaError_t launch_chain_bf16(const ChainArgs& a) { return launch_chain_dtype<BF16>(a); }
}  // namespace sv
