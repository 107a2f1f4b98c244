// Tensor-core decode kernel (placeholder until written).
#include "spa_attn.cuh"

namespace spa {
int mma_supported(int, int, int, int) { return 0; }
int mma_key_tile() { return 64; }
int launch_attention_mma(const AttnParams&, int, int, int, cudaStream_t) { return SPA_ERR_UNSUPPORTED; }
}  // namespace spa
