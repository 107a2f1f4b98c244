// tcgen05 ragged-prefill kernel (placeholder until written).
#include "spa_attn.cuh"

namespace spa {
int prefill_supported(const spa_attention_args_t*) { return 0; }
int launch_prefill(const AttnParams&, int, cudaStream_t) { return SPA_ERR_UNSUPPORTED; }
}  // namespace spa
