// tree_verify_attn, tensor-core prefix kernel (tcgen05 / TMEM / TMA).
#include "attn.cuh"

namespace tv {

bool attn_tc_supported(const tv_attn_args*) { return false; }

cudaError_t launch_attn_tc(const AttnParams&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace tv
