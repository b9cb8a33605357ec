// Backward of the gathered causal attention (placeholder until the tcgen05
// kernels land).
#include "lh_sm100.cuh"

cudaError_t lh_launch_attn_bwd(int BH, int64_t S, int d, float scale, const lh_bf16* qg,
                               const lh_bf16* kg, const lh_bf16* vg, const lh_bf16* dog,
                               const float* lse, const float* delta, lh_bf16* dqg,
                               lh_bf16* dkg, lh_bf16* dvg, int* status, cudaStream_t st,
                               int* launches) {
  return cudaErrorNotSupported;
}
