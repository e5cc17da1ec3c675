// Explicit instantiations of the two-tile attention kernel (bf16, d64).
// Split across files so the kernels compile in parallel.
#include "attn_pingpong.cuh"

namespace wf {
template cudaError_t launch_attn_pp<__nv_bfloat16, 64, 0, 64, kKindPlain>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__nv_bfloat16, 64, 0, 96, kKindPlain>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__nv_bfloat16, 64, 0, 128, kKindPlain>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__nv_bfloat16, 64, 0, 64, kKindFuse>(const AttnParams &, int, cudaStream_t);  // fused cache write
}  // namespace wf
