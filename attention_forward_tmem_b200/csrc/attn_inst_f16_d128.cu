// Explicit instantiations of the two-tile attention kernel (f16, d128).
// Split across files so the kernels compile in parallel.
#include "attn_pingpong.cuh"

namespace wf {
template cudaError_t launch_attn_pp<__half, 128, 0, 64, kKindPlain>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__half, 128, 0, 96, kKindPlain>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__half, 128, 0, 128, kKindPlain>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__half, 128, 0, 128, kKindFuse>(const AttnParams &, int, cudaStream_t);  // fused cache write
}  // namespace wf
