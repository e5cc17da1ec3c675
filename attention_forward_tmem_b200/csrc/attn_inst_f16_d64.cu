// Explicit instantiations of the two-tile attention kernel (fp16, d64).
// Split across files so the kernels compile in parallel.
#include "attn_pingpong.cuh"

namespace wf {
template cudaError_t launch_attn_pp<__half, 64, 0, 64, false>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__half, 64, 0, 96, false>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__half, 64, 0, 128, false>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__half, 64, 0, 64, true>(const AttnParams &, int, cudaStream_t);  // fused cache write
}  // namespace wf
