// Explicit instantiations of the two-tile attention kernel (f16, d64, explicit masks).
// Split across files so the kernels compile in parallel.
#include "attn_pingpong.cuh"

namespace wf {
template cudaError_t launch_attn_pp<__half, 64, 0, 64, kKindMask>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__half, 64, 0, 96, kKindMask>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn_pp<__half, 64, 0, 128, kKindMask>(const AttnParams &, int, cudaStream_t);
}  // namespace wf
