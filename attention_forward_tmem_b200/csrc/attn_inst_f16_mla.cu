// Explicit instantiations of the two-tile attention kernel (f16, mla).
// Split across files so the kernels compile in parallel.
#include "attn_pingpong.cuh"

namespace wf {
template cudaError_t launch_attn_pp<__half, 128, 64, 128, kKindPlain>(const AttnParams &, int, cudaStream_t);
}  // namespace wf
