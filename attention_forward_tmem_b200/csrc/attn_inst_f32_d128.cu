// Explicit instantiations of the single-tile attention kernel (f32, d128; TF32 MMA).
// Split across files so the kernels compile in parallel.
#include "attn_kernel.cuh"

namespace wf {
template cudaError_t launch_attn<float, 128, 0, 64>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn<float, 128, 0, 96>(const AttnParams &, int, cudaStream_t);
template cudaError_t launch_attn<float, 128, 0, 128>(const AttnParams &, int, cudaStream_t);
}  // namespace wf
