// Explicit instantiations of the attention kernel (bf16, mla).
// Split across files so the kernels compile in parallel.
#include "attn_kernel.cuh"

namespace wf {
template cudaError_t launch_attn<__nv_bfloat16, 128, 64, 128>(const AttnParams &, int, cudaStream_t);
}  // namespace wf
