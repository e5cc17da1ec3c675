// attn_registry.cu -- maps (dtype, head sizes) to a compiled attention kernel.
#include <cuda_bf16.h>

#include "attn_params.h"

namespace wf {

template <typename T, int DQK, int DROPE, int DV>
cudaError_t launch_attn(const AttnParams &p, int grid, cudaStream_t stream);

AttnLaunchFn find_attn_kernel(int dtype, int dqk, int drope, int dv) {
#define WF_CASE(T, TI, Q, R, V) \
  if (dtype == TI && dqk == Q && drope == R && dv == V) return &launch_attn<T, Q, R, V>;
  WF_CASE(__nv_bfloat16, 1, 64, 0, 64)
  WF_CASE(__nv_bfloat16, 1, 64, 0, 96)
  WF_CASE(__nv_bfloat16, 1, 64, 0, 128)
  WF_CASE(__nv_bfloat16, 1, 96, 0, 64)
  WF_CASE(__nv_bfloat16, 1, 96, 0, 96)
  WF_CASE(__nv_bfloat16, 1, 96, 0, 128)
  WF_CASE(__nv_bfloat16, 1, 128, 0, 64)
  WF_CASE(__nv_bfloat16, 1, 128, 0, 96)
  WF_CASE(__nv_bfloat16, 1, 128, 0, 128)
  WF_CASE(__nv_bfloat16, 1, 128, 64, 128)
  WF_CASE(float, 0, 64, 0, 64)
  WF_CASE(float, 0, 64, 0, 96)
  WF_CASE(float, 0, 64, 0, 128)
  WF_CASE(float, 0, 96, 0, 64)
  WF_CASE(float, 0, 96, 0, 96)
  WF_CASE(float, 0, 96, 0, 128)
  WF_CASE(float, 0, 128, 0, 64)
  WF_CASE(float, 0, 128, 0, 96)
  WF_CASE(float, 0, 128, 0, 128)
#undef WF_CASE
  return nullptr;
}

}  // namespace wf
