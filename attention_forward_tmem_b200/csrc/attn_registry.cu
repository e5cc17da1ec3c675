// attn_registry.cu -- maps (dtype, head sizes, kernel kind) to a compiled
// attention kernel.  bf16 and fp16 run the two-tile kernel (256-row work
// units) in three instances (plain, fused cache write, explicit masks); fp32
// runs the single-tile TF32 kernel (128-row work units), whose tiles are twice
// as large.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "attn_params.h"

namespace wf {

template <typename T, int DQK, int DROPE, int DV>
cudaError_t launch_attn(const AttnParams &p, int grid, cudaStream_t stream);
template <typename T, int DQK, int DROPE, int DV, int kKind>
cudaError_t launch_attn_pp(const AttnParams &p, int grid, cudaStream_t stream);

AttnKernel find_attn_kernel(int dtype, int dqk, int drope, int dv, int kind) {
  // kernels that also write a BlockKVCache chunk (head sizes 64 and 128)
  if (kind == kKindFuse) {
#define WF_CASE_FUSED(T, TI, Q, V) \
  if (dtype == TI && dqk == Q && drope == 0 && dv == V) return {&launch_attn_pp<T, Q, 0, V, kKindFuse>, 2 * kBlockM};
    WF_CASE_FUSED(__nv_bfloat16, kElemBF16, 64, 64)
    WF_CASE_FUSED(__nv_bfloat16, kElemBF16, 128, 128)
    WF_CASE_FUSED(__half, kElemF16, 64, 64)
    WF_CASE_FUSED(__half, kElemF16, 128, 128)
#undef WF_CASE_FUSED
    return {nullptr, 0};
  }
  // 16-bit: the plain instance (no mask / causal) or the explicit-mask one
  // (dense layout, no rope part)
#define WF_CASE_PP(T, TI, Q, R, V) \
  if (dtype == TI && dqk == Q && drope == R && dv == V) { \
    if (kind == kKindMask) return R == 0 ? AttnKernel{&launch_attn_pp<T, Q, 0, V, kKindMask>, 2 * kBlockM} \
                                        : AttnKernel{nullptr, 0}; \
    return {&launch_attn_pp<T, Q, R, V, kKindPlain>, 2 * kBlockM}; \
  }
#define WF_CASE_PP16(Q, R, V) \
  WF_CASE_PP(__nv_bfloat16, kElemBF16, Q, R, V) \
  WF_CASE_PP(__half, kElemF16, Q, R, V)
// fp32: the single-tile TF32 kernel handles every mask kind
#define WF_CASE_1T(T, TI, Q, R, V) \
  if (dtype == TI && dqk == Q && drope == R && dv == V) return {&launch_attn<T, Q, R, V>, kBlockM};
  WF_CASE_PP16(64, 0, 64)
  WF_CASE_PP16(64, 0, 96)
  WF_CASE_PP16(64, 0, 128)
  WF_CASE_PP16(96, 0, 64)
  WF_CASE_PP16(96, 0, 96)
  WF_CASE_PP16(96, 0, 128)
  WF_CASE_PP16(128, 0, 64)
  WF_CASE_PP16(128, 0, 96)
  WF_CASE_PP16(128, 0, 128)
  WF_CASE_PP16(128, 64, 128)
  WF_CASE_1T(float, kElemF32, 64, 0, 64)
  WF_CASE_1T(float, kElemF32, 64, 0, 96)
  WF_CASE_1T(float, kElemF32, 64, 0, 128)
  WF_CASE_1T(float, kElemF32, 96, 0, 64)
  WF_CASE_1T(float, kElemF32, 96, 0, 96)
  WF_CASE_1T(float, kElemF32, 96, 0, 128)
  WF_CASE_1T(float, kElemF32, 128, 0, 64)
  WF_CASE_1T(float, kElemF32, 128, 0, 96)
  WF_CASE_1T(float, kElemF32, 128, 0, 128)
#undef WF_CASE_PP
#undef WF_CASE_PP16
#undef WF_CASE_1T
  return {nullptr, 0};
}

}  // namespace wf
