// transpose.cu -- V^T for the fp32 (TF32) attention path.
//
// The TF32 tensor-core MMA accepts its B operand only K-major, i.e. for
// O += P V the keys must be contiguous: V [rows, D] is copied to
// V^T [batch][head][D][ld] (ld = rows rounded up to 4 so every row of V^T
// starts on a 16-byte boundary).  bf16 needs no copy: V is used MN-major.
#include <cstdint>

#include "attn_params.h"

namespace wf {
namespace {

constexpr int kTile = 32;

__global__ void __launch_bounds__(kTile * 8) transpose_v_kernel(
    const float *__restrict__ v, int64_t s_row, int64_t s_head, int64_t s_batch, int32_t rows,
    int32_t heads, int32_t batch, int32_t d, float *__restrict__ vt, int64_t ld) {
  __shared__ float tile[kTile][kTile + 1];
  const int32_t r0 = blockIdx.x * kTile, d0 = blockIdx.y * kTile;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int32_t bh = blockIdx.z; bh < heads * batch; bh += gridDim.z) {
    const int32_t b = bh / heads, h = bh % heads;
    const float *src = v + b * s_batch + h * s_head;
    float *dst = vt + (int64_t)bh * d * ld;
#pragma unroll
    for (int i = 0; i < kTile; i += 8) {
      const int32_t r = r0 + ty + i, c = d0 + tx;
      if (r < rows && c < d) tile[ty + i][tx] = src[(int64_t)r * s_row + c];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kTile; i += 8) {
      const int32_t c = d0 + ty + i, r = r0 + tx;
      if (r < rows && c < d) dst[(int64_t)c * ld + r] = tile[tx][ty + i];
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_transpose_v(const float *v, int64_t s_row, int64_t s_head, int64_t s_batch,
                               int32_t rows, int32_t heads, int32_t batch, int32_t d, float *vt,
                               int64_t ld, cudaStream_t stream) {
  if (rows == 0 || d == 0 || heads == 0 || batch == 0) return cudaSuccess;
  const int64_t bh = (int64_t)heads * batch;
  dim3 grid((rows + kTile - 1) / kTile, (d + kTile - 1) / kTile, (unsigned)(bh < 65535 ? bh : 65535));
  transpose_v_kernel<<<grid, dim3(kTile, 8), 0, stream>>>(v, s_row, s_head, s_batch, rows, heads,
                                                          batch, d, vt, ld);
  return cudaGetLastError();
}

}  // namespace wf
