// merge.cu -- combine attention results computed over disjoint key sets.
//
// The pages name the uses (context-parallel attention in "Core 注意力",
// section "选择最窄的入口"; calcType RING in the "MLA Prefill" parameter
// table) but not the step; it follows from the softmax definition.  For a row
// whose keys were split into sets s = 1..S, each with its normalised result
// out_s and natural-log LSE lse_s:
//     lse = ln sum_s exp(lse_s),      out = sum_s exp(lse_s - lse) * out_s.
// A set with lse_s = -inf (no visible key) has weight 0; a row with every
// set at -inf is 0 with LSE -inf.  The largest lse_s is subtracted before
// exponentiating.
//
// One warp per row, four consecutive columns per lane per pass (128 columns
// a pass); HBM-bound: it reads S partial rows and writes one.  With at most
// four parts (the split-KV case) every load of a row (the parts' LSEs and
// their columns) is issued at once, so a row costs one memory latency.
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "attn_params.h"
#include "sm100_ptx.cuh"

namespace wf {
namespace {

constexpr int kMergeWarps = 8;
constexpr float kLog2eM = 1.4426950408889634f;
constexpr float kLn2M = 0.6931471805599453f;

__device__ __forceinline__ void load4(const void *base, int64_t idx, int32_t type, float (&v)[4]) {
  if (type == kElemF32) {
    const float4 f = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + idx);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    return;
  }
  const uint2 u = *reinterpret_cast<const uint2 *>(reinterpret_cast<const uint16_t *>(base) + idx);
  float2 a, b;
  if (type == kElemBF16) {
    a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  } else {
    a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
    b = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
  }
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

__device__ __forceinline__ void store4(void *base, int64_t idx, int32_t type, const float (&v)[4]) {
  if (type == kElemF32) {
    *reinterpret_cast<float4 *>(reinterpret_cast<float *>(base) + idx) = make_float4(v[0], v[1], v[2], v[3]);
    return;
  }
  uint2 u;
  if (type == kElemBF16) {
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
  } else {
    u.x = pack_f16x2(v[0], v[1]);
    u.y = pack_f16x2(v[2], v[3]);
  }
  *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(base) + idx) = u;
}

__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(const __grid_constant__ MergeParams mp) {
  pdl_wait();                        // the partial rows of the previous launch
  pdl_trigger();
  int64_t rows = mp.rows;
  if (mp.sched) {
    if (mp.sched[1] != 0) return;                                   // lengths were rejected
    rows = min(rows, (int64_t)mp.sched[mp.sched_tokens] * mp.n2);   // rows of the sequences
  }
  const int64_t r = (int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const int64_t i2 = r % mp.n2, i01 = r / mp.n2;
  const int64_t i1 = i01 % mp.n1, i0 = i01 / mp.n1;

  // Weights: lane s holds part s's LSE (parts beyond 32 in further rounds);
  // the warp reduces the max and the sum by shuffles.
  float top = -INFINITY;
  for (int s0 = 0; s0 < mp.n_split; s0 += 32) {
    const int s = s0 + lane;
    const float ls = s < mp.n_split ? mp.lses[s * mp.l_ss + r * mp.l_sr] : -INFINITY;
    top = fmaxf(top, ls);
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, d));
  const bool empty = top == -INFINITY;
  float total = 0.f;
  if (!empty) {
    for (int s0 = 0; s0 < mp.n_split; s0 += 32) {
      const int s = s0 + lane;
      const float ls = s < mp.n_split ? mp.lses[s * mp.l_ss + r * mp.l_sr] : -INFINITY;
      total += ls == -INFINITY ? 0.f : ex2_approx((ls - top) * kLog2eM);
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) total += __shfl_xor_sync(0xffffffffu, total, d);
  }
  const float inv = empty ? 0.f : 1.f / total;

  const int64_t obase = i0 * mp.o_s0 + i1 * mp.o_s1 + i2 * mp.o_s2;
  for (int c = lane * 4; c < mp.dv; c += 128) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (!empty) {
      // four parts' rows in flight at a time
      for (int s = 0; s < mp.n_split; s += 4) {
        float v[4][4], w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          w[k] = 0.f;
          if (s + k < mp.n_split) {
            const float ls = mp.lses[(s + k) * mp.l_ss + r * mp.l_sr];
            if (ls != -INFINITY) {                       // weight 0: its row may be anything
              w[k] = ex2_approx((ls - top) * kLog2eM) * inv;
              load4(mp.parts, (s + k) * mp.p_ss + r * mp.p_sr + c, mp.parts_type, v[k]);
            }
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (w[k] != 0.f)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e] = fmaf(w[k], v[k][e], acc[e]);
      }
    }
    store4(mp.out, obase + c, mp.out_type, acc);
  }
  if (mp.lse && lane == 0)
    mp.lse[i0 * mp.e_s0 + i1 * mp.e_s1 + i2 * mp.e_s2] = empty ? -INFINITY : top + __log2f(total) * kLn2M;
}

// At most kFewParts parts and Dv <= 128: each lane loads every part's LSE
// (the same words in every lane) and its four columns of every part in one
// batch, then combines them without shuffles.
constexpr int kFewParts = 4;
__global__ void __launch_bounds__(kMergeWarps * 32) merge_few_kernel(const __grid_constant__ MergeParams mp) {
  pdl_wait();
  pdl_trigger();
  int64_t rows = mp.rows;
  if (mp.sched) {
    if (mp.sched[1] != 0) return;
    rows = min(rows, (int64_t)mp.sched[mp.sched_tokens] * mp.n2);
  }
  const int64_t r = (int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const int c = lane * 4;
  const bool col = c < mp.dv;
  float ls[kFewParts], v[kFewParts][4];
#pragma unroll
  for (int s = 0; s < kFewParts; ++s) {
    ls[s] = s < mp.n_split ? mp.lses[s * mp.l_ss + r * mp.l_sr] : -INFINITY;
    v[s][0] = v[s][1] = v[s][2] = v[s][3] = 0.f;
    if (s < mp.n_split && col) load4(mp.parts, s * mp.p_ss + r * mp.p_sr + c, mp.parts_type, v[s]);
  }
  float top = ls[0];
#pragma unroll
  for (int s = 1; s < kFewParts; ++s) top = fmaxf(top, ls[s]);
  const bool empty = top == -INFINITY;
  float w[kFewParts], total = 0.f;
#pragma unroll
  for (int s = 0; s < kFewParts; ++s) {
    w[s] = (empty || ls[s] == -INFINITY) ? 0.f : ex2_approx((ls[s] - top) * kLog2eM);
    total += w[s];
  }
  const float inv = empty ? 0.f : 1.f / total;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int s = 0; s < kFewParts; ++s)
    if (w[s] != 0.f)                                  // weight 0: its row may be anything
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = fmaf(w[s] * inv, v[s][e], acc[e]);
  const int64_t i2 = r % mp.n2, i01 = r / mp.n2;
  const int64_t i1 = i01 % mp.n1, i0 = i01 / mp.n1;
  if (col) store4(mp.out, i0 * mp.o_s0 + i1 * mp.o_s1 + i2 * mp.o_s2 + c, mp.out_type, acc);
  if (mp.lse && lane == 0)
    mp.lse[i0 * mp.e_s0 + i1 * mp.e_s1 + i2 * mp.e_s2] = empty ? -INFINITY : top + __log2f(total) * kLn2M;
}

__global__ void fill_f32_kernel(float *dst, int64_t n, float v) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = v;
}

}  // namespace

cudaError_t launch_fill_f32(float *dst, int64_t n, float v, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 8);
  return launch_pdl(fill_f32_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, dst, n, v);
}

cudaError_t launch_merge(const MergeParams &mp, cudaStream_t stream) {
  if (mp.rows <= 0) return cudaSuccess;
  const int64_t blocks = (mp.rows + kMergeWarps - 1) / kMergeWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (mp.n_split <= kFewParts && mp.dv <= 128)
    return launch_pdl(merge_few_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kMergeWarps * 32), 0,
                      stream, mp);
  return launch_pdl(merge_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kMergeWarps * 32), 0, stream, mp);
}

}  // namespace wf
