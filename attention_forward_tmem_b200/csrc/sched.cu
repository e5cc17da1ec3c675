// sched.cu -- work order for packed (varlen) sequences.
//
// Packed sequences ("MLA Prefill", parameter table: qSeqLen / kvSeqLen int32
// [batch]; sequence b occupies the rows after those of sequences 0..b-1).  One
// CTA of 1024 threads:
//   1. prefix sums of the q and kv lengths, and the work units per sequence
//      (`unit_rows` query rows each);
//   2. a length check (non-negative, sums within the tensors; with padded K/V
//      every kv length within the padded length);
//   3. the sequences ordered by unit count, longest first (counting sort), and
//      the prefix sums of units x headNum in that order.
// The attention kernel enumerates its work items from these (see attn_params.h).
#include <cstdint>

#include "attn_params.h"
#include "sm100_ptx.cuh"

namespace wf {
namespace {

constexpr int kSchedThreads = 1024;
constexpr int kHistBins = 4096;

// Exclusive scan of one int64 per thread across the block; returns the block total.
__device__ int64_t block_exclusive_scan(int64_t v, int64_t &excl, int64_t *warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int64_t n = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int64_t w = warp_tot[lane];
    int64_t wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int64_t n = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += n;
    }
    warp_tot[lane] = wi - w;          // exclusive prefix of the warp totals
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  excl = warp_tot[warp] + incl - v;
  const int64_t total = warp_tot[32];
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kSchedThreads) sched_prep_kernel(
    const int32_t *__restrict__ q_len, const int32_t *__restrict__ k_len, int32_t batch,
    int64_t n_q_tokens, int64_t n_k_tokens, int64_t k_max_len, int32_t head_num,
    int32_t *__restrict__ ws,
    int32_t unit_rows, SchedLayout sl, int32_t *__restrict__ status) {
  __shared__ int64_t warp_tot[33];
  __shared__ int32_t hist[kHistBins];
  __shared__ int32_t bad;
  __shared__ int64_t carry_q, carry_k, carry_w;
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (tid == 0) {
    bad = 0;
    carry_q = carry_k = carry_w = 0;
  }
  for (int i = tid; i < kHistBins; i += kSchedThreads) hist[i] = 0;
  __syncthreads();
  auto units_of = [&](int64_t lq) -> int64_t { return lq > 0 ? (lq + unit_rows - 1) / unit_rows : 0; };
  auto bin_of = [&](int64_t nu) -> int32_t {
    return kHistBins - 1 - static_cast<int32_t>(nu < kHistBins - 1 ? nu : kHistBins - 1);
  };

  // 1. prefix sums of the lengths, and the unit-count histogram
  for (int32_t base = 0; base < batch; base += kSchedThreads) {
    const int32_t b = base + tid;
    int64_t lq = 0, lk = 0;
    if (b < batch) {
      lq = q_len[b];
      lk = k_len[b];
      if (lq < 0 || lk < 0 || lk > k_max_len) atomicOr(&bad, 1);
      else atomicAdd(&hist[bin_of(units_of(lq))], 1);
    }
    int64_t eq, ek;
    const int64_t tq = block_exclusive_scan(lq, eq, warp_tot);
    const int64_t tk = block_exclusive_scan(lk, ek, warp_tot);
    if (b < batch) {
      ws[sl.cu_q + b] = static_cast<int32_t>(carry_q + eq);
      ws[sl.cu_k + b] = static_cast<int32_t>(carry_k + ek);
    }
    __syncthreads();
    if (tid == 0) {
      carry_q += tq;
      carry_k += tk;
    }
    __syncthreads();
  }
  if (tid == 0) {
    if (carry_q > n_q_tokens || carry_k > n_k_tokens) bad = 1;
    ws[sl.cu_q + batch] = static_cast<int32_t>(carry_q);
    ws[sl.cu_k + batch] = static_cast<int32_t>(carry_k);
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      ws[0] = 0;
      ws[1] = 1;
      atomicCAS(status, 0, kDevInvalidArg);
    }
    return;
  }

  // 2. counting sort of the sequences by unit count, longest first (the order
  //    inside one count is unspecified; it changes no result)
  {
    int32_t v[4], s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[i] = hist[tid * 4 + i];
      s += v[i];
    }
    int64_t excl;
    block_exclusive_scan(s, excl, warp_tot);
    int32_t run = static_cast<int32_t>(excl);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hist[tid * 4 + i] = run;
      run += v[i];
    }
  }
  __syncthreads();
  for (int32_t b = tid; b < batch; b += kSchedThreads) {
    const int64_t lq = ws[sl.cu_q + b + 1] - ws[sl.cu_q + b];
    ws[sl.order + atomicAdd(&hist[bin_of(units_of(lq))], 1)] = b;
  }
  __syncthreads();

  // 3. prefix sums of units x headNum in that order
  for (int32_t base = 0; base < batch; base += kSchedThreads) {
    const int32_t k = base + tid;
    int64_t w = 0;
    if (k < batch) {
      const int32_t b = ws[sl.order + k];
      w = units_of(ws[sl.cu_q + b + 1] - ws[sl.cu_q + b]) * head_num;
    }
    int64_t ew;
    const int64_t tw = block_exclusive_scan(w, ew, warp_tot);
    if (k < batch) ws[sl.cu_work + k] = static_cast<int32_t>(carry_w + ew);
    __syncthreads();
    if (tid == 0) carry_w += tw;
    __syncthreads();
  }
  if (tid == 0) {
    ws[sl.cu_work + batch] = static_cast<int32_t>(carry_w);
    ws[0] = static_cast<int32_t>(carry_w);
    ws[1] = 0;
  }
}

}  // namespace

cudaError_t launch_sched_prep(const int32_t *q_len, const int32_t *k_len, int32_t batch,
                              int64_t n_q_tokens, int64_t n_k_tokens, int64_t k_max_len,
                              int32_t head_num, int32_t unit_rows, int32_t *ws,
                              const SchedLayout &sl, int32_t *status, cudaStream_t stream) {
  static_assert(kHistBins == 4 * kSchedThreads, "scan covers 4 bins per thread");
  return launch_pdl(sched_prep_kernel, dim3(1), dim3(kSchedThreads), 0, stream, q_len, k_len, batch,
                    n_q_tokens, n_k_tokens, k_max_len, head_num, ws, unit_rows, sl, status);
}

}  // namespace wf
