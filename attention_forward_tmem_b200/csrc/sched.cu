// sched.cu -- varlen tile schedule for the attention kernel.
//
// Packed sequences ("MLA Prefill", parameter table: qSeqLen / kvSeqLen int32
// [batch]; sequence b occupies the rows after those of sequences 0..b-1).  One
// CTA of 1024 threads:
//   1. prefix sums of the q lengths, kv lengths and q-tile counts;
//   2. a length check (non-negative, sums within the tensors);
//   3. the (sequence, work unit) entries ordered by the KV-tile count of the
//      unit's last row, longest first (counting sort over the count), so the
//      persistent attention CTAs take the long causal units first and finish
//      together.  A work unit is `unit_rows` consecutive query rows.
// The attention kernel then maps work item t to entry t / headNum and head
// t % headNum, so the heads of one GQA group run next to each other.
#include <cstdint>

#include "attn_params.h"

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

__device__ __forceinline__ int32_t kv_tiles(int32_t q0, int32_t rows, int32_t lq, int32_t lk,
                                            int32_t causal) {
  int32_t kend = lk;
  if (causal) kend = min(kend, min(q0 + rows, lq) + (lk - lq));
  return kend > 0 ? (kend + kBlockN - 1) / kBlockN : 0;
}

__global__ void __launch_bounds__(kSchedThreads) sched_prep_kernel(
    const int32_t *__restrict__ q_len, const int32_t *__restrict__ k_len, int32_t batch,
    int64_t n_q_tokens, int64_t n_k_tokens, int32_t causal, int32_t *__restrict__ ws,
    int32_t unit_rows, SchedLayout sl, int32_t *__restrict__ status) {
  __shared__ int64_t warp_tot[33];
  __shared__ int32_t hist[kHistBins];
  __shared__ int32_t bad;
  __shared__ int64_t carry_q, carry_k, carry_t;
  const int tid = threadIdx.x;
  if (tid == 0) {
    bad = 0;
    carry_q = carry_k = carry_t = 0;
  }
  __syncthreads();

  // 1. prefix sums, in chunks of the block size
  for (int32_t base = 0; base < batch; base += kSchedThreads) {
    const int32_t b = base + tid;
    int64_t lq = 0, lk = 0, nt = 0;
    if (b < batch) {
      lq = q_len[b];
      lk = k_len[b];
      if (lq < 0 || lk < 0) atomicOr(&bad, 1);
      nt = lq > 0 ? (lq + unit_rows - 1) / unit_rows : 0;
    }
    int64_t eq, ek, et;
    const int64_t tq = block_exclusive_scan(lq, eq, warp_tot);
    const int64_t tk = block_exclusive_scan(lk, ek, warp_tot);
    const int64_t tt = block_exclusive_scan(nt, et, warp_tot);
    if (b < batch) {
      ws[sl.cu_q + b] = static_cast<int32_t>(carry_q + eq);
      ws[sl.cu_k + b] = static_cast<int32_t>(carry_k + ek);
      ws[sl.cu_t + b] = static_cast<int32_t>(carry_t + et);
    }
    __syncthreads();
    if (tid == 0) {
      carry_q += tq;
      carry_k += tk;
      carry_t += tt;
    }
    __syncthreads();
  }
  if (tid == 0) {
    if (carry_q > n_q_tokens || carry_k > n_k_tokens || carry_t > sl.capacity) bad = 1;
    ws[sl.cu_q + batch] = static_cast<int32_t>(carry_q);
    ws[sl.cu_k + batch] = static_cast<int32_t>(carry_k);
    ws[sl.cu_t + batch] = static_cast<int32_t>(carry_t);
  }
  for (int i = tid; i < kHistBins; i += kSchedThreads) hist[i] = 0;
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      ws[0] = 0;
      ws[1] = 1;
      atomicCAS(status, 0, kDevInvalidArg);
    }
    return;
  }
  const int32_t n_entries = static_cast<int32_t>(carry_t);

  // 2. histogram of KV-tile counts; bin 0 holds the longest entries
  auto locate = [&](int32_t e, int32_t &b, int32_t &qt) {
    int32_t lo = 0, hi = batch - 1;         // last b with cu_t[b] <= e
    while (lo < hi) {
      const int32_t mid = (lo + hi + 1) >> 1;
      if (ws[sl.cu_t + mid] <= e) lo = mid; else hi = mid - 1;
    }
    b = lo;
    qt = e - ws[sl.cu_t + b];
  };
  auto bin_of = [&](int32_t b, int32_t qt) {
    const int32_t lq = ws[sl.cu_q + b + 1] - ws[sl.cu_q + b];
    const int32_t lk = ws[sl.cu_k + b + 1] - ws[sl.cu_k + b];
    const int32_t w = kv_tiles(qt * unit_rows, unit_rows, lq, lk, causal);
    return kHistBins - 1 - min(w, kHistBins - 1);
  };
  for (int32_t e = tid; e < n_entries; e += kSchedThreads) {
    int32_t b, qt;
    locate(e, b, qt);
    atomicAdd(&hist[bin_of(b, qt)], 1);
  }
  __syncthreads();

  // 3. exclusive scan of the histogram (4 bins per thread)
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

  // 4. scatter (order inside a bin is unspecified; it changes no result)
  for (int32_t e = tid; e < n_entries; e += kSchedThreads) {
    int32_t b, qt;
    locate(e, b, qt);
    const int32_t pos = atomicAdd(&hist[bin_of(b, qt)], 1);
    ws[sl.entries + 2 * pos] = b;
    ws[sl.entries + 2 * pos + 1] = qt;
  }
  if (tid == 0) {
    ws[0] = n_entries;
    ws[1] = 0;
  }
}

}  // namespace

cudaError_t launch_sched_prep(const int32_t *q_len, const int32_t *k_len, int32_t batch,
                              int64_t n_q_tokens, int64_t n_k_tokens, int32_t causal,
                              int32_t unit_rows, int32_t *ws, const SchedLayout &sl,
                              int32_t *status, cudaStream_t stream) {
  static_assert(kHistBins == 4 * kSchedThreads, "scan covers 4 bins per thread");
  sched_prep_kernel<<<1, kSchedThreads, 0, stream>>>(q_len, k_len, batch, n_q_tokens, n_k_tokens,
                                                     causal, ws, unit_rows, sl, status);
  return cudaGetLastError();
}

}  // namespace wf
