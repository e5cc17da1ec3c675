// noalloc.cu -- packed-sequence attention forward that allocates no memory.
//
// wf_attn_fwd keeps the packed-sequence schedule (prefix sums of the lengths
// and the longest-first work list) in a workspace it allocates on first use
// with cudaMalloc.  Some callers cannot allocate device memory once they are
// running: code captured into a CUDA graph that must not change the
// allocator's state, runtimes that hand the whole device to a pool at start-up
// and forbid further cudaMalloc, or embedded callers with a fixed memory
// budget.  wf_attn_fwd_varlen_noalloc serves them: the schedule lives in a
// file-scope __device__ array of fixed size, so the call never allocates.
//
// The array (kScheduleWords 32-bit words) exists on every GPU that loads the
// library, for as long as the process runs.  All calls share it: the schedule
// kernel writes every word the attention kernel then reads, so nothing has to
// be cleared between calls, but two calls whose work overlaps on the GPU (for
// example on two streams) overwrite each other's schedule and race.
#include <cmath>
#include <cstring>
#include <mutex>

#include "attn_params.h"
#include "runtime.h"

namespace wf {
namespace {

constexpr int64_t kScheduleWords = 65536;          // 256 KiB per device

__device__ __align__(256) int32_t g_noalloc_schedule[kScheduleWords];
// The attention kernel's work-item counters (zero at load; every launch
// leaves them zero).
__device__ __align__(16) int32_t g_noalloc_counters[4];

// Device addresses of the two arrays, looked up once per device (in host
// code an array's name is only a stand-in, not a device address).
std::mutex g_mu;
int32_t *g_sched_ptr[64] = {};
int32_t *g_counter_ptr[64] = {};

wf_status_t schedule_array(int dev, int32_t **out, int32_t **counters) {
  if (dev < 0 || dev >= 64) return fail(WF_ERR_NO_DEVICE, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_sched_ptr[dev]) {
    void *p = nullptr, *c = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_schedule);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(schedule array)");
    if ((e = cudaGetSymbolAddress(&c, g_noalloc_counters)) != cudaSuccess)
      return cuda_fail(e, "cudaGetSymbolAddress(counters)");
    g_sched_ptr[dev] = static_cast<int32_t *>(p);
    g_counter_ptr[dev] = static_cast<int32_t *>(c);
  }
  *out = g_sched_ptr[dev];
  *counters = g_counter_ptr[dev];
  return WF_OK;
}

}  // namespace

// Forget the looked-up addresses (wf_shutdown): after a device reset the
// next call looks them up again.
void forget_noalloc_addresses() {
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < 64; ++i) g_sched_ptr[i] = g_counter_ptr[i] = nullptr;
}

cudaError_t reset_noalloc_counters() {
  const int32_t zero[4] = {0, 0, 0, 0};
  return cudaMemcpyToSymbol(g_noalloc_counters, zero, sizeof(zero));
}

}  // namespace wf

using namespace wf;

extern "C" wf_status_t wf_attn_fwd_varlen_noalloc(
    const wf_tensor_t *q, const wf_tensor_t *qRope, const wf_tensor_t *k, const wf_tensor_t *kRope,
    const wf_tensor_t *v, const wf_tensor_t *qSeqLen, const wf_tensor_t *kvSeqLen, int32_t headNum,
    int32_t kvHeadNum, float qkScale, int32_t maskType, wf_tensor_t *out, void *stream) {
  clear_error();
  wf_status_t st;
  if (!q || !k || !v || !out || !qSeqLen || !kvSeqLen)
    return fail(WF_ERR_INVALID_ARG, "q, k, v, qSeqLen, kvSeqLen and out are required");
  if (q->dtype != WF_BF16)
    return fail(WF_ERR_UNSUPPORTED, "the allocation-free entry point takes bf16 tensors only");
  if (maskType != WF_MASK_NONE && maskType != WF_MASK_CAUSAL && maskType != WF_MASK_CAUSAL_TOP_LEFT)
    return fail(WF_ERR_UNSUPPORTED, "packed sequences take maskType NONE, CAUSAL or CAUSAL_TOP_LEFT");
  if (!std::isfinite(qkScale)) return fail(WF_ERR_INVALID_ARG, "qkScale is not finite");
  if ((qRope == nullptr) != (kRope == nullptr))
    return fail(WF_ERR_INVALID_ARG, "qRope and kRope are given together or not at all");
  if (headNum <= 0 || kvHeadNum <= 0 || headNum % kvHeadNum != 0)
    return fail(WF_ERR_INVALID_ARG, "headNum %d must be a positive multiple of kvHeadNum %d",
                headNum, kvHeadNum);
  const int32_t dt = WF_BF16;
  if ((st = check_tensor(q, "q", 3, dt, true)) != WF_OK) return st;
  if ((st = check_tensor(k, "k", 3, dt, true)) != WF_OK) return st;
  if ((st = check_tensor(v, "v", 3, dt, true)) != WF_OK) return st;
  if ((st = check_tensor(out, "out", 3, dt, true)) != WF_OK) return st;
  if ((st = check_tensor(qSeqLen, "qSeqLen", 1, WF_I32, false)) != WF_OK) return st;
  if ((st = check_tensor(kvSeqLen, "kvSeqLen", 1, WF_I32, false)) != WF_OK) return st;
  if (q->shape[1] != headNum || out->shape[1] != headNum)
    return fail(WF_ERR_INVALID_ARG, "q/out head dim must equal headNum %d", headNum);
  if (k->shape[1] != kvHeadNum || v->shape[1] != kvHeadNum)
    return fail(WF_ERR_INVALID_ARG, "k/v head dim must equal kvHeadNum %d", kvHeadNum);
  const int64_t dqk = q->shape[2], dv = v->shape[2];
  if (k->shape[2] != dqk || out->shape[2] != dv || k->shape[0] != v->shape[0] ||
      out->shape[0] != q->shape[0])
    return fail(WF_ERR_INVALID_ARG, "q/k/v/out shapes do not match");
  if (qSeqLen->shape[0] != kvSeqLen->shape[0])
    return fail(WF_ERR_INVALID_ARG, "qSeqLen and kvSeqLen have different lengths");
  if (qSeqLen->shape[0] > 0 && (qSeqLen->stride[0] != 1 || kvSeqLen->stride[0] != 1))
    return fail(WF_ERR_INVALID_ARG, "qSeqLen / kvSeqLen must be contiguous");
  int64_t drope = 0;
  if (qRope) {
    if ((st = check_tensor(qRope, "qRope", 3, dt, true)) != WF_OK) return st;
    if ((st = check_tensor(kRope, "kRope", 3, dt, true)) != WF_OK) return st;
    drope = qRope->shape[2];
    if (kRope->shape[2] != drope || qRope->shape[0] != q->shape[0] || qRope->shape[1] != headNum ||
        kRope->shape[0] != k->shape[0] || kRope->shape[1] != kvHeadNum)
      return fail(WF_ERR_INVALID_ARG, "qRope / kRope shapes do not match q / k");
    if (!(drope == 64 && dqk == 128 && dv == 128))
      return fail(WF_ERR_UNSUPPORTED, "rope part needs Dqk = Dv = 128 and a 64-wide rope");
  }
  const AttnKernel kern = find_attn_kernel(kElemBF16, (int)dqk, (int)drope, (int)dv, kKindPlain);
  if (!kern.launch)
    return fail(WF_ERR_UNSUPPORTED, "head sizes Dqk=%lld Dv=%lld are not implemented",
                (long long)dqk, (long long)dv);
  const int64_t B = qSeqLen->shape[0], tq = q->shape[0], tk = k->shape[0];
  if (B == 0 || tq == 0) return WF_OK;

  // schedule layout (same as wf_attn_fwd) and the size limit of the array
  const int64_t max_items = ((tq + kern.unit_rows - 1) / kern.unit_rows + B) * headNum;
  if (max_items > INT32_MAX) return fail(WF_ERR_UNSUPPORTED, "too many work items");
  SchedLayout sl{};
  sl.cu_q = 2;
  sl.cu_k = (int32_t)(sl.cu_q + B + 1);
  sl.order = (int32_t)(sl.cu_k + B + 1);
  sl.cu_work = (int32_t)(sl.order + B);
  sl.words = sl.cu_work + B + 1;
  if (sl.words > kScheduleWords)
    return fail(WF_ERR_INVALID_ARG,
                "schedule needs %lld words (batch %lld); the allocation-free entry point holds "
                "at most %lld: 4 * batch + 5 <= %lld, i.e. batch <= %lld",
                (long long)sl.words, (long long)B, (long long)kScheduleWords,
                (long long)kScheduleWords, (long long)((kScheduleWords - 5) / 4));

  DeviceState *ds = current_device_state(&st);
  if (!ds) return st;
  int dev = 0;
  cudaGetDevice(&dev);
  int32_t *ws = nullptr;
  int32_t *counters = nullptr;
  if ((st = schedule_array(dev, &ws, &counters)) != WF_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  const int64_t tkm = tk > 0 ? tk : 1;
  st = make_map(&p.tm_q, q->data, dt, dqk, tq, headNum, 1, q->stride[0], q->stride[1],
                q->stride[0] * tq, "q");
  if (st == WF_OK && drope)
    st = make_map(&p.tm_qr, qRope->data, dt, drope, tq, headNum, 1, qRope->stride[0],
                  qRope->stride[1], qRope->stride[0] * tq, "qRope");
  if (st == WF_OK && tk > 0) {
    st = make_map(&p.tm_k, k->data, dt, dqk, tkm, kvHeadNum, 1, k->stride[0], k->stride[1],
                  k->stride[0] * tkm, "k");
    if (st == WF_OK)
      st = make_map(&p.tm_v, v->data, dt, dv, tkm, kvHeadNum, 1, v->stride[0], v->stride[1],
                    v->stride[0] * tkm, "v");
    if (st == WF_OK && drope)
      st = make_map(&p.tm_kr, kRope->data, dt, drope, tkm, kvHeadNum, 1, kRope->stride[0],
                    kRope->stride[1], kRope->stride[0] * tkm, "kRope");
  }
  if (st != WF_OK) return st;
  if (!drope) p.tm_qr = p.tm_q;
  if (tk == 0) p.tm_k = p.tm_v = p.tm_q;
  if (!drope || tk == 0) p.tm_kr = p.tm_k;
  p.out = out->data;
  p.o_sb = 0;
  p.o_sh = out->stride[1];
  p.o_si = out->stride[0];
  p.mask_kind = maskType == WF_MASK_CAUSAL_TOP_LEFT ? kMaskCausal : maskType;
  p.causal_top_left = maskType == WF_MASK_CAUSAL_TOP_LEFT ? 1 : 0;
  p.batch = (int32_t)B;
  p.hq = headNum;
  p.hkv = kvHeadNum;
  p.group = headNum / kvHeadNum;
  p.varlen = 1;
  p.n_split = 1;
  p.unit_rows = kern.unit_rows;
  p.scale_log2 = qkScale * 1.4426950408889634f;
  p.status = ds->status;
  p.timeout_cycles = 2LL << 30;
  p.ws = ws;
  p.sl = sl;
  p.counters = counters;
  cudaError_t e = launch_sched_prep(static_cast<const int32_t *>(qSeqLen->data),
                                    static_cast<const int32_t *>(kvSeqLen->data), (int32_t)B, tq,
                                    tk, tk, headNum, kern.unit_rows, ws, sl, ds->status, cs);
  if (e != cudaSuccess) return cuda_fail(e, "sched_prep launch");
  e = kern.launch(p, ds->sm_count, cs);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  return WF_OK;
}
