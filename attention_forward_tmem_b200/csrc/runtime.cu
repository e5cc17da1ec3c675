// runtime.cu -- C ABI of the attention forward: argument checks, TMA
// descriptors, per-device state and the launch.
//
// Argument set and meaning: "MLA Prefill" (CANN ATB docs), section "定义" and
// its parameter table (Q, QRope, K, kRope, V, qSeqLen, kvSeqLen, mask,
// headNum, qkScale, kvHeadNum, maskType, attenOut; every call returns a
// status); dense [B, H, L, D] layout and mask meaning: "Core 注意力"
// (WorldFoundry docs), example section.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "attn_params.h"
#include "runtime.h"

namespace wf {

// ------------------------------------------------------------------ errors
static thread_local std::string g_last_error;

wf_status_t fail(wf_status_t st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}
void clear_error() { g_last_error.clear(); }

wf_status_t cuda_fail(cudaError_t e, const char *what) {
  return fail(WF_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t dtype_size(int32_t dtype) {
  switch (dtype) {
    case WF_F32: return 4;
    case WF_BF16: return 2;
    case WF_F16: return 2;
    case WF_U8: return 1;
    case WF_I32: return 4;
    default: return 0;
  }
}

// ----------------------------------------------------------- device state
__device__ int32_t g_device_status;   // one status word per device
// starts at 1 so that the zero-initialised per-kernel records read "not set"
std::atomic<uint32_t> g_setup_generation{1};

static std::mutex g_mu;
static std::map<int, DeviceState> g_devices;
static std::map<std::pair<int, cudaStream_t>, std::pair<int32_t *, size_t>> g_workspaces;

DeviceState *current_device_state(wf_status_t *st) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *st = fail(WF_ERR_NO_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_devices.find(dev);
  if (it != g_devices.end()) return &it->second;
  DeviceState ds;
  if ((e = cudaDeviceGetAttribute(&ds.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&ds.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&ds.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&ds.l2_bytes, cudaDevAttrL2CacheSize, dev)) != cudaSuccess) {
    *st = cuda_fail(e, "cudaDeviceGetAttribute");
    return nullptr;
  }
  if (ds.cc_major != 10 || ds.cc_minor != 0) {
    *st = fail(WF_ERR_NO_DEVICE, "device %d is sm_%d%d; this library runs on sm_100 (B200)", dev,
               ds.cc_major, ds.cc_minor);
    return nullptr;
  }
  if ((e = cudaGetSymbolAddress(reinterpret_cast<void **>(&ds.status), g_device_status)) != cudaSuccess) {
    *st = cuda_fail(e, "cudaGetSymbolAddress(status)");
    return nullptr;
  }
  return &g_devices.emplace(dev, ds).first->second;
}

// Workspace of one (device, stream): a header with the two-tile kernel's
// work-item counters, then the varlen schedule tables, V^T (fp32) and the
// split-KV partials.  Calls on different streams get different workspaces,
// so they may overlap.
constexpr size_t kWorkspaceHeader = 256;
static wf_status_t stream_workspace(int dev, cudaStream_t stream, size_t bytes, int32_t **out) {
  std::lock_guard<std::mutex> lock(g_mu);
  auto &slot = g_workspaces[{dev, stream}];
  if (slot.second < bytes) {
    if (slot.first) {
      // the old buffer may still be read by work queued on this stream
      cudaError_t e = cudaStreamSynchronize(stream);
      if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
      cudaFree(slot.first);
      slot.first = nullptr;
      slot.second = 0;
    }
    size_t sz = bytes < (1u << 20) ? (1u << 20) : bytes;
    void *p = nullptr;
    cudaError_t e = cudaMalloc(&p, sz);
    if (e != cudaSuccess) return fail(WF_ERR_NO_MEMORY, "cudaMalloc(%zu): %s", sz, cudaGetErrorString(e));
    // the header (work-item counters) starts at zero; kernels leave it zero
    if ((e = cudaMemsetAsync(p, 0, kWorkspaceHeader, stream)) != cudaSuccess) {
      cudaFree(p);
      return cuda_fail(e, "cudaMemsetAsync(workspace header)");
    }
    slot.first = static_cast<int32_t *>(p);
    slot.second = sz;
  }
  *out = slot.first;
  return WF_OK;
}

// Scratch of one (device, stream) for calls that run several attention calls
// (dual chunk attention): separate from the workspace those calls use.
static std::map<std::pair<int, cudaStream_t>, std::pair<void *, size_t>> g_scratch;

wf_status_t stream_scratch(cudaStream_t stream, size_t bytes, void **out) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_mu);
  auto &slot = g_scratch[{dev, stream}];
  if (slot.second < bytes) {
    if (slot.first) {
      cudaError_t e = cudaStreamSynchronize(stream);
      if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
      cudaFree(slot.first);
      slot.first = nullptr;
      slot.second = 0;
    }
    void *p = nullptr;
    cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) return fail(WF_ERR_NO_MEMORY, "cudaMalloc(%zu): %s", bytes, cudaGetErrorString(e));
    slot.first = p;
    slot.second = bytes;
  }
  *out = slot.first;
  return WF_OK;
}

// ----------------------------------------------------------- TMA descriptors
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// 4-d map (D, rows, heads, batch) with a (128 B of D) x 128 rows box, 128-byte
// swizzle, zero fill outside the tensor.  Strides in elements.
wf_status_t make_map(CUtensorMap *map, const void *base, int32_t dtype, int64_t d,
                            int64_t rows, int64_t heads, int64_t batch, int64_t s_row,
                            int64_t s_head, int64_t s_batch, const char *name, int32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(WF_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const size_t es = dtype_size(dtype);
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads, (cuuint64_t)batch};
  const cuuint64_t strides[3] = {(cuuint64_t)(s_row * es), (cuuint64_t)(s_head * es),
                                 (cuuint64_t)(s_batch * es)};
  const cuuint32_t box[4] = {(cuuint32_t)(128 / es), (cuuint32_t)box_rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = dtype == WF_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : dtype == WF_F16  ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, dt, 4, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(WF_ERR_INVALID_ARG, "%s: tensor map rejected (CUresult %d)", name, (int)r);
  return WF_OK;
}

// ------------------------------------------------------------- validation
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t numel(const wf_tensor_t *t) {
  int64_t n = 1;
  for (int i = 0; i < t->ndim; ++i) n *= t->shape[i];
  return n;
}

// Basic descriptor checks: ndim, dtype, non-negative shape, last stride 1,
// 16-byte alignment of the base and of every other stride.
wf_status_t check_tensor(const wf_tensor_t *t, const char *name, int ndim, int32_t dtype,
                         bool need_tma_layout) {
  if (!t) return fail(WF_ERR_INVALID_ARG, "%s is NULL", name);
  if (t->ndim != ndim) return fail(WF_ERR_INVALID_ARG, "%s: expected %d dims, got %d", name, ndim, t->ndim);
  if (t->dtype != dtype)
    return fail(WF_ERR_INVALID_ARG, "%s: dtype %d does not match %d", name, t->dtype, dtype);
  for (int i = 0; i < ndim; ++i) {
    if (t->shape[i] < 0) return fail(WF_ERR_INVALID_ARG, "%s: negative dim %d", name, i);
    if (t->shape[i] > INT32_MAX) return fail(WF_ERR_UNSUPPORTED, "%s: dim %d above 2^31-1", name, i);
  }
  if (numel(t) == 0) return WF_OK;
  if (!t->data) return fail(WF_ERR_INVALID_ARG, "%s: NULL data", name);
  if (need_tma_layout) {
    const size_t es = dtype_size(dtype);
    if (t->stride[ndim - 1] != 1 && t->shape[ndim - 1] > 1)
      return fail(WF_ERR_INVALID_ARG, "%s: last dimension must be contiguous", name);
    if (!aligned16(t->data)) return fail(WF_ERR_INVALID_ARG, "%s: data not 16-byte aligned", name);
    for (int i = 0; i < ndim - 1; ++i) {
      if (t->stride[i] < 0 || (t->stride[i] * (int64_t)es) % 16 != 0)
        return fail(WF_ERR_INVALID_ARG, "%s: stride %d is not a multiple of 16 bytes", name, i);
      if (t->stride[i] * (int64_t)es >= (int64_t(1) << 40))
        return fail(WF_ERR_UNSUPPORTED, "%s: stride %d too large", name, i);
    }
  }
  return WF_OK;
}

// The new chunk of a fused cache write (see attn_fwd_fused).
struct FuseArgs {
  const wf_tensor_t *k_chunk, *v_chunk;
  int64_t lo, hi;
  bool *declined;     // set when the call is valid attention but not fusable
};

constexpr int32_t kMaxSplits = 128;        // largest numSplits accepted
constexpr int64_t kMinTilesPerSplit = 4;   // automatic split: KV tiles per split, at least

static int32_t elem_type(int32_t dtype) {
  return dtype == WF_F32 ? kElemF32 : dtype == WF_F16 ? kElemF16 : kElemBF16;
}
int32_t elem_type_of(int32_t dtype) { return elem_type(dtype); }

struct Dims {
  bool varlen, kv_padded;
  int64_t batch, lq, lk, tq, tk, dqk, dv, drope;
};

}  // namespace wf

using namespace wf;

extern "C" {

static wf_status_t attn_fwd_impl(const wf_tensor_t *q, const wf_tensor_t *qRope, const wf_tensor_t *k,
                                 const wf_tensor_t *kRope, const wf_tensor_t *v,
                                 const wf_tensor_t *qSeqLen, const wf_tensor_t *kvSeqLen,
                                 const wf_tensor_t *mask, int32_t headNum, int32_t kvHeadNum,
                                 float qkScale, int32_t maskType, wf_tensor_t *out, wf_tensor_t *lse,
                                 int32_t numSplits, void *stream, uint32_t debug_flags,
                                 int64_t timeout_cycles, const FuseArgs *fuse);

wf_status_t wf_attn_fwd(const wf_tensor_t *q, const wf_tensor_t *qRope, const wf_tensor_t *k,
                        const wf_tensor_t *kRope, const wf_tensor_t *v, const wf_tensor_t *qSeqLen,
                        const wf_tensor_t *kvSeqLen, const wf_tensor_t *mask, int32_t headNum,
                        int32_t kvHeadNum, float qkScale, int32_t maskType, wf_tensor_t *out,
                        void *stream) {
  return attn_fwd_impl(q, qRope, k, kRope, v, qSeqLen, kvSeqLen, mask, headNum, kvHeadNum, qkScale,
                       maskType, out, nullptr, 0, stream, 0u, 0, nullptr);
}

wf_status_t wf_attn_fwd_ex(const wf_tensor_t *q, const wf_tensor_t *qRope, const wf_tensor_t *k,
                           const wf_tensor_t *kRope, const wf_tensor_t *v, const wf_tensor_t *qSeqLen,
                           const wf_tensor_t *kvSeqLen, const wf_tensor_t *mask, int32_t headNum,
                           int32_t kvHeadNum, float qkScale, int32_t maskType, wf_tensor_t *out,
                           wf_tensor_t *lse, int32_t numSplits, void *stream) {
  return attn_fwd_impl(q, qRope, k, kRope, v, qSeqLen, kvSeqLen, mask, headNum, kvHeadNum, qkScale,
                       maskType, out, lse, numSplits, stream, 0u, 0, nullptr);
}

wf_status_t wf_attn_fwd_debug(const wf_tensor_t *q, const wf_tensor_t *qRope, const wf_tensor_t *k,
                              const wf_tensor_t *kRope, const wf_tensor_t *v,
                              const wf_tensor_t *qSeqLen, const wf_tensor_t *kvSeqLen,
                              const wf_tensor_t *mask, int32_t headNum, int32_t kvHeadNum,
                              float qkScale, int32_t maskType, wf_tensor_t *out, void *stream,
                              uint32_t debug_flags, int64_t timeout_cycles) {
  return attn_fwd_impl(q, qRope, k, kRope, v, qSeqLen, kvSeqLen, mask, headNum, kvHeadNum, qkScale,
                       maskType, out, nullptr, 0, stream, debug_flags, timeout_cycles, nullptr);
}

}  // extern "C"

wf_status_t wf::attn_fwd_fused(const wf_tensor_t *q, const wf_tensor_t *k_view, const wf_tensor_t *v_view,
                               const wf_tensor_t *k_chunk, const wf_tensor_t *v_chunk, int64_t lo,
                               int64_t hi, int32_t headNum, int32_t kvHeadNum, float qkScale,
                               wf_tensor_t *out, void *stream, bool *declined) {
  *declined = false;
  const FuseArgs f{k_chunk, v_chunk, lo, hi, declined};
  return attn_fwd_impl(q, nullptr, k_view, nullptr, v_view, nullptr, nullptr, nullptr, headNum,
                       kvHeadNum, qkScale, WF_MASK_NONE, out, nullptr, 0, stream, 0u, 0, &f);
}

extern "C" {

wf_status_t wf_attn_merge(const wf_tensor_t *outParts, const wf_tensor_t *lseParts, wf_tensor_t *out,
                          wf_tensor_t *lse, void *stream) {
  clear_error();
  wf_status_t st;
  if (!outParts || !lseParts || !out) return fail(WF_ERR_INVALID_ARG, "outParts, lseParts and out are required");
  const int32_t pdt = outParts->dtype, odt = out->dtype;
  auto float_type = [](int32_t t) { return t == WF_F32 || t == WF_BF16 || t == WF_F16; };
  if (!float_type(pdt) || !float_type(odt))
    return fail(WF_ERR_UNSUPPORTED, "outParts / out dtype must be WF_F32, WF_BF16 or WF_F16");
  if ((st = check_tensor(outParts, "outParts", 3, pdt, true)) != WF_OK) return st;
  if ((st = check_tensor(lseParts, "lseParts", 2, WF_F32, false)) != WF_OK) return st;
  if ((st = check_tensor(out, "out", 2, odt, true)) != WF_OK) return st;
  if (lse && (st = check_tensor(lse, "lse", 1, WF_F32, false)) != WF_OK) return st;
  const int64_t S = outParts->shape[0], R = outParts->shape[1], dv = outParts->shape[2];
  if (lseParts->shape[0] != S || lseParts->shape[1] != R)
    return fail(WF_ERR_INVALID_ARG, "lseParts must be [%lld, %lld]", (long long)S, (long long)R);
  if (out->shape[0] != R || out->shape[1] != dv)
    return fail(WF_ERR_INVALID_ARG, "out must be [%lld, %lld]", (long long)R, (long long)dv);
  if (lse && lse->shape[0] != R) return fail(WF_ERR_INVALID_ARG, "lse must be [%lld]", (long long)R);
  if (dv % 4 != 0) return fail(WF_ERR_UNSUPPORTED, "head size %lld is not a multiple of 4", (long long)dv);
  if (S < 1 && R > 0) return fail(WF_ERR_INVALID_ARG, "at least one part is needed");
  if ((numel(lseParts) > 0 && reinterpret_cast<uintptr_t>(lseParts->data) % 4) ||
      (lse && numel(lse) > 0 && reinterpret_cast<uintptr_t>(lse->data) % 4))
    return fail(WF_ERR_INVALID_ARG, "lse tensors must be 4-byte aligned");
  if (R == 0 || dv == 0) return WF_OK;
  DeviceState *ds = current_device_state(&st);
  if (!ds) return st;
  MergeParams mp{};
  mp.parts = outParts->data;
  mp.parts_type = elem_type(pdt);
  mp.p_ss = outParts->stride[0];
  mp.p_sr = outParts->stride[1];
  mp.lses = static_cast<const float *>(lseParts->data);
  mp.l_ss = lseParts->stride[0];
  mp.l_sr = lseParts->stride[1];
  mp.n_split = (int32_t)S;
  mp.dv = (int32_t)dv;
  mp.rows = R;
  mp.n1 = 1;
  mp.n2 = R;
  mp.out = out->data;
  mp.out_type = elem_type(odt);
  mp.o_s2 = out->stride[0];
  if (lse) {
    mp.lse = static_cast<float *>(lse->data);
    mp.e_s2 = lse->stride[0];
  }
  cudaError_t e = launch_merge(mp, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return WF_OK;
}

// The forward behind every attention entry point.
static wf_status_t attn_fwd_impl(const wf_tensor_t *q, const wf_tensor_t *qRope, const wf_tensor_t *k,
                                 const wf_tensor_t *kRope, const wf_tensor_t *v,
                                 const wf_tensor_t *qSeqLen, const wf_tensor_t *kvSeqLen,
                                 const wf_tensor_t *mask, int32_t headNum, int32_t kvHeadNum,
                                 float qkScale, int32_t maskType, wf_tensor_t *out, wf_tensor_t *lse,
                                 int32_t numSplits, void *stream, uint32_t debug_flags,
                                 int64_t timeout_cycles, const FuseArgs *fuse) {
  clear_error();
  wf_status_t st;
  if (!q || !k || !v || !out) return fail(WF_ERR_INVALID_ARG, "q, k, v and out are required");
  const int32_t dt = q->dtype;
  if (dt != WF_BF16 && dt != WF_F16 && dt != WF_F32)
    return fail(WF_ERR_UNSUPPORTED, "q dtype %d: only WF_BF16, WF_F16 and WF_F32 are implemented", dt);
  if (maskType < WF_MASK_NONE || maskType > WF_MASK_CAUSAL_TOP_LEFT)
    return fail(WF_ERR_INVALID_ARG, "maskType %d out of range", maskType);
  if (!std::isfinite(qkScale)) return fail(WF_ERR_INVALID_ARG, "qkScale is not finite");
  if ((qSeqLen == nullptr) != (kvSeqLen == nullptr))
    return fail(WF_ERR_INVALID_ARG, "qSeqLen and kvSeqLen are given together or not at all");
  if ((qRope == nullptr) != (kRope == nullptr))
    return fail(WF_ERR_INVALID_ARG, "qRope and kRope are given together or not at all");
  if (headNum <= 0 || kvHeadNum <= 0 || headNum % kvHeadNum != 0)
    return fail(WF_ERR_INVALID_ARG, "headNum %d must be a positive multiple of kvHeadNum %d", headNum,
                kvHeadNum);

  Dims d{};
  d.varlen = qSeqLen != nullptr;
  // Packed queries with 4-d K / V: the padded layout [batch, max_seq, kvHead, D]
  // ("MLA Prefill" table rows K / V: [batch, max_seq, kv_head * D]).
  d.kv_padded = d.varlen && k->ndim == 4;
  // The TF32 path reads V^T with the key index as the innermost TMA
  // coordinate; a packed sequence may start at any token, which breaks the
  // 16-byte rule on that coordinate, so fp32 is dense-only.
  if (d.varlen && dt == WF_F32)
    return fail(WF_ERR_UNSUPPORTED, "WF_F32 inputs are supported in the dense layout only");
  const int nd = d.varlen ? 3 : 4;                     // q / out dims
  const int knd = d.varlen && !d.kv_padded ? 3 : 4;    // k / v dims
  if ((st = check_tensor(q, "q", nd, dt, true)) != WF_OK) return st;
  if ((st = check_tensor(k, "k", knd, dt, true)) != WF_OK) return st;
  if ((st = check_tensor(v, "v", knd, dt, true)) != WF_OK) return st;
  if ((st = check_tensor(out, "out", nd, dt, true)) != WF_OK) return st;
  const int rd = d.varlen ? 0 : 2;                     // q / out row dim
  const int khd = d.kv_padded ? 2 : 1;                 // k / v head dim
  const int krd = !d.varlen ? 2 : (d.kv_padded ? 1 : 0);   // k / v row dim
  if (q->shape[1] != headNum || out->shape[1] != headNum)
    return fail(WF_ERR_INVALID_ARG, "q/out head dim must equal headNum %d", headNum);
  if (k->shape[khd] != kvHeadNum || v->shape[khd] != kvHeadNum)
    return fail(WF_ERR_INVALID_ARG, "k/v head dim must equal kvHeadNum %d", kvHeadNum);
  d.dqk = q->shape[nd - 1];
  d.dv = v->shape[knd - 1];
  if (k->shape[knd - 1] != d.dqk) return fail(WF_ERR_INVALID_ARG, "q and k head sizes differ");
  if (out->shape[nd - 1] != d.dv) return fail(WF_ERR_INVALID_ARG, "out and v head sizes differ");
  if (k->shape[krd] != v->shape[krd]) return fail(WF_ERR_INVALID_ARG, "k and v lengths differ");
  if (out->shape[rd] != q->shape[rd]) return fail(WF_ERR_INVALID_ARG, "out and q lengths differ");
  if (!d.varlen) {
    d.batch = q->shape[0];
    if (k->shape[0] != d.batch || v->shape[0] != d.batch || out->shape[0] != d.batch)
      return fail(WF_ERR_INVALID_ARG, "batch sizes differ");
    d.lq = q->shape[2];
    d.lk = k->shape[2];
  } else {
    if ((st = check_tensor(qSeqLen, "qSeqLen", 1, WF_I32, false)) != WF_OK) return st;
    if ((st = check_tensor(kvSeqLen, "kvSeqLen", 1, WF_I32, false)) != WF_OK) return st;
    if (qSeqLen->shape[0] != kvSeqLen->shape[0])
      return fail(WF_ERR_INVALID_ARG, "qSeqLen and kvSeqLen have different lengths");
    if (qSeqLen->shape[0] > 0 && (qSeqLen->stride[0] != 1 || kvSeqLen->stride[0] != 1))
      return fail(WF_ERR_INVALID_ARG, "qSeqLen / kvSeqLen must be contiguous");
    d.batch = qSeqLen->shape[0];
    d.tq = q->shape[0];
    d.tk = k->shape[krd];          // packed: kv tokens; padded: max_seq
    if (d.kv_padded && (k->shape[0] != d.batch || v->shape[0] != d.batch))
      return fail(WF_ERR_INVALID_ARG, "padded k/v first dim must equal the batch %lld", (long long)d.batch);
  }
  d.drope = 0;
  if (qRope) {
    if ((st = check_tensor(qRope, "qRope", nd, dt, true)) != WF_OK) return st;
    if ((st = check_tensor(kRope, "kRope", knd, dt, true)) != WF_OK) return st;
    d.drope = qRope->shape[nd - 1];
    if (kRope->shape[knd - 1] != d.drope) return fail(WF_ERR_INVALID_ARG, "qRope/kRope sizes differ");
    for (int i = 0; i < nd - 1; ++i)
      if (qRope->shape[i] != q->shape[i]) return fail(WF_ERR_INVALID_ARG, "qRope shape does not match q");
    for (int i = 0; i < knd - 1; ++i)
      if (kRope->shape[i] != k->shape[i]) return fail(WF_ERR_INVALID_ARG, "kRope shape does not match k");
  }

  // lse: out's shape without the head-size dim, fp32, any strides
  if (lse) {
    if ((st = check_tensor(lse, "lse", nd - 1, WF_F32, false)) != WF_OK) return st;
    for (int i = 0; i < nd - 1; ++i)
      if (lse->shape[i] != out->shape[i])
        return fail(WF_ERR_INVALID_ARG, "lse must have out's shape without its last dim");
    if (numel(lse) > 0 && reinterpret_cast<uintptr_t>(lse->data) % 4)
      return fail(WF_ERR_INVALID_ARG, "lse: data not 4-byte aligned");
  }
  if (numSplits < 0 || numSplits > kMaxSplits)
    return fail(WF_ERR_INVALID_ARG, "numSplits %d: 0 (automatic) or 1..%d", numSplits, kMaxSplits);

  // mask
  const bool explicit_mask = maskType == WF_MASK_BOOL_KEEP || maskType == WF_MASK_ADDITIVE;
  if (!explicit_mask && mask) return fail(WF_ERR_INVALID_ARG, "mask given but maskType is %d", maskType);
  int64_t ms[4] = {0, 0, 0, 0};
  int32_t mask_dtype = kMaskU8;
  if (explicit_mask) {
    if (d.varlen)
      return fail(WF_ERR_UNSUPPORTED, "explicit masks are supported in the dense layout only");
    if (!mask) return fail(WF_ERR_INVALID_ARG, "maskType %d needs a mask tensor", maskType);
    if (mask->ndim != 4) return fail(WF_ERR_INVALID_ARG, "mask must have 4 dims [B|1, H|1, Lq, Lk]");
    if (maskType == WF_MASK_BOOL_KEEP) {
      if (mask->dtype != WF_U8) return fail(WF_ERR_INVALID_ARG, "bool keep-mask dtype must be WF_U8");
      mask_dtype = kMaskU8;
    } else {
      if (mask->dtype == WF_F32) mask_dtype = kMaskF32;
      else if (mask->dtype == WF_BF16 && dt == WF_BF16) mask_dtype = kMaskBF16;
      else if (mask->dtype == WF_F16 && dt == WF_F16) mask_dtype = kMaskF16;
      else return fail(WF_ERR_INVALID_ARG, "additive mask dtype must be WF_F32 or q's dtype");
    }
    const int64_t full[4] = {d.batch, headNum, d.lq, d.lk};
    for (int i = 0; i < 4; ++i) {
      if (mask->shape[i] == full[i]) ms[i] = mask->stride[i];
      else if (mask->shape[i] == 1) ms[i] = 0;
      else return fail(WF_ERR_INVALID_ARG, "mask dim %d is %lld, expected %lld or 1", i,
                       (long long)mask->shape[i], (long long)full[i]);
      if (full[i] > 1 && mask->shape[i] == full[i] && ms[i] < 0)
        return fail(WF_ERR_INVALID_ARG, "mask stride %d is negative", i);
    }
    if (numel(mask) > 0 && !mask->data) return fail(WF_ERR_INVALID_ARG, "mask: NULL data");
  }

  // supported head sizes
  if (d.drope && !(d.drope == 64 && d.dqk == 128 && d.dv == 128 && dt != WF_F32))
    return fail(WF_ERR_UNSUPPORTED, "rope part needs 16-bit inputs, Dqk = Dv = 128 and a 64-wide rope");
  AttnKernel kern = find_attn_kernel(elem_type(dt), (int)d.dqk, (int)d.drope, (int)d.dv,
                                     explicit_mask ? kKindMask : kKindPlain);
  if (!kern.launch)
    return fail(WF_ERR_UNSUPPORTED, "head sizes Dqk=%lld Dv=%lld (rope %lld) are not implemented",
                (long long)d.dqk, (long long)d.dv, (long long)d.drope);

  if (fuse) {
    const int64_t n = fuse->hi - fuse->lo;
    if (d.varlen || maskType != WF_MASK_NONE || d.drope || dt == WF_F32 || fuse->lo < 0 ||
        fuse->lo % kBlockN || n <= 0 || n % kBlockN || fuse->hi > d.lk) {
      *fuse->declined = true;       // dense 16-bit, no mask or rope, 128-key boundaries only
      return WF_OK;
    }
    for (const wf_tensor_t *t : {fuse->k_chunk, fuse->v_chunk}) {
      if ((st = check_tensor(t, "chunk", 4, dt, true)) != WF_OK) return st;
      if (t->shape[0] != d.batch || t->shape[1] != kvHeadNum || t->shape[2] != n)
        return fail(WF_ERR_INVALID_ARG, "chunk must be [B, kvHeadNum, %lld, D]", (long long)n);
    }
    if (fuse->k_chunk->shape[3] != d.dqk || fuse->v_chunk->shape[3] != d.dv)
      return fail(WF_ERR_INVALID_ARG, "chunk head sizes differ from k / v");
    // the kernel instance that also writes the chunk, where one is built
    const AttnKernel fk = find_attn_kernel(elem_type(dt), (int)d.dqk, 0, (int)d.dv, kKindFuse);
    if (!fk.launch) {
      *fuse->declined = true;
      return WF_OK;
    }
    kern = fk;
  }

  // nothing to compute?
  if (d.batch == 0 || numel(q) == 0) return WF_OK;

  DeviceState *ds = current_device_state(&st);
  if (!ds) return st;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  const int64_t n_keys = d.varlen ? d.tk : d.lk;   // rows of k / v
  // q / k / v maps: (D, rows, heads, batch).  Dense: rows = sequence
  // positions, batch = B.  Packed: rows = tokens of all sequences, batch = 1.
  // Padded K / V: (D, max_seq, heads, batch), like the dense layout.
  struct MapArgs { int64_t rows, batch, s_row, s_head, s_batch; };
  auto dims_of = [&](const wf_tensor_t *t, int64_t rows, bool kv) -> MapArgs {
    if (!d.varlen) return {rows, d.batch, t->stride[2], t->stride[1], t->stride[0]};
    if (kv && d.kv_padded) return {rows, d.batch, t->stride[1], t->stride[2], t->stride[0]};
    return {rows, 1, t->stride[0], t->stride[1], t->stride[0] * rows};
  };
  auto map_of = [&](CUtensorMap *m, const wf_tensor_t *t, int64_t dd, int64_t rows, int64_t heads,
                    bool kv, const char *name) {
    const MapArgs a = dims_of(t, rows, kv);
    return make_map(m, t->data, dt, dd, a.rows, heads, a.batch, a.s_row, a.s_head, a.s_batch, name);
  };
  const int64_t n_q = d.varlen ? d.tq : d.lq;
  st = map_of(&p.tm_q, q, d.dqk, n_q, headNum, false, "q");
  if (st == WF_OK && d.drope) st = map_of(&p.tm_qr, qRope, d.drope, n_q, headNum, false, "qRope");
  if (st == WF_OK && n_keys > 0) {
    st = map_of(&p.tm_k, k, d.dqk, n_keys, kvHeadNum, true, "k");
    if (st == WF_OK && dt != WF_F32) st = map_of(&p.tm_v, v, d.dv, n_keys, kvHeadNum, true, "v");
    if (st == WF_OK && d.drope) st = map_of(&p.tm_kr, kRope, d.drope, n_keys, kvHeadNum, true, "kRope");
  }
  if (st != WF_OK) return st;
  if (st == WF_OK && fuse) {
    st = map_of(&p.tm_kc, fuse->k_chunk, d.dqk, fuse->hi - fuse->lo, kvHeadNum, true, "k chunk");
    if (st == WF_OK) st = map_of(&p.tm_vc, fuse->v_chunk, d.dv, fuse->hi - fuse->lo, kvHeadNum, true, "v chunk");
    p.fuse_lo = (int32_t)fuse->lo;
    p.fuse_hi = (int32_t)fuse->hi;
  }
  if (st != WF_OK) return st;
  if (!fuse) p.tm_kc = p.tm_vc = p.tm_q;     // never read
  // Maps that are never read (no rope part, or no key at all): copies of q's
  // so that every descriptor passed to the kernel is well formed.
  if (!d.drope) p.tm_qr = p.tm_q;
  if (n_keys == 0) p.tm_k = p.tm_v = p.tm_q;
  if (!d.drope || n_keys == 0) p.tm_kr = p.tm_k;

  p.out = out->data;
  if (!d.varlen) {
    p.o_sb = out->stride[0];
    p.o_sh = out->stride[1];
    p.o_si = out->stride[2];
    // Output rows through shared memory and TMA stores (two-tile kernel,
    // head size 128, no split; see pp_softmax): where the map's rules hold
    // (16-byte aligned base, strides multiples of 16 bytes), 32-row boxes.
    const int64_t es = (int64_t)dtype_size(dt);
    const auto al16 = [&](int64_t v) { return (v * es) % 16 == 0; };
    if (dt != WF_F32 && d.dv == 128 && d.lq > 0 && (reinterpret_cast<uintptr_t>(out->data) & 15) == 0 &&
        al16(p.o_si) && al16(p.o_sh) && al16(p.o_sb) && p.o_si > 0 && p.o_sh > 0 && p.o_sb > 0 &&
        make_map(&p.tm_o, out->data, dt, d.dv, d.lq, headNum, d.batch, p.o_si, p.o_sh, p.o_sb, "out", 32) == WF_OK)
      p.tma_out = 1;
    else
      clear_error();
  } else {
    p.o_sb = 0;
    p.o_sh = out->stride[1];
    p.o_si = out->stride[0];
  }
  if (lse) {
    p.lse = static_cast<float *>(lse->data);
    p.l_sb = d.varlen ? 0 : lse->stride[0];
    p.l_sh = lse->stride[1];
    p.l_si = d.varlen ? lse->stride[0] : lse->stride[2];
  }
  p.mask = explicit_mask ? mask->data : nullptr;
  p.m_sb = ms[0];
  p.m_sh = ms[1];
  p.m_si = ms[2];
  p.m_sj = ms[3];
  p.mask_kind = maskType == WF_MASK_CAUSAL_TOP_LEFT ? kMaskCausal : maskType;
  p.causal_top_left = maskType == WF_MASK_CAUSAL_TOP_LEFT ? 1 : 0;
  p.mask_dtype = mask_dtype;
  p.batch = (int32_t)d.batch;
  p.hq = headNum;
  p.hkv = kvHeadNum;
  p.group = headNum / kvHeadNum;
  p.varlen = d.varlen ? 1 : 0;
  p.kv_padded = d.kv_padded ? 1 : 0;
  p.scale_log2 = qkScale * 1.4426950408889634f;
  p.status = ds->status;
  p.timeout_cycles = timeout_cycles > 0 ? timeout_cycles : (2LL << 30);
  p.debug_flags = debug_flags;

  // Split-KV: automatic only in the dense layout (the packed unit count is
  // known on the device alone), when the units cannot fill the SMs: as many
  // splits as fill them, each with at least kMinTilesPerSplit KV tiles.
  const int64_t dense_units = d.varlen ? 0 : ((d.lq + kern.unit_rows - 1) / kern.unit_rows) * d.batch * headNum;
  int32_t n_split = numSplits > 0 ? numSplits : 1;
  if (numSplits == 0 && !d.varlen && n_keys > 0 && dense_units > 0 && dense_units < ds->sm_count) {
    const int64_t by_grid = ds->sm_count / dense_units;
    const int64_t by_len = ((d.lk + kBlockN - 1) / kBlockN) / kMinTilesPerSplit;
    n_split = (int32_t)std::max<int64_t>(1, std::min(by_grid, by_len));
  }
  p.n_split = n_split;
  if (n_split > 1) p.tma_out = 0;           // partial rows in fp32 go to the workspace

  // Per-stream workspace: [schedule tables (varlen)] [V^T (fp32)] [split
  // partials: out fp32, lse fp32], 256-byte aligned parts.
  SchedLayout sl{};
  size_t sched_bytes = 0;
  if (d.varlen) {
    const int64_t B = d.batch;
    const int64_t max_items = ((d.tq + kern.unit_rows - 1) / kern.unit_rows + B) * headNum * n_split;
    if (max_items > INT32_MAX) return fail(WF_ERR_UNSUPPORTED, "too many work items");
    sl.cu_q = 2;
    sl.cu_k = (int32_t)(sl.cu_q + B + 1);
    sl.order = (int32_t)(sl.cu_k + B + 1);
    sl.cu_work = (int32_t)(sl.order + B);
    sl.words = sl.cu_work + B + 1;
    sched_bytes = ((size_t)sl.words * 4 + 255) & ~size_t(255);
  }
  const int64_t vt_ld = (n_keys + 3) & ~int64_t(3);
  const int64_t vt_batch = d.varlen ? 1 : d.batch;
  const size_t vt_bytes =
      dt == WF_F32 ? ((size_t)(vt_batch * kvHeadNum * d.dv * vt_ld) * 4 + 255) & ~size_t(255) : 0;
  const int64_t part_rows = n_split > 1 ? (d.varlen ? d.tq : d.batch * d.lq) * headNum : 0;
  const size_t part_o_bytes = ((size_t)n_split * part_rows * d.dv * 4 + 255) & ~size_t(255);
  const size_t part_l_bytes = ((size_t)n_split * part_rows * 4 + 255) & ~size_t(255);
  const size_t ws_bytes = kWorkspaceHeader + sched_bytes + vt_bytes + part_o_bytes + part_l_bytes;
  int32_t *ws_base = nullptr;
  if ((st = stream_workspace(dev, cs, ws_bytes, &ws_base)) != WF_OK) return st;
  p.counters = ws_base;
  int32_t *ws = ws_base + kWorkspaceHeader / 4;      // schedule tables
  if (n_split > 1) {
    uint8_t *base = reinterpret_cast<uint8_t *>(ws) + sched_bytes + vt_bytes;
    p.part_o = reinterpret_cast<float *>(base);
    p.part_lse = reinterpret_cast<float *>(base + part_o_bytes);
    p.part_rows = part_rows;
    // the two-tile kernel's staged stores of partial rows (dense, head size 128)
    if (!d.varlen && dt != WF_F32 && d.dv == 128 &&
        make_map(&p.tm_po, p.part_o, WF_F32, d.dv, part_rows, n_split, 1, d.dv, part_rows * d.dv,
                 (int64_t)n_split * part_rows * d.dv, "split partials", 32) == WF_OK)
      p.tma_part = 1;
    else
      clear_error();
  }
  if (dt == WF_F32) {
    float *vt = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(ws) + sched_bytes);
    if (n_keys > 0) {
      const int64_t s_row = d.varlen ? v->stride[0] : v->stride[2];
      const int64_t s_head = v->stride[1];
      const int64_t s_batch = d.varlen ? 0 : v->stride[0];
      cudaError_t e = launch_transpose_v(static_cast<const float *>(v->data), s_row, s_head, s_batch,
                                         (int32_t)n_keys, kvHeadNum, (int32_t)vt_batch, (int32_t)d.dv,
                                         vt, vt_ld, cs);
      if (e != cudaSuccess) return cuda_fail(e, "V transpose launch");
      // V^T as (keys, Dv rows, heads, batch): the kernel loads (128-byte key span) x 128 rows
      st = make_map(&p.tm_v, vt, dt, n_keys, d.dv, kvHeadNum, vt_batch, vt_ld, d.dv * vt_ld,
                    kvHeadNum * d.dv * vt_ld, "V^T");
      if (st != WF_OK) return st;
    } else {
      p.tm_v = p.tm_q;    // never read: no key
    }
  }

  int grid = ds->sm_count;
  p.unit_rows = kern.unit_rows;
  if (!d.varlen) {
    p.lq = (int32_t)d.lq;
    p.lk = (int32_t)d.lk;
    const int64_t per_bh = (d.lq + kern.unit_rows - 1) / kern.unit_rows;
    const int64_t units = dense_units;
    if (units * n_split > INT32_MAX)
      return fail(WF_ERR_UNSUPPORTED, "too many work items (%lld)", (long long)(units * n_split));
    p.units_per_bh = (int32_t)per_bh;
    p.n_units_dense = (int32_t)units;
    // Causal units differ in length.  Block by block (locality first), with
    // fewer items in a (batch, kv head) block than SMs, several blocks run at
    // once and the last blocks' longest units start near the end of the
    // launch, leaving SMs idle while they finish (causal GQA prefill at B 4,
    // 32/8 heads, L 4096: 64 items a block on 148 SMs; ncu: SM active 93% of
    // the elapsed cycles).  There the last blocks,
    // about two waves of items, are claimed by unit rank instead, so the
    // launch ends on short units (SM active 98%).  Only those blocks: in unit
    // rank order over all 32 blocks of that workload the K / V of every block stayed in
    // use, were read ~3 times, and the extra DRAM power cost the gain back
    // under the power cap.  With more items a block than SMs the last block
    // fills the machine, longest first, by itself.
    const int64_t items_per_block = per_bh * (headNum / kvHeadNum);
    const int64_t blocks = d.batch * kvHeadNum;
    p.unit_major = 0;
    if (p.mask_kind == kMaskCausal && per_bh > 1 && blocks > 1 && items_per_block < ds->sm_count)
      p.unit_major = (int32_t)std::min<int64_t>(blocks, (2 * ds->sm_count + items_per_block - 1) / items_per_block);
    if (units * n_split < grid) grid = (int)(units * n_split);
  } else {
    const int64_t B = d.batch;
    cudaError_t e = launch_sched_prep(static_cast<const int32_t *>(qSeqLen->data),
                                      static_cast<const int32_t *>(kvSeqLen->data), (int32_t)B,
                                      d.tq, d.kv_padded ? INT64_MAX : d.tk, d.tk, headNum,
                                      kern.unit_rows, ws, sl, ds->status, cs);
    if (e != cudaSuccess) return cuda_fail(e, "sched_prep launch");
    p.ws = ws;
    p.sl = sl;
  }
  cudaError_t e = kern.launch(p, grid, cs);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  if (n_split > 1) {
    MergeParams mp{};
    mp.parts = p.part_o;
    mp.p_ss = part_rows * d.dv;
    mp.p_sr = d.dv;
    mp.lses = p.part_lse;
    mp.l_ss = part_rows;
    mp.l_sr = 1;
    mp.n_split = n_split;
    mp.dv = (int32_t)d.dv;
    mp.rows = part_rows;
    mp.out = out->data;
    mp.out_type = elem_type(dt);
    mp.lse = p.lse;
    if (!d.varlen) {       // row = (b * H + h) * Lq + i
      mp.n1 = headNum;
      mp.n2 = d.lq;
      mp.o_s0 = p.o_sb; mp.o_s1 = p.o_sh; mp.o_s2 = p.o_si;
      mp.e_s0 = p.l_sb; mp.e_s1 = p.l_sh; mp.e_s2 = p.l_si;
    } else {               // row = token * H + h
      mp.n1 = d.tq;
      mp.n2 = headNum;
      mp.o_s1 = p.o_si; mp.o_s2 = p.o_sh;
      mp.e_s1 = p.l_si; mp.e_s2 = p.l_sh;
      mp.sched = ws;
      mp.sched_tokens = sl.cu_q + (int32_t)d.batch;
    }
    if ((e = launch_merge(mp, cs)) != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  return WF_OK;
}

wf_status_t wf_get_device_status(void *stream) {
  clear_error();
  wf_status_t st;
  DeviceState *ds = current_device_state(&st);
  if (!ds) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int32_t v = 0;
  if ((e = cudaMemcpy(&v, ds->status, sizeof(v), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "reading the device status");
  const int32_t zero = 0;
  if ((e = cudaMemcpy(ds->status, &zero, sizeof(zero), cudaMemcpyHostToDevice)) != cudaSuccess)
    return cuda_fail(e, "clearing the device status");
  if (v == kDevTimeout) {
    // Every CTA of an aborted launch still leaves the work-item counters at
    // zero; reset them anyway (all workspaces on this device and the fixed
    // arrays) so that a later call starts clean whatever the abort left.
    int dev = 0;
    cudaGetDevice(&dev);
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    {
      std::lock_guard<std::mutex> lock(g_mu);
      for (auto &kv : g_workspaces)
        if (kv.first.first == dev && kv.second.first &&
            (e = cudaMemset(kv.second.first, 0, kWorkspaceHeader)) != cudaSuccess)
          return cuda_fail(e, "resetting the workspace counters");
    }
    if ((e = reset_noalloc_counters()) != cudaSuccess) return cuda_fail(e, "resetting the fixed counters");
    return fail(WF_ERR_TIMEOUT, "a bounded device wait ran out");
  }
  if (v == kDevInvalidArg) return fail(WF_ERR_INVALID_ARG, "device-side length check failed");
  if (v != 0) return fail(WF_ERR_CUDA, "device status %d", v);
  return WF_OK;
}

const char *wf_last_error_message(void) { return g_last_error.c_str(); }

int32_t wf_version(void) { return WF_ATTN_VERSION; }

void wf_shutdown(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto &kv : g_workspaces) {
    if (kv.second.first) {
      cudaSetDevice(kv.first.first);
      cudaFree(kv.second.first);
    }
  }
  g_workspaces.clear();
  for (auto &kv : g_scratch) {
    if (kv.second.first) {
      cudaSetDevice(kv.first.first);
      cudaFree(kv.second.first);
    }
  }
  g_scratch.clear();
  // cached device addresses (status word, fixed arrays): looked up again on
  // next use, so that calls after a device reset see the new addresses
  g_devices.clear();
  g_setup_generation.fetch_add(1);
  cudaSetDevice(cur);
  forget_noalloc_addresses();
}

}  // extern "C"
