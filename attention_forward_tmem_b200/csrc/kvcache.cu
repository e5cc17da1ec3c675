// kvcache.cu -- BlockKVCache: host-side rolling state and the ring-slot write.
//
// "Core 注意力" (WorldFoundry docs), section "Block KV cache 的调用顺序":
// every chunk goes before_update -> update -> cached_k/cached_v ->
// after_update; repeating the current chunk index overwrites the same logical
// chunk, the index plus one appends or rolls the window, a skipped index is an
// error; sink_size is a prefix that is never evicted, window_size the rolling
// region, their sum is the cache length and divisible by chunk_size.
//
// Readings where the page is silent: the first index is 0; an out-of-order
// call returns WF_ERR_ORDER and changes nothing; sink_size is a multiple of
// chunk_size and the window holds at least one chunk; update takes exactly
// chunk_size positions; chunk c lives in slot c while c < sink/chunk and in
// sink/chunk + (c - sink/chunk) mod (window/chunk) afterwards.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <type_traits>

#include "attn_params.h"
#include "runtime.h"
#include "sm100_ptx.cuh"

using namespace wf;

struct wf_kvcache {
  wf_tensor_t k, v;     // caller-owned buffers as given
  int32_t seq_dim;
  int64_t chunk, sink, window, n_sink, n_window, n_slots;
  int64_t committed, current;
  int32_t phase;        // 0 idle, 1 before_update done, 2 update done, 3 cached done
};

namespace {

enum { kIdle = 0, kBefore = 1, kUpdated = 2, kCached = 3 };

int64_t slot_of(const wf_kvcache *c, int64_t idx) {
  if (idx < c->n_sink) return idx;
  return c->n_sink + (idx - c->n_sink) % c->n_window;
}

int64_t visible_len(const wf_kvcache *c, int64_t idx) {
  const int64_t n = idx + 1 < c->n_slots ? idx + 1 : c->n_slots;
  return c->chunk * n;
}

// Logical [B, H, L, D] view of a 4-d tensor whose sequence dim is seq_dim
// (2: [B, H, L, D]; 1: [B, L, H, D]).  Strides in elements.
struct View {
  int64_t B, H, L, D;
  int64_t sb, sh, sl;
};
View logical(const wf_tensor_t *t, int32_t seq_dim) {
  View v;
  v.B = t->shape[0];
  v.sb = t->stride[0];
  v.D = t->shape[3];
  if (seq_dim == 2) {
    v.H = t->shape[1]; v.sh = t->stride[1];
    v.L = t->shape[2]; v.sl = t->stride[2];
  } else {
    v.L = t->shape[1]; v.sl = t->stride[1];
    v.H = t->shape[2]; v.sh = t->stride[2];
  }
  return v;
}

// Copy jobs: `rows` = B*H*C rows of `upr` units each, source row (b, h, t) ->
// destination row (b, h, dst_t0 + t); strides in bytes.  One launch runs up
// to two jobs (the chunk's K and V), one per grid row.
struct CopyJob {
  const uint8_t *src;
  uint8_t *dst;
  int64_t s_b, s_h, s_t, d_b, d_h, d_t, dst_t0, upr, total;
};
struct CopyJobs {
  CopyJob job[2];
  int64_t H, C;
};

// `unit` bytes (U) per element, chosen on the host so every access is aligned
// to it; each thread keeps four elements' loads in flight before it stores
// them.  kNarrow: element counts and row counts fit 32 bits, so the index
// arithmetic is 32-bit.
template <typename U, bool kNarrow>
__global__ void __launch_bounds__(256) copy_rows_kernel(const __grid_constant__ CopyJobs cj) {
  pdl_wait();
  pdl_trigger();
  const CopyJob &j = cj.job[blockIdx.y];
  using I = typename std::conditional<kNarrow, uint32_t, int64_t>::type;
  const I upr = static_cast<I>(j.upr), C = static_cast<I>(cj.C), H = static_cast<I>(cj.H);
  const I total = static_cast<I>(j.total);
  const I stride = static_cast<I>(gridDim.x) * blockDim.x;
  for (I base = static_cast<I>(blockIdx.x) * blockDim.x + threadIdx.x; base < total; base += 4 * stride) {
    U v[4];
    U *d[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const I i = base + k * stride;
      d[k] = nullptr;
      if (i < total) {
        const I row = i / upr, u = i - row * upr;
        const I t = row % C, bh = row / C;
        const I h = bh % H, b = bh / H;
        v[k] = *(reinterpret_cast<const U *>(j.src + (int64_t)b * j.s_b + (int64_t)h * j.s_h + (int64_t)t * j.s_t) + u);
        d[k] = reinterpret_cast<U *>(j.dst + (int64_t)b * j.d_b + (int64_t)h * j.d_h +
                                     (j.dst_t0 + (int64_t)t) * j.d_t) + u;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (d[k]) *d[k] = v[k];
  }
}

// One copy: C positions of every (b, h) row from src (starting at src_t0) to
// dst (starting at dst_t0); views are logical [B, H, L, D].
struct CopyReq {
  const void *src_base;
  View s;
  int64_t src_t0;
  void *dst_base;
  View d;
  int64_t dst_t0;
};

// Largest power of two (at most 16) that divides x.
int64_t gcd_pow2_unit(int64_t x) {
  for (int64_t u = 16; u > 1; u >>= 1)
    if (x % u == 0) return u;
  return 1;
}

static int64_t unit_of(const CopyReq &r, size_t es) {
  const int64_t row_bytes = r.s.D * (int64_t)es;
  int64_t unit = gcd_pow2_unit(row_bytes);
  const uint8_t *src = static_cast<const uint8_t *>(r.src_base) + r.src_t0 * r.s.sl * (int64_t)es;
  const int64_t vals[] = {(int64_t)reinterpret_cast<uintptr_t>(src),
                          (int64_t)reinterpret_cast<uintptr_t>(r.dst_base), r.s.sb * (int64_t)es,
                          r.s.sh * (int64_t)es, r.s.sl * (int64_t)es, r.d.sb * (int64_t)es,
                          r.d.sh * (int64_t)es, r.d.sl * (int64_t)es};
  for (int64_t x : vals)
    while (unit > 1 && x % unit != 0) unit >>= 1;
  return unit;
}

static CopyJob job_of(const CopyReq &r, int64_t C, size_t es, int64_t unit) {
  CopyJob j;
  j.src = static_cast<const uint8_t *>(r.src_base) + r.src_t0 * r.s.sl * (int64_t)es;
  j.dst = static_cast<uint8_t *>(r.dst_base);
  j.s_b = r.s.sb * es; j.s_h = r.s.sh * es; j.s_t = r.s.sl * es;
  j.d_b = r.d.sb * es; j.d_h = r.d.sh * es; j.d_t = r.d.sl * es;
  j.dst_t0 = r.dst_t0;
  j.upr = r.s.D * (int64_t)es / unit;
  j.total = r.s.B * r.s.H * C * j.upr;
  return j;
}

template <typename U>
static cudaError_t launch_copy(const CopyJobs &cj, int n_jobs, int64_t max_total, cudaStream_t stream) {
  const int threads = 256;
  int64_t blocks = (max_total + 4 * threads - 1) / (4 * threads);
  if (blocks > 148 * 8) blocks = 148 * 8;
  const dim3 grid((unsigned)blocks, (unsigned)n_jobs);
  const bool narrow = max_total < (int64_t(1) << 31) && cj.C < (int64_t(1) << 31) && cj.H < (int64_t(1) << 31);
  if (narrow) return launch_pdl(copy_rows_kernel<U, true>, grid, dim3(threads), 0, stream, cj);
  return launch_pdl(copy_rows_kernel<U, false>, grid, dim3(threads), 0, stream, cj);
}

// Copy one or two requests (K and V of a chunk) of C positions each; both in
// one launch when their element sizes agree, else one launch each.
wf_status_t copy_positions(const CopyReq *reqs, int n, int64_t C, size_t es, cudaStream_t stream) {
  CopyReq live[2];
  int m = 0;
  for (int i = 0; i < n; ++i)
    if (reqs[i].s.B * reqs[i].s.H * C > 0 && reqs[i].s.D > 0) live[m++] = reqs[i];
  if (m == 0) return WF_OK;
  int64_t units[2] = {unit_of(live[0], es), m > 1 ? unit_of(live[1], es) : 0};
  const bool together = m == 2 && units[0] == units[1];
  for (int first = 0; first < m; first += together ? 2 : 1) {
    const int cnt = together ? 2 : 1;
    const int64_t unit = units[first];
    CopyJobs cj{};
    cj.H = live[first].s.H;
    cj.C = C;
    int64_t max_total = 0;
    for (int k = 0; k < cnt; ++k) {
      cj.job[k] = job_of(live[first + k], C, es, unit);
      max_total = std::max(max_total, cj.job[k].total);
    }
    cudaError_t e;
    switch (unit) {
      case 16: e = launch_copy<uint4>(cj, cnt, max_total, stream); break;
      case 8: e = launch_copy<uint2>(cj, cnt, max_total, stream); break;
      case 4: e = launch_copy<uint32_t>(cj, cnt, max_total, stream); break;
      case 2: e = launch_copy<uint16_t>(cj, cnt, max_total, stream); break;
      default: e = launch_copy<uint8_t>(cj, cnt, max_total, stream); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "cache copy launch");
  }
  return WF_OK;
}

wf_status_t check_buf(const wf_tensor_t *t, const char *name) {
  if (!t) return fail(WF_ERR_INVALID_ARG, "%s is NULL", name);
  if (t->ndim != 4) return fail(WF_ERR_INVALID_ARG, "%s must have 4 dims", name);
  if (dtype_size(t->dtype) == 0) return fail(WF_ERR_INVALID_ARG, "%s: unknown dtype %d", name, t->dtype);
  for (int i = 0; i < 4; ++i)
    if (t->shape[i] <= 0) return fail(WF_ERR_INVALID_ARG, "%s: dim %d must be positive", name, i);
  if (t->stride[3] != 1 && t->shape[3] > 1)
    return fail(WF_ERR_INVALID_ARG, "%s: last dimension must be contiguous", name);
  if (!t->data) return fail(WF_ERR_INVALID_ARG, "%s: NULL data", name);
  return WF_OK;
}

// Same shape as the buffer except `seq_extent` positions along seq_dim.
wf_status_t check_like(const wf_tensor_t *t, const wf_tensor_t *buf, int32_t seq_dim,
                       int64_t seq_extent, const char *name) {
  if (!t) return fail(WF_ERR_INVALID_ARG, "%s is NULL", name);
  if (t->ndim != 4 || t->dtype != buf->dtype)
    return fail(WF_ERR_INVALID_ARG, "%s: must be 4-d with the buffer's dtype", name);
  for (int i = 0; i < 4; ++i) {
    const int64_t want = (i == seq_dim) ? seq_extent : buf->shape[i];
    if (t->shape[i] != want)
      return fail(WF_ERR_INVALID_ARG, "%s: dim %d is %lld, expected %lld", name, i,
                  (long long)t->shape[i], (long long)want);
  }
  if (t->stride[3] != 1 && t->shape[3] > 1)
    return fail(WF_ERR_INVALID_ARG, "%s: last dimension must be contiguous", name);
  if (!t->data) return fail(WF_ERR_INVALID_ARG, "%s: NULL data", name);
  return WF_OK;
}

}  // namespace

extern "C" {

wf_status_t wf_kvcache_create(const wf_tensor_t *k_buf, const wf_tensor_t *v_buf, int32_t seq_dim,
                              int64_t chunk_size, int64_t sink_size, int64_t window_size,
                              wf_kvcache_t **out) {
  clear_error();
  wf_status_t st;
  if (!out) return fail(WF_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if ((st = check_buf(k_buf, "k_buf")) != WF_OK) return st;
  if ((st = check_buf(v_buf, "v_buf")) != WF_OK) return st;
  if (seq_dim != 1 && seq_dim != 2) return fail(WF_ERR_INVALID_ARG, "seq_dim must be 1 or 2");
  if (k_buf->dtype != v_buf->dtype) return fail(WF_ERR_INVALID_ARG, "k_buf and v_buf dtypes differ");
  for (int i = 0; i < 3; ++i)
    if (k_buf->shape[i] != v_buf->shape[i])
      return fail(WF_ERR_INVALID_ARG, "k_buf and v_buf differ in dim %d", i);
  const int64_t L = k_buf->shape[seq_dim];
  if (chunk_size <= 0 || sink_size < 0 || window_size < 0)
    return fail(WF_ERR_INVALID_ARG, "chunk_size must be positive, sink/window non-negative");
  if (sink_size + window_size != L)
    return fail(WF_ERR_INVALID_ARG, "sink_size + window_size (%lld) must equal the cache length %lld",
                (long long)(sink_size + window_size), (long long)L);
  if (L % chunk_size != 0) return fail(WF_ERR_INVALID_ARG, "cache length is not divisible by chunk_size");
  if (sink_size % chunk_size != 0) return fail(WF_ERR_INVALID_ARG, "sink_size must be a multiple of chunk_size");
  if (window_size < chunk_size) return fail(WF_ERR_INVALID_ARG, "the window must hold at least one chunk");
  wf_kvcache *c = new (std::nothrow) wf_kvcache;
  if (!c) return fail(WF_ERR_NO_MEMORY, "host allocation failed");
  c->k = *k_buf;
  c->v = *v_buf;
  c->seq_dim = seq_dim;
  c->chunk = chunk_size;
  c->sink = sink_size;
  c->window = window_size;
  c->n_sink = sink_size / chunk_size;
  c->n_window = window_size / chunk_size;
  c->n_slots = c->n_sink + c->n_window;
  c->committed = -1;
  c->current = -1;
  c->phase = kIdle;
  *out = c;
  return WF_OK;
}

wf_status_t wf_kvcache_before_update(wf_kvcache_t *c, int64_t idx) {
  clear_error();
  if (!c) return fail(WF_ERR_INVALID_ARG, "cache is NULL");
  if (c->phase != kIdle) return fail(WF_ERR_ORDER, "before_update while chunk %lld is in progress", (long long)c->current);
  const bool ok = c->committed < 0 ? idx == 0 : (idx == c->committed || idx == c->committed + 1);
  if (!ok)
    return fail(WF_ERR_ORDER, "chunk index %lld cannot follow %lld (repeat or +1 only, first is 0)",
                (long long)idx, (long long)c->committed);
  c->current = idx;
  c->phase = kBefore;
  return WF_OK;
}

wf_status_t wf_kvcache_update(wf_kvcache_t *c, const wf_tensor_t *k, const wf_tensor_t *v, void *stream) {
  clear_error();
  wf_status_t st;
  if (!c) return fail(WF_ERR_INVALID_ARG, "cache is NULL");
  if (c->phase != kBefore) return fail(WF_ERR_ORDER, "update without before_update");
  if ((st = check_like(k, &c->k, c->seq_dim, c->chunk, "k")) != WF_OK) return st;
  if ((st = check_like(v, &c->v, c->seq_dim, c->chunk, "v")) != WF_OK) return st;
  const int64_t t0 = slot_of(c, c->current) * c->chunk;
  const size_t es = dtype_size(c->k.dtype);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  {
    const CopyReq reqs[2] = {{k->data, logical(k, c->seq_dim), 0, c->k.data, logical(&c->k, c->seq_dim), t0},
                             {v->data, logical(v, c->seq_dim), 0, c->v.data, logical(&c->v, c->seq_dim), t0}};
    if ((st = copy_positions(reqs, 2, c->chunk, es, cs)) != WF_OK) return st;
  }
  c->phase = kUpdated;
  return WF_OK;
}

static void make_view(const wf_tensor_t *buf, int32_t seq_dim, int64_t vis, wf_tensor_t *out) {
  View lv = logical(buf, seq_dim);
  out->data = buf->data;
  out->dtype = buf->dtype;
  out->ndim = 4;
  out->shape[0] = lv.B; out->stride[0] = lv.sb;
  out->shape[1] = lv.H; out->stride[1] = lv.sh;
  out->shape[2] = vis;  out->stride[2] = lv.sl;
  out->shape[3] = lv.D; out->stride[3] = buf->stride[3];
}

wf_status_t wf_kvcache_update_attend(wf_kvcache_t *c, const wf_tensor_t *k, const wf_tensor_t *v,
                                     const wf_tensor_t *q, int32_t headNum, float qkScale,
                                     wf_tensor_t *out, void *stream) {
  clear_error();
  wf_status_t st;
  if (!c) return fail(WF_ERR_INVALID_ARG, "cache is NULL");
  if (c->phase != kBefore) return fail(WF_ERR_ORDER, "update_attend without before_update");
  if ((st = check_like(k, &c->k, c->seq_dim, c->chunk, "k")) != WF_OK) return st;
  if ((st = check_like(v, &c->v, c->seq_dim, c->chunk, "v")) != WF_OK) return st;
  const int64_t vis = visible_len(c, c->current);
  wf_tensor_t kv, vv, kc, vc;
  make_view(&c->k, c->seq_dim, vis, &kv);
  make_view(&c->v, c->seq_dim, vis, &vv);
  make_view(k, c->seq_dim, c->chunk, &kc);      // the chunk in the logical [B, H, C, D] layout
  make_view(v, c->seq_dim, c->chunk, &vc);
  const int64_t lo = slot_of(c, c->current) * c->chunk;
  const int32_t kv_heads = (int32_t)kv.shape[1];
  bool declined = false;
  st = attn_fwd_fused(q, &kv, &vv, &kc, &vc, lo, lo + c->chunk, headNum, kv_heads, qkScale, out, stream,
                      &declined);
  if (st != WF_OK) return st;                   // argument error: nothing written
  if (declined) {                               // not fusable: the copies, then the attention
    const size_t es = dtype_size(c->k.dtype);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const CopyReq reqs[2] = {{k->data, logical(k, c->seq_dim), 0, c->k.data, logical(&c->k, c->seq_dim), lo},
                             {v->data, logical(v, c->seq_dim), 0, c->v.data, logical(&c->v, c->seq_dim), lo}};
    if ((st = copy_positions(reqs, 2, c->chunk, es, cs)) != WF_OK) return st;
    if ((st = wf_attn_fwd(q, nullptr, &kv, nullptr, &vv, nullptr, nullptr, nullptr, headNum, kv_heads,
                          qkScale, WF_MASK_NONE, out, stream)) != WF_OK)
      return st;
  }
  c->phase = kCached;
  return WF_OK;
}

wf_status_t wf_kvcache_cached(wf_kvcache_t *c, wf_tensor_t *k_view, wf_tensor_t *v_view, int64_t *visible) {
  clear_error();
  if (!c) return fail(WF_ERR_INVALID_ARG, "cache is NULL");
  if (c->phase != kUpdated && c->phase != kCached) return fail(WF_ERR_ORDER, "cached before update");
  const int64_t vis = visible_len(c, c->current);
  if (k_view) make_view(&c->k, c->seq_dim, vis, k_view);
  if (v_view) make_view(&c->v, c->seq_dim, vis, v_view);
  if (visible) *visible = vis;
  c->phase = kCached;
  return WF_OK;
}

wf_status_t wf_kvcache_after_update(wf_kvcache_t *c, int64_t idx) {
  clear_error();
  if (!c) return fail(WF_ERR_INVALID_ARG, "cache is NULL");
  if (c->phase != kCached) return fail(WF_ERR_ORDER, "after_update before cached_k / cached_v");
  if (idx != c->current)
    return fail(WF_ERR_ORDER, "after_update(%lld) while chunk %lld is in progress", (long long)idx,
                (long long)c->current);
  c->committed = idx;
  c->phase = kIdle;
  return WF_OK;
}

wf_status_t wf_kvcache_get_state(const wf_kvcache_t *c, int64_t *cur, int64_t *committed,
                                 int64_t *slot, int64_t *visible, int32_t *phase) {
  clear_error();
  if (!c) return fail(WF_ERR_INVALID_ARG, "cache is NULL");
  if (cur) *cur = c->current;
  if (committed) *committed = c->committed;
  if (slot) *slot = c->current >= 0 ? slot_of(c, c->current) : -1;
  if (visible) {
    if (c->phase == kUpdated || c->phase == kCached) *visible = visible_len(c, c->current);
    else *visible = c->committed >= 0 ? visible_len(c, c->committed) : 0;
  }
  if (phase) *phase = c->phase;
  return WF_OK;
}

wf_status_t wf_kvcache_set_state(wf_kvcache_t *c, int64_t committed) {
  clear_error();
  if (!c) return fail(WF_ERR_INVALID_ARG, "cache is NULL");
  if (c->phase != kIdle)
    return fail(WF_ERR_ORDER, "set_state while chunk %lld is in progress", (long long)c->current);
  if (committed < -1) return fail(WF_ERR_INVALID_ARG, "committed index %lld < -1", (long long)committed);
  c->committed = committed;
  c->current = committed;
  return WF_OK;
}

wf_status_t wf_kvcache_gather_logical(wf_kvcache_t *c, wf_tensor_t *k_out, wf_tensor_t *v_out, void *stream) {
  clear_error();
  wf_status_t st;
  if (!c) return fail(WF_ERR_INVALID_ARG, "cache is NULL");
  if (c->phase != kUpdated && c->phase != kCached) return fail(WF_ERR_ORDER, "gather before update");
  const int64_t vis = visible_len(c, c->current);
  if ((st = check_like(k_out, &c->k, c->seq_dim, vis, "k_out")) != WF_OK) return st;
  if ((st = check_like(v_out, &c->v, c->seq_dim, vis, "v_out")) != WF_OK) return st;
  const size_t es = dtype_size(c->k.dtype);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // logical order: sink chunks, then the window's chunks oldest first
  const int64_t cur = c->current;
  int64_t pos = 0;
  auto emit = [&](int64_t idx) -> wf_status_t {
    const int64_t src_t0 = slot_of(c, idx) * c->chunk;
    const CopyReq reqs[2] = {
        {c->k.data, logical(&c->k, c->seq_dim), src_t0, k_out->data, logical(k_out, c->seq_dim), pos * c->chunk},
        {c->v.data, logical(&c->v, c->seq_dim), src_t0, v_out->data, logical(v_out, c->seq_dim), pos * c->chunk}};
    wf_status_t s2 = copy_positions(reqs, 2, c->chunk, es, cs);
    ++pos;
    return s2;
  };
  const int64_t sink_end = cur + 1 < c->n_sink ? cur + 1 : c->n_sink;
  for (int64_t i = 0; i < sink_end; ++i)
    if ((st = emit(i)) != WF_OK) return st;
  int64_t first = cur - c->n_window + 1;
  if (first < c->n_sink) first = c->n_sink;
  for (int64_t i = first; i <= cur; ++i)
    if ((st = emit(i)) != WF_OK) return st;
  return WF_OK;
}

void wf_kvcache_destroy(wf_kvcache_t *c) { delete c; }

}  // extern "C"
