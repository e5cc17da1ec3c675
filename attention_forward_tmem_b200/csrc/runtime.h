// runtime.h -- host-side helpers shared by the C-ABI translation units.
#pragma once
#include <cstdarg>
#include <cstdint>
#include <cuda_runtime.h>

#include <cuda.h>

#include "wf_attn.h"

namespace wf {

// Record `msg` as this thread's last error and return `st`.
wf_status_t fail(wf_status_t st, const char *fmt, ...);
void clear_error();

// CUDA error -> WF_ERR_CUDA with the call's name in the message.
wf_status_t cuda_fail(cudaError_t e, const char *what);

size_t dtype_size(int32_t dtype);

// Per-device state: SM count, status word address.
struct DeviceState {
  int sm_count = 0;
  int l2_bytes = 0;
  int cc_major = 0, cc_minor = 0;
  int32_t *status = nullptr;     // address of the device status word
};
// Current device's state (lazily initialised), or nullptr with the error set.
DeviceState *current_device_state(wf_status_t *st);
// Tensor helpers shared by the entry points (runtime.cu).
wf_status_t check_tensor(const wf_tensor_t *t, const char *name, int ndim, int32_t dtype,
                         bool need_tma_layout);
int64_t numel(const wf_tensor_t *t);

// Attention over a cache view whose key rows [lo, hi) are the new chunk
// k_chunk / v_chunk ([B, Hkv, hi - lo, D], logical layout), which the kernel
// reads from there and also stores into the view's rows (fused cache write).
// Needs the dense layout, no mask, no rope, 16-bit types and lo, hi multiples
// of 128: otherwise, with arguments that are valid for plain attention, it
// launches nothing, sets *declined and returns WF_OK.
wf_status_t attn_fwd_fused(const wf_tensor_t *q, const wf_tensor_t *k_view, const wf_tensor_t *v_view,
                           const wf_tensor_t *k_chunk, const wf_tensor_t *v_chunk, int64_t lo,
                           int64_t hi, int32_t headNum, int32_t kvHeadNum, float qkScale,
                           wf_tensor_t *out, void *stream, bool *declined);
// Per-(device, stream) scratch for calls that compose several attention calls;
// grown on demand (synchronizing the stream first), freed by wf_shutdown.
wf_status_t stream_scratch(cudaStream_t stream, size_t bytes, void **out);
// Element type code (ElemType) of a wf_dtype_t.
int32_t elem_type_of(int32_t dtype);
// Fill n floats with v (device, asynchronous).
cudaError_t launch_fill_f32(float *dst, int64_t n, float v, cudaStream_t stream);

// Zero the allocation-free entry's work-item counters on the current device
// (noalloc.cu); used after a launch was aborted.
cudaError_t reset_noalloc_counters();
// Forget the fixed arrays' device addresses (looked up again on next use).
void forget_noalloc_addresses();
// 4-d TMA map (D, rows, heads, batch), (128 bytes of D) x 128 rows box,
// 128-byte swizzle, zero fill outside the tensor; strides in elements.
wf_status_t make_map(CUtensorMap *map, const void *base, int32_t dtype, int64_t d, int64_t rows,
                     int64_t heads, int64_t batch, int64_t s_row, int64_t s_head, int64_t s_batch,
                     const char *name, int32_t box_rows = 128);

}  // namespace wf
