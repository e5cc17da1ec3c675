// runtime.h -- host-side helpers shared by the C-ABI translation units.
#pragma once
#include <cstdarg>
#include <cstdint>
#include <cuda_runtime.h>

#include "wf_attn.h"

namespace wf {

// Record `msg` as this thread's last error and return `st`.
wf_status_t fail(wf_status_t st, const char *fmt, ...);
void clear_error();

// CUDA error -> WF_ERR_CUDA with the call's name in the message.
wf_status_t cuda_fail(cudaError_t e, const char *what);

size_t dtype_size(int32_t dtype);

// Per-device state: SM count, status word address, schedule workspace.
struct DeviceState {
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  int32_t *status = nullptr;     // address of the device status word
  int32_t *ws = nullptr;         // schedule workspace
  size_t ws_bytes = 0;
};
// Current device's state (lazily initialised), or nullptr with the error set.
DeviceState *current_device_state(wf_status_t *st);
// Grow the current device's workspace to at least `bytes`.
wf_status_t ensure_workspace(DeviceState *ds, size_t bytes);

}  // namespace wf
