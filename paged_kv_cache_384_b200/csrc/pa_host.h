// pa_host.h -- host-side helpers shared by the library's translation units (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/pagedattn.h"

namespace pa {

// Record a message for pa_last_error() on this thread and return `st`.
pa_status fail(pa_status st, const char* fmt, ...);
// Map a CUDA error to PA_ERR_CUDA with "<what>: <cuda message>".
pa_status cuda_fail(cudaError_t err, const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device and its SM count (cached per device).  PA_ERR_CUDA if no device.
pa_status current_device(int* device, int* sm_count);

// Per-translation-unit device error words: each TU with kernels registers a reader.
using DeviceErrorReader = cudaError_t (*)(uint32_t* flags, int clear);
void register_device_error_reader(DeviceErrorReader reader);

// Launch `fn` as a programmatic dependent of the previous kernel on `stream`: it may be
// scheduled before that kernel finishes; the kernel itself must execute
// griddepcontrol.wait before touching memory the previous kernel may write.
cudaError_t launch_dependent(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             void** args);

// Profiling hooks used by paged_attention_decode.
bool profiling_enabled();
// Returns three events (before partition, between kernels, after merge) to record, or
// nullptrs when profiling is off or the event pool cannot grow.
void profiling_next_events(cudaEvent_t* ev);

}  // namespace pa
