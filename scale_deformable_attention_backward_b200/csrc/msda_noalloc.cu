// msda_noalloc.cu -- msda_backward_noalloc: the cell-sorted backward with its
// scratch in a fixed device array that the library owns, for callers that cannot
// allocate device memory when they call the op.
//
// Such callers exist: a host framework that owns the whole device memory pool and
// lets no other allocator in, or code on a latency-critical path where
// cudaMalloc / cudaFree would block or synchronize the device.  They pass inputs
// and outputs; the scratch the sorted backward needs (msda_backward_workspace_size
// bytes) comes from `noalloc_scratch` below, which every device that loads this
// library holds until the process exits.
#include <cstdint>
#include <cuda_runtime.h>

#include "msda.h"

namespace {

// The scratch: one copy per device, reserved when the library's module is loaded
// there.
static __device__ __align__(256) unsigned char noalloc_scratch[MSDA_NOALLOC_SCRATCH_BYTES];

// In host code `noalloc_scratch` names a host-side stand-in, not device memory,
// so its device address is looked up with the device current.  The lookup runs
// on every call: it allocates nothing once the module is loaded, and the
// address it returns always belongs to the current context (a cached one would
// not survive cudaDeviceReset or a switch to another context).
msda_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, noalloc_scratch) != cudaSuccess || p == nullptr)
    return MSDA_ERR_CUDA;
  *out = p;
  return MSDA_OK;
}

}  // namespace

extern "C" msda_status msda_backward_noalloc(
    int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq, int64_t L, int64_t K,
    msda_dtype value_dtype, const void* value, const int64_t* spatial_shapes,
    const int64_t* level_start_index, const float* sampling_locations,
    const float* attention_weights, const float* grad_output, float* grad_value,
    float* grad_sampling_locations, float* grad_attention_weights, void* stream) {
  // The cell-sorted path behind this entry point is float32 only.
  if (value_dtype != MSDA_F32) return MSDA_ERR_UNSUPPORTED;
  size_t need = 0;
  msda_status st = msda_backward_workspace_size(B, S, M, D, Lq, L, K, &need);
  if (st != MSDA_OK) return st;
  if (need > MSDA_NOALLOC_SCRATCH_BYTES) return MSDA_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != MSDA_OK) return st;
  return msda_backward(B, S, M, D, Lq, L, K, value_dtype, value, spatial_shapes,
                       level_start_index, sampling_locations, attention_weights, grad_output,
                       grad_value, grad_sampling_locations, grad_attention_weights, scratch,
                       MSDA_NOALLOC_SCRATCH_BYTES, stream);
}
