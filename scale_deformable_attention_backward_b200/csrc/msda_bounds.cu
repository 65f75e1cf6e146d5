// msda_bounds.cu -- the bounds checks of the debug build (MSDA_DEBUG_BOUNDS,
// libmsda_debug.so): the buffers each call registers for the kernels' checks
// (in_bounds, msda_device.cuh), the record of the first refused access, and the
// two entry points that read the record and clip the registered buffers.  The
// release build compiles the same entry points to MSDA_ERR_UNSUPPORTED and
// arm_bounds to nothing.
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "msda.h"
#include "msda_device.cuh"
#include "msda_launch.h"

namespace msda {

#ifdef MSDA_DEBUG_BOUNDS

__device__ BoundsRanges bounds_ranges;
__device__ unsigned long long bounds_error;

namespace {
// msda_debug_bounds_clip's caps on the value and grad_value buffers (0: none).
std::atomic<unsigned long long> clip_value{0}, clip_grad_value{0};

void set_range(BoundsRanges& r, int i, const void* p, long long bytes, unsigned long long cap) {
  if (p == nullptr || bytes <= 0) return;
  unsigned long long n = static_cast<unsigned long long>(bytes);
  if (cap != 0 && cap < n) n = cap;
  r.lo[i] = reinterpret_cast<unsigned long long>(p);
  r.hi[i] = r.lo[i] + n;
}
}  // namespace

cudaError_t arm_bounds(const void* value, long long value_bytes, const void* grad_output,
                       long long grad_output_bytes, const void* grad_value,
                       long long grad_value_bytes, const void* workspace,
                       long long workspace_bytes, cudaStream_t stream) {
  BoundsRanges r{};
  set_range(r, 0, value, value_bytes, clip_value.load());
  set_range(r, 1, grad_output, grad_output_bytes, 0);
  set_range(r, 2, grad_value, grad_value_bytes, clip_grad_value.load());
  set_range(r, 3, workspace, workspace_bytes, 0);
  // From pageable host memory: the copy is staged before this call returns.
  return cudaMemcpyToSymbolAsync(bounds_ranges, &r, sizeof(r), 0, cudaMemcpyHostToDevice, stream);
}

#else

cudaError_t arm_bounds(const void*, long long, const void*, long long, const void*, long long,
                       const void*, long long, cudaStream_t) {
  return cudaSuccess;
}

#endif

}  // namespace msda

extern "C" msda_status msda_debug_bounds_check(int* kind, uint64_t* address) {
  if (kind == nullptr || address == nullptr) return MSDA_ERR_NULL_POINTER;
  *kind = 0;
  *address = 0;
#ifdef MSDA_DEBUG_BOUNDS
  unsigned long long rec = 0;
  if (cudaMemcpyFromSymbol(&rec, msda::bounds_error, sizeof(rec)) != cudaSuccess)
    return MSDA_ERR_CUDA;
  const unsigned long long zero = 0;
  if (cudaMemcpyToSymbol(msda::bounds_error, &zero, sizeof(zero)) != cudaSuccess)
    return MSDA_ERR_CUDA;
  *kind = static_cast<int>(rec >> 60);
  *address = rec & ((1ull << 60) - 1);
  return MSDA_OK;
#else
  return MSDA_ERR_UNSUPPORTED;
#endif
}

extern "C" msda_status msda_debug_bounds_clip(uint64_t value_bytes, uint64_t grad_value_bytes) {
#ifdef MSDA_DEBUG_BOUNDS
  msda::clip_value.store(value_bytes);
  msda::clip_grad_value.store(grad_value_bytes);
  return MSDA_OK;
#else
  (void)value_bytes;
  (void)grad_value_bytes;
  return MSDA_ERR_UNSUPPORTED;
#endif
}
