// msda_api.cu -- the C ABI declared in include/msda.h: argument validation on
// the host, then one launch sequence on the caller's stream.  No allocation,
// no state, no host synchronisation (except the opt-in MSDA_VALIDATE=1 check,
// which copies the two small metadata arrays to the host).  The debug build
// (MSDA_DEBUG_BOUNDS) first registers each call's buffers for its bounds
// checks (arm_bounds, one small stream-ordered copy).
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <cuda_runtime.h>

#include "msda.h"
#include "msda_launch.h"

namespace {

constexpr int64_t kLimit = int64_t(1) << 62;

// a * b * ... without overflow; false if the product reaches kLimit.
bool product_ok(std::initializer_list<int64_t> xs, int64_t* out) {
  int64_t p = 1;
  for (int64_t x : xs) {
    if (x == 0) {
      *out = 0;
      return true;
    }
  }
  for (int64_t x : xs) {
    if (p > kLimit / x) return false;
    p *= x;
  }
  *out = p;
  return true;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int pow2_at_least(int64_t n) {
  int p = 1;
  while (p < n && p < 32) p <<= 1;
  return p;
}

bool validate_env() {
  static const bool on = [] {
    const char* v = std::getenv("MSDA_VALIDATE");
    return v != nullptr && v[0] != '\0' && std::strcmp(v, "0") != 0;
  }();
  return on;
}

// Host check of device metadata, only when MSDA_VALIDATE is set.
msda_status check_device_metadata(int64_t S, int64_t L, const int64_t* shapes,
                                  const int64_t* starts) {
  int64_t hs[2 * msda::kMaxLevels], hl[msda::kMaxLevels];
  if (cudaMemcpy(hs, shapes, sizeof(int64_t) * 2 * L, cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(hl, starts, sizeof(int64_t) * L, cudaMemcpyDeviceToHost) != cudaSuccess)
    return MSDA_ERR_CUDA;
  return msda_check_metadata(S, L, hs, hl);
}

struct Common {
  int64_t value_elems = 0, point_elems = 0, out_elems = 0;
};

msda_status check_common(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq, int64_t L,
                         int64_t K, Common* c) {
  if (B < 0 || S < 0 || M < 0 || D < 0 || Lq < 0 || L < 0 || K < 0) return MSDA_ERR_BAD_SHAPE;
  if (L < 1 || L > msda::kMaxLevels || K < 1 || K > msda::kMaxPoints) return MSDA_ERR_UNSUPPORTED;
  if (!product_ok({B, S, M, D}, &c->value_elems) ||
      !product_ok({B, Lq, M, L, K, 2}, &c->point_elems) ||
      !product_ok({B, Lq, M, D}, &c->out_elems))
    return MSDA_ERR_BAD_SHAPE;
  // The kernels address one image's value block [S, M, D] with 32-bit offsets.
  int64_t per_image = 0;
  if (!product_ok({S, M, D}, &per_image) || per_image >= (int64_t(1) << 31))
    return MSDA_ERR_UNSUPPORTED;
  return MSDA_OK;
}

msda_status output_projection(int64_t rows, int64_t c_in, int64_t c_out, const float* x,
                              const float* weight, const float* bias, float* y, bool precise,
                              void* stream) {
  if (rows < 0 || c_in < 0 || c_out < 0) return MSDA_ERR_BAD_SHAPE;
  if (c_in % 8 != 0 || c_in < 8 || c_in > 4096 || c_out % 16 != 0 || c_out < 16 ||
      c_out > 256 || rows > static_cast<int64_t>(INT32_MAX) - 128)
    return MSDA_ERR_UNSUPPORTED;
  int64_t xe = 0, ye = 0;
  if (!product_ok({rows, c_in}, &xe) || !product_ok({rows, c_out}, &ye))
    return MSDA_ERR_BAD_SHAPE;
  if (rows == 0) return MSDA_OK;
  if (x == nullptr || weight == nullptr || y == nullptr) return MSDA_ERR_NULL_POINTER;
  if (!aligned(x, 16) || !aligned(weight, 16) || !aligned(y, 16) || !aligned(bias, 4))
    return MSDA_ERR_MISALIGNED;
  return msda::launch_projection(x, weight, bias, y, rows, static_cast<int>(c_in),
                                 static_cast<int>(c_out), precise,
                                 static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MSDA_OK
             : MSDA_ERR_CUDA;
}

}  // namespace

extern "C" {

msda_status msda_forward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq, int64_t L,
                         int64_t K, msda_dtype value_dtype, const void* value,
                         const int64_t* spatial_shapes, const int64_t* level_start_index,
                         const float* sampling_locations, const float* attention_weights,
                         void* output, void* stream) {
  Common c;
  msda_status st = check_common(B, S, M, D, Lq, L, K, &c);
  if (st != MSDA_OK) return st;
  if (value_dtype != MSDA_F32 && value_dtype != MSDA_BF16) return MSDA_ERR_UNSUPPORTED;
  const int E = value_dtype == MSDA_F32 ? 4 : 8;
  if (D % E != 0 || M > INT32_MAX || D > INT32_MAX) return MSDA_ERR_UNSUPPORTED;
  if (c.out_elems == 0) return MSDA_OK;
  if ((c.value_elems > 0 && value == nullptr) || spatial_shapes == nullptr ||
      level_start_index == nullptr || sampling_locations == nullptr ||
      attention_weights == nullptr || output == nullptr)
    return MSDA_ERR_NULL_POINTER;
  if (!aligned(value, 16) || !aligned(output, 16) || !aligned(sampling_locations, 8) ||
      !aligned(attention_weights, 4) || !aligned(spatial_shapes, 8) ||
      !aligned(level_start_index, 8))
    return MSDA_ERR_MISALIGNED;
  if (validate_env()) {
    st = check_device_metadata(S, L, spatial_shapes, level_start_index);
    if (st != MSDA_OK) return st;
  }
  msda::ForwardArgs a;
  a.value = value;
  a.spatial_shapes = spatial_shapes;
  a.level_start_index = level_start_index;
  a.sampling_locations = sampling_locations;
  a.attention_weights = attention_weights;
  a.output = output;
  a.B = B;
  a.S = S;
  a.Lq = Lq;
  a.M = static_cast<int>(M);
  a.D = static_cast<int>(D);
  a.L = static_cast<int>(L);
  a.K = static_cast<int>(K);
  a.bf16 = value_dtype == MSDA_BF16;
  const int64_t nvec = D / E;
  a.lanes = pow2_at_least(nvec);
  a.chunks = static_cast<int>((nvec + a.lanes - 1) / a.lanes);
  a.groups = B * Lq * M * a.chunks;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (msda::arm_bounds(value, c.value_elems * (a.bf16 ? 2 : 4), nullptr, 0, nullptr, 0, nullptr,
                       0, s) != cudaSuccess)
    return MSDA_ERR_CUDA;
  return msda::launch_forward(a, s) == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

msda_status msda_backward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq, int64_t L,
                          int64_t K, msda_dtype value_dtype, const void* value,
                          const int64_t* spatial_shapes, const int64_t* level_start_index,
                          const float* sampling_locations, const float* attention_weights,
                          const void* grad_output, float* grad_value,
                          float* grad_sampling_locations, float* grad_attention_weights,
                          void* workspace, size_t workspace_bytes, void* stream) {
  Common c;
  msda_status st = check_common(B, S, M, D, Lq, L, K, &c);
  if (st != MSDA_OK) return st;
  // bfloat16 value / grad_output: scratch-free path only.
  if (value_dtype != MSDA_F32 && !(value_dtype == MSDA_BF16 && workspace == nullptr))
    return MSDA_ERR_UNSUPPORTED;
  const uintptr_t in_align = value_dtype == MSDA_F32 ? 16 : 8;
  if (D % 4 != 0 || D > 256 || M > INT32_MAX) return MSDA_ERR_UNSUPPORTED;
  // The cell-sorted path holds a head's channels in one sub-warp: D <= 128.
  if (workspace != nullptr && D > 128) return MSDA_ERR_UNSUPPORTED;
  if (workspace != nullptr) {
    size_t need = 0;
    st = msda_backward_workspace_size(B, S, M, D, Lq, L, K, &need);
    if (st != MSDA_OK) return st;
    if (workspace_bytes < need) return MSDA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return MSDA_ERR_MISALIGNED;
  }
  if (c.value_elems == 0 && c.out_elems == 0) return MSDA_OK;
  if (c.value_elems > 0 && grad_value == nullptr) return MSDA_ERR_NULL_POINTER;
  if (!aligned(grad_value, 16)) return MSDA_ERR_MISALIGNED;
  const bool work = c.out_elems > 0;
  if (work && (value == nullptr || spatial_shapes == nullptr || level_start_index == nullptr ||
               sampling_locations == nullptr || attention_weights == nullptr ||
               grad_output == nullptr || grad_sampling_locations == nullptr ||
               grad_attention_weights == nullptr))
    return MSDA_ERR_NULL_POINTER;
  if (work && (!aligned(value, in_align) || !aligned(grad_output, in_align) ||
               !aligned(sampling_locations, 8) || !aligned(grad_sampling_locations, 8) ||
               !aligned(attention_weights, 4) || !aligned(grad_attention_weights, 4) ||
               !aligned(spatial_shapes, 8) || !aligned(level_start_index, 8)))
    return MSDA_ERR_MISALIGNED;
  if (work && validate_env()) {
    st = check_device_metadata(S, L, spatial_shapes, level_start_index);
    if (st != MSDA_OK) return st;
  }
  msda::BackwardArgs a;
  a.value = value;
  a.bf16 = value_dtype == MSDA_BF16;
  a.spatial_shapes = spatial_shapes;
  a.level_start_index = level_start_index;
  a.sampling_locations = sampling_locations;
  a.attention_weights = attention_weights;
  a.grad_output = grad_output;
  a.grad_value = grad_value;
  a.grad_sampling_locations = grad_sampling_locations;
  a.grad_attention_weights = grad_attention_weights;
  a.B = B;
  a.S = S;
  a.Lq = Lq;
  a.M = static_cast<int>(M);
  a.D = static_cast<int>(D);
  a.L = static_cast<int>(L);
  a.K = static_cast<int>(K);
  // Lanes of one channel pass (at most 128 channels; wider heads run as passes).
  a.lanes = pow2_at_least((D > 128 ? 128 : D) / 4);
  a.groups = work ? B * Lq * M : 0;
  a.value_elements = c.value_elems;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long in_bytes = a.bf16 ? 2 : 4;
  if (msda::arm_bounds(value, c.value_elems * in_bytes, grad_output, c.out_elems * in_bytes,
                       grad_value, c.value_elems * 4, workspace,
                       static_cast<long long>(workspace != nullptr ? workspace_bytes : 0),
                       s) != cudaSuccess)
    return MSDA_ERR_CUDA;
  const cudaError_t err = workspace != nullptr ? msda::launch_backward_sorted(a, workspace, s)
                                               : msda::launch_backward(a, s);
  return err == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

msda_status msda_backward_deterministic_workspace_size(int64_t B, int64_t S, int64_t M,
                                                       int64_t D, int64_t Lq, int64_t L,
                                                       int64_t K, size_t* bytes) {
  if (bytes == nullptr) return MSDA_ERR_NULL_POINTER;
  *bytes = 0;
  Common c;
  const msda_status st = check_common(B, S, M, D, Lq, L, K, &c);
  if (st != MSDA_OK) return st;
  if (c.value_elems > (kLimit - msda::kFixedHeaderBytes) / 8) return MSDA_ERR_UNSUPPORTED;
  *bytes = static_cast<size_t>(msda::kFixedHeaderBytes + 8 * c.value_elems);
  return MSDA_OK;
}

msda_status msda_backward_deterministic(int64_t B, int64_t S, int64_t M, int64_t D,
                                        int64_t Lq, int64_t L, int64_t K,
                                        msda_dtype value_dtype, const void* value,
                                        const int64_t* spatial_shapes,
                                        const int64_t* level_start_index,
                                        const float* sampling_locations,
                                        const float* attention_weights,
                                        const void* grad_output, float* grad_value,
                                        float* grad_sampling_locations,
                                        float* grad_attention_weights, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  Common c;
  msda_status st = check_common(B, S, M, D, Lq, L, K, &c);
  if (st != MSDA_OK) return st;
  if (value_dtype != MSDA_F32 && value_dtype != MSDA_BF16) return MSDA_ERR_UNSUPPORTED;
  if (D % 4 != 0 || D > 128 || M > INT32_MAX) return MSDA_ERR_UNSUPPORTED;
  size_t need = 0;
  st = msda_backward_deterministic_workspace_size(B, S, M, D, Lq, L, K, &need);
  if (st != MSDA_OK) return st;
  if (c.value_elems == 0 && c.out_elems == 0) return MSDA_OK;
  if (workspace == nullptr) return MSDA_ERR_NULL_POINTER;
  if (workspace_bytes < need) return MSDA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return MSDA_ERR_MISALIGNED;
  const uintptr_t in_align = value_dtype == MSDA_F32 ? 16 : 8;
  if (c.value_elems > 0 && grad_value == nullptr) return MSDA_ERR_NULL_POINTER;
  if (!aligned(grad_value, 16)) return MSDA_ERR_MISALIGNED;
  const bool work = c.out_elems > 0;
  if (work && (value == nullptr || spatial_shapes == nullptr || level_start_index == nullptr ||
               sampling_locations == nullptr || attention_weights == nullptr ||
               grad_output == nullptr || grad_sampling_locations == nullptr ||
               grad_attention_weights == nullptr))
    return MSDA_ERR_NULL_POINTER;
  if (work && (!aligned(value, in_align) || !aligned(grad_output, in_align) ||
               !aligned(sampling_locations, 8) || !aligned(grad_sampling_locations, 8) ||
               !aligned(attention_weights, 4) || !aligned(grad_attention_weights, 4) ||
               !aligned(spatial_shapes, 8) || !aligned(level_start_index, 8)))
    return MSDA_ERR_MISALIGNED;
  if (work && validate_env()) {
    st = check_device_metadata(S, L, spatial_shapes, level_start_index);
    if (st != MSDA_OK) return st;
  }
  msda::BackwardArgs a;
  a.value = value;
  a.bf16 = value_dtype == MSDA_BF16;
  a.spatial_shapes = spatial_shapes;
  a.level_start_index = level_start_index;
  a.sampling_locations = sampling_locations;
  a.attention_weights = attention_weights;
  a.grad_output = grad_output;
  a.grad_value = grad_value;
  a.grad_sampling_locations = grad_sampling_locations;
  a.grad_attention_weights = grad_attention_weights;
  a.B = B;
  a.S = S;
  a.Lq = Lq;
  a.M = static_cast<int>(M);
  a.D = static_cast<int>(D);
  a.L = static_cast<int>(L);
  a.K = static_cast<int>(K);
  a.lanes = pow2_at_least(D / 4);
  a.groups = work ? B * Lq * M : 0;
  a.value_elements = c.value_elems;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long in_bytes = a.bf16 ? 2 : 4;
  if (msda::arm_bounds(value, c.value_elems * in_bytes, grad_output, c.out_elems * in_bytes,
                       grad_value, c.value_elems * 4, workspace,
                       static_cast<long long>(workspace_bytes), s) != cudaSuccess)
    return MSDA_ERR_CUDA;
  return msda::launch_backward_deterministic(a, workspace, s) == cudaSuccess ? MSDA_OK
                                                                             : MSDA_ERR_CUDA;
}

msda_status msda_output_projection(int64_t rows, int64_t c_in, int64_t c_out, const float* x,
                                   const float* weight, const float* bias, float* y,
                                   void* stream) {
  return output_projection(rows, c_in, c_out, x, weight, bias, y, false, stream);
}

msda_status msda_output_projection_f32(int64_t rows, int64_t c_in, int64_t c_out,
                                       const float* x, const float* weight, const float* bias,
                                       float* y, void* stream) {
  return output_projection(rows, c_in, c_out, x, weight, bias, y, true, stream);
}

msda_status msda_output_projection_check(int* failed) {
  if (failed == nullptr) return MSDA_ERR_NULL_POINTER;
  int* flag = nullptr;
  if (msda::projection_failed_flag(&flag) != cudaSuccess) return MSDA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(failed, flag, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(flag, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return MSDA_ERR_CUDA;
  return MSDA_OK;
}

msda_status msda_wait_check(int* failed) {
  if (failed == nullptr) return MSDA_ERR_NULL_POINTER;
  int* flag = nullptr;
  if (msda::tiled_wait_flag(&flag) != cudaSuccess) return MSDA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(failed, flag, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(flag, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return MSDA_ERR_CUDA;
  return MSDA_OK;
}

msda_status msda_fused_forward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                               int64_t L, int64_t K, int64_t R, msda_dtype value_dtype,
                               const void* value, const int64_t* spatial_shapes,
                               const int64_t* level_start_index, const float* reference_points,
                               const float* sampling_offsets, const float* attention_logits,
                               void* output, void* stream) {
  Common c;
  msda_status st = check_common(B, S, M, D, Lq, L, K, &c);
  if (st != MSDA_OK) return st;
  if (R != 2 && R != 4) return MSDA_ERR_BAD_SHAPE;
  if (value_dtype != MSDA_F32 && value_dtype != MSDA_BF16) return MSDA_ERR_UNSUPPORTED;
  const int E = value_dtype == MSDA_F32 ? 4 : 8;
  if (D % E != 0 || M > INT32_MAX || D > INT32_MAX) return MSDA_ERR_UNSUPPORTED;
  if (c.out_elems == 0) return MSDA_OK;
  if ((c.value_elems > 0 && value == nullptr) || spatial_shapes == nullptr ||
      level_start_index == nullptr || reference_points == nullptr ||
      sampling_offsets == nullptr || attention_logits == nullptr || output == nullptr)
    return MSDA_ERR_NULL_POINTER;
  if (!aligned(value, 16) || !aligned(output, 16) || !aligned(sampling_offsets, 8) ||
      !aligned(reference_points, 4) || !aligned(attention_logits, 4) ||
      !aligned(spatial_shapes, 8) || !aligned(level_start_index, 8))
    return MSDA_ERR_MISALIGNED;
  if (validate_env()) {
    st = check_device_metadata(S, L, spatial_shapes, level_start_index);
    if (st != MSDA_OK) return st;
  }
  msda::FusedArgs a{};
  a.value = value;
  a.spatial_shapes = spatial_shapes;
  a.level_start_index = level_start_index;
  a.reference_points = reference_points;
  a.sampling_offsets = sampling_offsets;
  a.attention_logits = attention_logits;
  a.output = output;
  a.S = S;
  a.Lq = Lq;
  a.M = static_cast<int>(M);
  a.D = static_cast<int>(D);
  a.L = static_cast<int>(L);
  a.K = static_cast<int>(K);
  a.R = static_cast<int>(R);
  a.bf16 = value_dtype == MSDA_BF16;
  const int64_t nvec = D / E;
  a.lanes = pow2_at_least(nvec);
  a.chunks = static_cast<int>((nvec + a.lanes - 1) / a.lanes);
  a.groups = B * Lq * M * a.chunks;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (msda::arm_bounds(value, c.value_elems * (a.bf16 ? 2 : 4), nullptr, 0, nullptr, 0, nullptr,
                       0, s) != cudaSuccess)
    return MSDA_ERR_CUDA;
  return msda::launch_fused_forward(a, s) == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

msda_status msda_fused_backward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                                int64_t L, int64_t K, int64_t R, msda_dtype value_dtype,
                                const void* value, const int64_t* spatial_shapes,
                                const int64_t* level_start_index, const float* reference_points,
                                const float* sampling_offsets, const float* attention_logits,
                                const void* grad_output, float* grad_value,
                                float* grad_sampling_offsets, float* grad_attention_logits,
                                float* grad_reference_points, void* stream) {
  Common c;
  msda_status st = check_common(B, S, M, D, Lq, L, K, &c);
  if (st != MSDA_OK) return st;
  if (R != 2 && R != 4) return MSDA_ERR_BAD_SHAPE;
  if (value_dtype != MSDA_F32 && value_dtype != MSDA_BF16) return MSDA_ERR_UNSUPPORTED;
  const uintptr_t in_align = value_dtype == MSDA_F32 ? 16 : 8;
  if (D % 4 != 0 || D > 128 || M > INT32_MAX) return MSDA_ERR_UNSUPPORTED;
  int64_t ref_elems = 0;
  if (!product_ok({B, Lq, L, R}, &ref_elems)) return MSDA_ERR_BAD_SHAPE;
  if (c.value_elems == 0 && c.out_elems == 0) return MSDA_OK;
  if (c.value_elems > 0 && grad_value == nullptr) return MSDA_ERR_NULL_POINTER;
  if (!aligned(grad_value, 16) || !aligned(grad_reference_points, 4)) return MSDA_ERR_MISALIGNED;
  const bool work = c.out_elems > 0;
  if (work && (value == nullptr || spatial_shapes == nullptr || level_start_index == nullptr ||
               reference_points == nullptr || sampling_offsets == nullptr ||
               attention_logits == nullptr || grad_output == nullptr ||
               grad_sampling_offsets == nullptr || grad_attention_logits == nullptr))
    return MSDA_ERR_NULL_POINTER;
  if (work && (!aligned(value, in_align) || !aligned(grad_output, in_align) ||
               !aligned(sampling_offsets, 8) || !aligned(grad_sampling_offsets, 8) ||
               !aligned(reference_points, 4) || !aligned(attention_logits, 4) ||
               !aligned(grad_attention_logits, 4) || !aligned(spatial_shapes, 8) ||
               !aligned(level_start_index, 8)))
    return MSDA_ERR_MISALIGNED;
  if (work && validate_env()) {
    st = check_device_metadata(S, L, spatial_shapes, level_start_index);
    if (st != MSDA_OK) return st;
  }
  msda::FusedArgs a{};
  a.value = value;
  a.spatial_shapes = spatial_shapes;
  a.level_start_index = level_start_index;
  a.reference_points = reference_points;
  a.sampling_offsets = sampling_offsets;
  a.attention_logits = attention_logits;
  a.grad_output = grad_output;
  a.bf16 = value_dtype == MSDA_BF16;
  a.grad_value = grad_value;
  a.grad_sampling_offsets = grad_sampling_offsets;
  a.grad_attention_logits = grad_attention_logits;
  a.grad_reference_points = work ? grad_reference_points : nullptr;
  a.S = S;
  a.Lq = Lq;
  a.M = static_cast<int>(M);
  a.D = static_cast<int>(D);
  a.L = static_cast<int>(L);
  a.K = static_cast<int>(K);
  a.R = static_cast<int>(R);
  a.lanes = pow2_at_least(D / 4);
  a.chunks = 1;
  a.groups = work ? B * Lq * M : 0;
  a.value_elements = c.value_elems;
  a.reference_elements = ref_elems;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long in_bytes = a.bf16 ? 2 : 4;
  if (msda::arm_bounds(value, c.value_elems * in_bytes, grad_output, c.out_elems * in_bytes,
                       grad_value, c.value_elems * 4, nullptr, 0, s) != cudaSuccess)
    return MSDA_ERR_CUDA;
  return msda::launch_fused_backward(a, s) == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

msda_status msda_backward_workspace_size(int64_t B, int64_t S, int64_t M, int64_t D,
                                         int64_t Lq, int64_t L, int64_t K, size_t* bytes) {
  if (bytes == nullptr) return MSDA_ERR_NULL_POINTER;
  *bytes = 0;
  Common c;
  const msda_status st = check_common(B, S, M, D, Lq, L, K, &c);
  if (st != MSDA_OK) return st;
  // Point ids, record positions and cell keys are 32-bit in the sorted pass.
  int64_t keys = 0;
  if (c.point_elems / 2 >= (int64_t(1) << 31) || !product_ok({B, M, 2 * S + 2 * L}, &keys) ||
      keys >= (int64_t(1) << 31))
    return MSDA_ERR_UNSUPPORTED;
  *bytes = static_cast<size_t>(
      msda::sorted_layout(B, S, M, Lq, static_cast<int>(L), static_cast<int>(K)).bytes);
  return MSDA_OK;
}

msda_status msda_check_metadata(int64_t S, int64_t L, const int64_t* shapes,
                                const int64_t* starts) {
  if (L < 0 || S < 0) return MSDA_ERR_BAD_SHAPE;
  if (L > 0 && (shapes == nullptr || starts == nullptr)) return MSDA_ERR_NULL_POINTER;
  int64_t total = 0;
  for (int64_t l = 0; l < L; ++l) {
    const int64_t h = shapes[2 * l], w = shapes[2 * l + 1];
    if (h < 1 || w < 1 || h >= msda::kMaxLevelExtent || w >= msda::kMaxLevelExtent)
      return MSDA_ERR_BAD_SHAPE;
    if (starts[l] != total) return MSDA_ERR_BAD_SHAPE;
    total += h * w;
    if (total > S) return MSDA_ERR_BAD_SHAPE;
  }
  return total == S ? MSDA_OK : MSDA_ERR_BAD_SHAPE;
}

const char* msda_status_string(int status) {
  switch (status) {
    case MSDA_OK: return "ok";
    case MSDA_ERR_NULL_POINTER: return "a required pointer is NULL";
    case MSDA_ERR_BAD_SHAPE: return "negative size, size overflow or inconsistent level metadata";
    case MSDA_ERR_UNSUPPORTED: return "unsupported dtype, head dim, level count or point count";
    case MSDA_ERR_MISALIGNED: return "a pointer is not aligned as required";
    case MSDA_ERR_CUDA: return "a CUDA launch or runtime call failed";
    case MSDA_ERR_WORKSPACE: return "the workspace is smaller than msda_backward_workspace_size";
    default: return "unknown status";
  }
}

int msda_version(void) { return 100; }

}  // extern "C"
