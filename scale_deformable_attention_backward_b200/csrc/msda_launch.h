// msda_launch.h -- internal launch interface between the C ABI (msda_api.cu)
// and the kernels.  Arguments arrive here already validated.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace msda {

constexpr int kMaxLevels = 16;
constexpr int kMaxPoints = 64;
constexpr int kMaxLevelExtent = 1 << 22;  // H_l, W_l below 2^22: float coordinates stay exact

struct ForwardArgs {
  const void* value;
  const int64_t* spatial_shapes;
  const int64_t* level_start_index;
  const float* sampling_locations;
  const float* attention_weights;
  void* output;
  long long B, S, Lq;
  int M, D, L, K;
  bool bf16;
  int lanes;         // lanes per work group: a power of two <= 32
  int chunks;        // channel chunks per (b, q, m): ceil(D / (lanes * elements per lane))
  long long groups;  // B * Lq * M * chunks
};

struct BackwardArgs {
  const void* value;               // float32, or bfloat16 (scratch-free path only)
  const int64_t* spatial_shapes;
  const int64_t* level_start_index;
  const float* sampling_locations;
  const float* attention_weights;
  const void* grad_output;         // value's dtype
  float* grad_value;
  float* grad_sampling_locations;
  float* grad_attention_weights;
  long long B, S, Lq;
  int M, D, L, K;
  bool bf16;         // value / grad_output dtype
  int lanes;         // lanes per (b, q, m) group; D <= 4 * lanes
  long long groups;  // B * Lq * M
  long long value_elements;  // B * S * M * D (grad_value is zeroed first)
};

// The core fed with raw reference points, offsets and logits (msda_fused.cu).
struct FusedArgs {
  const void* value;
  const int64_t* spatial_shapes;
  const int64_t* level_start_index;
  const float* reference_points;   // [B, Lq, L, R]
  const float* sampling_offsets;   // [B, Lq, M, L, K, 2]
  const float* attention_logits;   // [B, Lq, M, L * K]
  long long S, Lq;
  int M, D, L, K, R;
  bool bf16;
  int lanes;                       // forward: as ForwardArgs; backward: D <= 4 * lanes
  int chunks;                      // forward channel chunks per (b, q, m); 1 for the backward
  long long groups;                // B * Lq * M * chunks
  void* output;                    // forward
  const void* grad_output;         // backward: value's dtype
  float* grad_value;
  float* grad_sampling_offsets;
  float* grad_attention_logits;
  float* grad_reference_points;    // may be null: not computed
  long long value_elements;        // B * S * M * D
  long long reference_elements;    // B * Lq * L * R
};

cudaError_t launch_fused_forward(const FusedArgs& a, cudaStream_t stream);
// The pipelined forward kernel forming the inputs in registers; returns
// cudaErrorNotSupported (having launched nothing) unless L*K <= 2 * lanes <= 32.
cudaError_t launch_fused_forward_pipelined(const FusedArgs& a, cudaStream_t stream);
cudaError_t launch_fused_backward(const FusedArgs& a, cudaStream_t stream);

// Scratch layout of the cell-sorted backward (msda_backward_sorted.cu).
struct SortedLayout {
  long long cells_per_bm;  // keys per (b, m): bound on sum_l (H_l + 1)(W_l + 1) from S, L
  long long keys;          // B * M * cells_per_bm cell keys
  long long segments;      // B * M * L: one (b, m, level) each
  long long segment_len;   // Lq * K points per segment
  long long chunks;        // hist / place blocks per segment
  long long points;        // B * Lq * M * L * K
  long long counts;        // keys * chunks (chunk, cell) counters
  long long scan_tiles;
  long long bytes;         // workspace bytes
};

SortedLayout sorted_layout(long long B, long long S, long long M, long long Lq, int L, int K);

cudaError_t launch_forward(const ForwardArgs& a, cudaStream_t stream);
// Whether the encoder-form forward kernels apply: the queries are the value's
// pixels (Lq == S), D * sizeof(T) is 64, 128 or 256 bytes, K <= 8,
// B * Lq * M < 2^31 and S < 2^26.
bool forward_tiles_apply(const ForwardArgs& a);
// The encoder-form forward with shared-memory value windows (msda_forward_tiled.cu).
cudaError_t launch_forward_tiled(const ForwardArgs& a, cudaStream_t stream);
// The same tiles gathered through L1 (msda_forward_l1.cu).
cudaError_t launch_forward_l1(const ForwardArgs& a, cudaStream_t stream);
// Device address of the flag a tiled kernel sets when one of its bounded waits
// runs out (msda_forward_tiled.cu).
cudaError_t tiled_wait_flag(int** flag);
// Backward with one vector atomic per point corner (no scratch).
cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t stream);
// Backward with the points grouped by cell; `workspace` holds sorted_layout().bytes.
cudaError_t launch_backward_sorted(const BackwardArgs& a, void* workspace, cudaStream_t stream);
cudaError_t launch_zero(float* p, long long n, cudaStream_t stream);

// Debug build (MSDA_DEBUG_BOUNDS): registers the call's buffers, in bytes, for
// the kernels' bounds checks, stream-ordered (msda_bounds.cu).  A null pointer
// or a size of 0 registers nothing in that slot.  The release build does
// nothing and returns cudaSuccess.
cudaError_t arm_bounds(const void* value, long long value_bytes, const void* grad_output,
                       long long grad_output_bytes, const void* grad_value,
                       long long grad_value_bytes, const void* workspace,
                       long long workspace_bytes, cudaStream_t stream);

// Output projection Y = X Wt^T + bias on the tensor cores (msda_proj.cu):
// rows x c_in float32 X, c_out x c_in Wt; c_in % 8 == 0, c_out % 16 == 0,
// 16 <= c_out <= 256, all pointers 16-byte aligned (bias 4-byte, may be null).
// precise: float32 accuracy from three TF32 products per step (3 x TF32).
cudaError_t launch_projection(const float* x, const float* weight, const float* bias, float* y,
                              long long rows, int c_in, int c_out, bool precise,
                              cudaStream_t stream);
// Device address of the flag a projection CTA sets when its MMA wait times out.
cudaError_t projection_failed_flag(int** flag);

// Deterministic backward (msda_backward.cu): the scratch-free kernel with the
// grad_value contributions accumulated exactly as scaled 64-bit integers.  The
// workspace holds a kFixedHeaderBytes header, then 8 bytes per grad_value element.
constexpr int kScaleBlocks = 512;
constexpr long long kFixedHeaderBytes = 8192;
cudaError_t launch_backward_deterministic(const BackwardArgs& a, void* workspace,
                                          cudaStream_t stream);

}  // namespace msda
