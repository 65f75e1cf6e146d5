/*
 * msda.h -- C ABI of the B200 (sm_100a) multi-scale deformable attention core
 * (MSDeformAttn): forward and training backward.
 *
 * The operator, per batch b, query q, head m and channel d:
 *
 *   out[b, q, m*D + d] = sum_{l < L} sum_{k < K} A[b,q,m,l,k] *
 *                        bilinear_l(value[b, :, m, d]; loc[b,q,m,l,k])
 *
 * "Deformable DETR Deformable Transformers for End-to-End Object Detection"
 * (paper notes), 核心洞察 2, multi-scale deformable attention equation -- the part
 * inside the per-head output projection W_m, with the value projection W'_m
 * already applied to `value`.  The sampling rule is the one of
 * "Deformable DETR模型解读（附源码+论文）", ms_deform_attn_core_pytorch: level l is
 * the row-major H_l x W_l block of `value` starting at token
 * level_start_index[l]; location component 0 is x (scaled by W_l), component 1
 * is y (scaled by H_l); the pixel coordinate is x = loc_x * W_l - 0.5 (grid_sample,
 * align_corners=False, grid = 2*loc - 1); the four corners floor(x) + {0,1} x
 * floor(y) + {0,1} are weighted bilinearly and a corner outside the map reads
 * zero (padding_mode='zeros').  The call interface mirrors
 * MSDeformAttnFunction.apply(value, spatial_shapes, level_start_index,
 * sampling_locations, attention_weights, im2col_step) of
 * "Deformable DETR模型解读", MultiScaleDeformableAttention.forward (im2col_step,
 * a batching knob of that implementation, does not change the result and has
 * no counterpart here).
 *
 * Conventions for every entry point
 *  - All tensor arguments are DEVICE pointers to contiguous row-major arrays
 *    owned by the caller.  The library allocates nothing at call time.  The
 *    state it keeps between calls is small and fixed: the scratch array of
 *    msda_backward_noalloc (reserved on each device with the library's device
 *    code), two device flags that record a bounded wait that ran out
 *    (msda_output_projection_check, msda_wait_check), and per-device caches of
 *    the SM count and of kernel attributes (the debug build adds its
 *    registered buffers and its record of refused accesses).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously on it; results are ready once the stream
 *    has been synchronised.  The compute entry points neither allocate nor
 *    synchronise, so they can be captured into a CUDA graph once a first call on
 *    the device has loaded their code (with the environment variable
 *    MSDA_VALIDATE unset: it reads the metadata back to the host).
 *  - Argument errors are detected on the host, before anything is enqueued, and
 *    returned synchronously; nothing is written in that case.  A failed launch
 *    returns MSDA_ERR_CUDA.  A fault during kernel execution surfaces at the
 *    caller's next synchronisation, as with any CUDA call.
 *  - spatial_shapes / level_start_index are read on the device only (no host
 *    synchronisation).  The kernels check each level (H, W >= 1, start >= 0,
 *    start + H*W <= S) before use and treat a level that fails the check as
 *    empty, so inconsistent metadata gives wrong numbers but never an
 *    out-of-bounds access.  msda_check_metadata() validates host copies.
 *  - Supported: value dtype float32 with D % 4 == 0, or bfloat16 with D % 8 == 0
 *    (each lane moves 16 bytes); 1 <= L <= 16; 1 <= K <= 64; every size >= 0,
 *    B*S*M*D and B*Lq*M*L*K*2 below 2^62, S*M*D below 2^31 (one image's value
 *    block is addressed with 32-bit offsets), H_l and W_l below 2^22.  `value`,
 *    `output`, `grad_output` and `grad_value` must be 16-byte aligned (the
 *    bfloat16 backward's `value` and `grad_output`: 8-byte),
 *    `sampling_locations` 8-byte aligned, the other arrays 4-byte aligned
 *    (8-byte for the int64 metadata).
 *  - B*Lq == 0 (or M == 0, or D == 0) is valid and launches nothing, except that
 *    msda_backward still zeroes grad_value.
 */
#ifndef MSDA_H
#define MSDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MSDA_OK = 0,
    MSDA_ERR_NULL_POINTER = 1,  /* a required pointer is NULL                        */
    MSDA_ERR_BAD_SHAPE = 2,     /* a size is negative or the metadata is inconsistent */
    MSDA_ERR_UNSUPPORTED = 3,   /* dtype, D, L or K outside the supported set         */
    MSDA_ERR_MISALIGNED = 4,    /* a pointer breaks the alignment rule above          */
    MSDA_ERR_CUDA = 5,          /* a CUDA launch or runtime call failed               */
    MSDA_ERR_WORKSPACE = 6      /* workspace smaller than msda_backward_workspace_size */
} msda_status;

typedef enum {
    MSDA_F32 = 0,   /* IEEE float32                                    */
    MSDA_BF16 = 1   /* bfloat16 (raw 16-bit, round-to-nearest-even out) */
} msda_dtype;

/*
 * Forward.  "Deformable DETR Deformable Transformers for End-to-End Object
 * Detection", multi-scale deformable attention equation; sampling as in
 * "Deformable DETR模型解读", ms_deform_attn_core_pytorch.
 *
 *   value               [B, S, M, D]        value_dtype   S = sum_l H_l * W_l
 *   spatial_shapes      [L, 2]  int64       row l = (H_l, W_l)
 *   level_start_index   [L]     int64       exclusive prefix sum of H_l * W_l
 *   sampling_locations  [B, Lq, M, L, K, 2] float32       (x, y) normalised
 *   attention_weights   [B, Lq, M, L, K]    float32       (softmax over L*K is
 *                                                          the caller's business)
 *   output              [B, Lq, M * D]      value_dtype   written; channel m*D + d
 *
 * Accumulation is float32 for both dtypes; a bfloat16 output is rounded to
 * nearest-even from the float32 sum.
 */
msda_status msda_forward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                         int64_t L, int64_t K, msda_dtype value_dtype,
                         const void *value, const int64_t *spatial_shapes,
                         const int64_t *level_start_index,
                         const float *sampling_locations,
                         const float *attention_weights, void *output,
                         void *stream);

/*
 * Training backward: the gradients of <grad_output, forward(...)> with respect
 * to value, sampling_locations and attention_weights.  The pages print no
 * backward; this is the exact derivative of the forward above, taken inside the
 * cell floor(x), floor(y) (one-sided at integer pixel coordinates), as the
 * autograd of the grid_sample formulation in "Deformable DETR模型解读",
 * ms_deform_attn_core_pytorch, gives it.  attention_weights are treated as
 * inputs (the softmax before them is not differentiated).
 *
 *   value, spatial_shapes, level_start_index, sampling_locations,
 *   attention_weights   as for msda_forward; D <= 256.  One sub-warp of at
 *                       most 32 lanes holds up to 128 of a head's channels,
 *                       4 per lane, and reduces each point's corner dot
 *                       products over them; a wider head runs as two channel
 *                       passes in stream order, the second adding its share of
 *                       grad_sampling_locations and grad_attention_weights.
 *                       D > 256, or D > 128 with a workspace (the cell-sorted
 *                       path keeps a head in one sub-warp), returns
 *                       MSDA_ERR_UNSUPPORTED.
 *                       value_dtype MSDA_F32,
 *                       or MSDA_BF16 without a workspace (value and
 *                       grad_output then only need 8-byte alignment; the
 *                       arithmetic and every gradient stay float32)
 *   grad_output              [B, Lq, M * D]        value_dtype
 *   grad_value               [B, S, M, D]          float32  overwritten: zeroed on
 *                                                  `stream`, then accumulated with
 *                                                  atomics (summation order, and so
 *                                                  the last bits, vary run to run)
 *   grad_sampling_locations  [B, Lq, M, L, K, 2]   float32  overwritten
 *   grad_attention_weights   [B, Lq, M, L, K]      float32  overwritten
 *   workspace, workspace_bytes
 *                 device scratch owned by the caller, 256-byte aligned, at least
 *                 msda_backward_workspace_size() bytes; its contents on entry do
 *                 not matter and are garbage on exit.  With a workspace the points
 *                 are grouped by bilinear cell first, so each cell's corners are
 *                 read once and each grad_value row gets one atomic per cell
 *                 instead of one per point.  workspace == NULL selects the
 *                 scratch-free path (one atomic per point corner), which
 *                 measured faster on the encoder training workload.  A
 *                 workspace that is too small returns MSDA_ERR_WORKSPACE.  Two
 *                 calls that overlap on the GPU must not share a workspace.
 */
msda_status msda_backward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                          int64_t L, int64_t K, msda_dtype value_dtype,
                          const void *value, const int64_t *spatial_shapes,
                          const int64_t *level_start_index,
                          const float *sampling_locations,
                          const float *attention_weights,
                          const void *grad_output, float *grad_value,
                          float *grad_sampling_locations,
                          float *grad_attention_weights, void *workspace,
                          size_t workspace_bytes, void *stream);

/*
 * Deterministic training backward: the same gradients as msda_backward, and
 * bit-identical from run to run, whatever the order in which the GPU
 * schedules the points (the float atomics of msda_backward land in an order
 * that varies, and so do the last bits of grad_value).  The pages have no
 * counterpart; it is the scratch-free path with every
 * grad_value contribution A w_ij gO[d] (the same float32 product) scaled by
 * 2^e, rounded to an integer and summed exactly with 64-bit integer atomics,
 * then converted to float32 once.  e comes from a deterministic pass over
 * the inputs (sum |A| times max |grad_output| bounds every element), so no sum
 * overflows; the result is closer to the exact sum than float atomics give.
 * grad_sampling_locations and grad_attention_weights are deterministic in the
 * scratch-free path already.  If an input (A or grad_output) is not finite,
 * the call falls back to float atomics, so that NaN and Inf propagate as in
 * msda_backward; the finite elements are then no longer guaranteed
 * bit-identical across runs.
 *
 *   arguments as msda_backward (value_dtype MSDA_F32 or MSDA_BF16), but
 *   D <= 128 (one pass: the integer accumulators' channel layout is per pass),
 *   workspace, workspace_bytes
 *       device scratch owned by the caller, 256-byte aligned, at least
 *       msda_backward_deterministic_workspace_size() bytes (8 bytes per
 *       grad_value element plus 8 KB); required (NULL returns
 *       MSDA_ERR_NULL_POINTER, too small MSDA_ERR_WORKSPACE).  Overlapping
 *       calls must not share it.
 */
msda_status msda_backward_deterministic(int64_t B, int64_t S, int64_t M, int64_t D,
                                        int64_t Lq, int64_t L, int64_t K,
                                        msda_dtype value_dtype, const void *value,
                                        const int64_t *spatial_shapes,
                                        const int64_t *level_start_index,
                                        const float *sampling_locations,
                                        const float *attention_weights,
                                        const void *grad_output, float *grad_value,
                                        float *grad_sampling_locations,
                                        float *grad_attention_weights, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* Bytes of workspace msda_backward_deterministic needs (host only). */
msda_status msda_backward_deterministic_workspace_size(int64_t B, int64_t S, int64_t M,
                                                       int64_t D, int64_t Lq, int64_t L,
                                                       int64_t K, size_t *bytes);

/*
 * The output projection after the op, on the tensor cores: a Linear layer,
 *   y[r, n] = sum_k x[r, k] * weight[n, k] + bias[n]
 * ("Deformable DETR模型解读（附源码+论文）", MultiScaleDeformableAttention.forward,
 * output_proj applied to the op's [N, Lq, M*D] output, rows = N * Lq).
 * tcgen05.mma kind::tf32: the operands are read as TF32 (the float32 top 19
 * bits), products are summed in float32, so |error| stays within about
 * 2^-9 * sum_k |x[r,k] * weight[n,k]|; bias is added in float32.
 *
 *   x       [rows, c_in]     float32, 16-byte aligned (c_in % 8 == 0, 8 <= c_in <= 4096)
 *   weight  [c_out, c_in]    float32, 16-byte aligned (nn.Linear's layout;
 *                            c_out % 16 == 0, 16 <= c_out <= 256)
 *   bias    [c_out]          float32, or NULL
 *   y       [rows, c_out]    float32, 16-byte aligned, written
 * rows == 0 launches nothing; rows above 2^31 - 129 give MSDA_ERR_UNSUPPORTED
 * (TMA tile coordinates are 32-bit).  The kernel's waits (for its
 * TMA copies, its MMAs and its epilogue) are bounded; if one ever runs out,
 * some rows are left unwritten and msda_output_projection_check reports it.
 */
msda_status msda_output_projection(int64_t rows, int64_t c_in, int64_t c_out, const float *x,
                                   const float *weight, const float *bias, float *y,
                                   void *stream);

/*
 * The same Linear layer at float32 accuracy (the pages' output_proj is a
 * float32 nn.Linear), still on the tensor cores: every operand element is split
 * into its TF32 head (its 13 low mantissa bits cleared) and the float32
 * remainder, and each K step takes three kind::tf32 MMAs, hi_x hi_w + hi_x lo_w +
 * lo_x hi_w, accumulated in float32.  The dropped lo_x lo_w term and the TF32
 * reading of the remainders leave each product within about 3 * 2^-20 of
 * |x w|; the float32 accumulation adds its own rounding, so
 * |error| <= 1e-5 * sum_k |x[r,k] * weight[n,k]| holds with margin for
 * c_in <= 4096.  Arguments, limits, status codes and the bounded waits
 * (msda_output_projection_check) as for msda_output_projection.
 */
msda_status msda_output_projection_f32(int64_t rows, int64_t c_in, int64_t c_out,
                                       const float *x, const float *weight, const float *bias,
                                       float *y, void *stream);

/*
 * *failed = 1 if a projection since the last check gave up waiting (for a
 * copy, an MMA or its epilogue), else 0; clears the flag.  Synchronises with the device (it copies the
 * flag to the host).
 */
msda_status msda_output_projection_check(int *failed);

/*
 * The op fused with the step before it: the sampling locations and attention
 * weights are formed inside the kernels from the raw reference points,
 * sampling offsets and attention logits, so neither is written to or read
 * from memory.  "Deformable DETR模型解读（附源码+论文）",
 * MultiScaleDeformableAttention.forward, and MSDeformAttn.forward on the
 * phdsky.com notes of "Deformable DETR Deformable Transformers for End-to-End
 * Object Detection":
 *
 *   A[b,q,m,:]  = softmax over the L*K logits attention_logits[b,q,m,:]
 *   R == 2:  loc[b,q,m,l,k] = ref[b,q,l] + off[b,q,m,l,k] / (W_l, H_l)
 *   R == 4:  loc[b,q,m,l,k] = ref[b,q,l,0:2] + off[b,q,m,l,k] / K * ref[b,q,l,2:4] * 0.5
 *            (a box reference: centre x, y and size w, h, all normalised)
 *
 * then out = msda_forward(value, ..., loc, A).  loc is formed in float32 with
 * each operation rounded once in the order written (the pages' float32
 * tensors compute it so), so its pixel cell is the one they get.
 *
 *   reference_points    [B, Lq, L, R]        float32, R = 2 or 4 (else
 *                                             MSDA_ERR_BAD_SHAPE)
 *   sampling_offsets    [B, Lq, M, L, K, 2]  float32, 8-byte aligned; pixels of
 *                                             level l for R == 2
 *   attention_logits    [B, Lq, M, L * K]    float32
 *   value, spatial_shapes, level_start_index, output, stream: as msda_forward.
 */
msda_status msda_fused_forward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                               int64_t L, int64_t K, int64_t R, msda_dtype value_dtype,
                               const void *value, const int64_t *spatial_shapes,
                               const int64_t *level_start_index,
                               const float *reference_points,
                               const float *sampling_offsets,
                               const float *attention_logits, void *output, void *stream);

/*
 * Backward of msda_fused_forward: the gradients of <grad_output, output> with
 * respect to value, sampling_offsets, attention_logits and (optionally)
 * reference_points.  With dloc, dA the core's gradients (msda_backward):
 *   d off          = dloc / (W_l, H_l)                (R == 2)
 *                  = dloc * ref[2:4] * 0.5 / K        (R == 4)
 *   d logits_i     = A_i * (dA_i - sum_j A_j dA_j)    over each (b, q, m)
 *   d ref[0:2]     = sum over (m, k) of dloc
 *   d ref[2:4]     = sum over (m, k) of dloc * off * 0.5 / K   (R == 4)
 * The derivative is that of the real-number formula (the float32 rounding of
 * loc is not differentiated); the pages print no backward.
 *
 *   value_dtype MSDA_F32, or MSDA_BF16 (value and grad_output bfloat16, 8-byte
 *       aligned; the arithmetic and every gradient stay float32, as in
 *       msda_backward); D <= 128 (one sub-warp per head: the softmax Jacobian
 *       revisits each point's dA, which a channel pass would not have complete)
 *   grad_output              [B, Lq, M * D]        value_dtype
 *   grad_value               [B, S, M, D]          overwritten (zeroed, then
 *                                                  atomics; 16-byte aligned)
 *   grad_sampling_offsets    [B, Lq, M, L, K, 2]   overwritten (8-byte aligned)
 *   grad_attention_logits    [B, Lq, M, L * K]     overwritten
 *   grad_reference_points    [B, Lq, L, R]         overwritten (zeroed, then
 *                                                  atomics), or NULL to skip it
 *                                                  (reference points are often
 *                                                  detached)
 * The scratch-free path of msda_backward is used; there is no workspace.
 */
msda_status msda_fused_backward(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                                int64_t L, int64_t K, int64_t R, msda_dtype value_dtype,
                                const void *value, const int64_t *spatial_shapes,
                                const int64_t *level_start_index,
                                const float *reference_points,
                                const float *sampling_offsets,
                                const float *attention_logits, const void *grad_output,
                                float *grad_value, float *grad_sampling_offsets,
                                float *grad_attention_logits,
                                float *grad_reference_points, void *stream);

/*
 * Bytes of workspace msda_backward needs for these sizes (host only; no device
 * access).  The bound depends on the sizes alone: a level of H x W pixels has
 * (H + 1)(W + 1) bilinear cells, and sum_l (H_l + 1)(W_l + 1) <= 2 S + 2 L.
 * For B=4, S=Lq=19947, M=8, L=K=4 it is about 276 MB.  Returns
 * MSDA_ERR_UNSUPPORTED when the sorted path's 32-bit cell and point ids would
 * overflow (B*M*(2S+2L) or B*Lq*M*L*K at 2^31 or more); the scratch-free path
 * still accepts those sizes.
 */
msda_status msda_backward_workspace_size(int64_t B, int64_t S, int64_t M, int64_t D,
                                         int64_t Lq, int64_t L, int64_t K,
                                         size_t *bytes);

/*
 * Size of the fixed device scratch of msda_backward_noalloc: 32 MiB, held by
 * every GPU that loads this library until the process exits.
 */
#define MSDA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * msda_backward without a workspace argument and without any allocation.  The
 * pages have no counterpart: this entry point exists for callers that cannot
 * allocate device memory at the time they call the op -- for instance a host
 * framework that owns the whole device memory pool and admits no other
 * allocator, or code on a latency-critical path where cudaMalloc / cudaFree
 * would block or synchronize the device.
 *
 * It computes what msda_backward computes with a workspace (the cell-sorted
 * path; arguments, layouts, ownership of the tensors and status codes as for
 * msda_backward), taking the scratch from one array of
 * MSDA_NOALLOC_SCRATCH_BYTES that the library holds on each device.  It calls
 * no cudaMalloc, cudaFree or other allocating routine.
 *   - value_dtype must be MSDA_F32 (grad_output is float32); MSDA_BF16 returns
 *     MSDA_ERR_UNSUPPORTED.
 *   - Sizes whose msda_backward_workspace_size exceeds MSDA_NOALLOC_SCRATCH_BYTES
 *     are rejected with MSDA_ERR_WORKSPACE before anything is enqueued (for
 *     example B=1, S=19947, M=8, D=32, L=K=4 fits up to Lq = 9259 queries).
 *   - First call on a device: CUDA loads device code lazily by default, so the
 *     first call there loads this path's kernels and reserves the 32 MiB array
 *     on that device -- device memory the CUDA driver takes at that moment, not
 *     through any allocator of the caller's.  A caller whose framework is about
 *     to take the whole memory pool should therefore make one warm-up call with
 *     a small real problem on each device before the pool is taken (or set
 *     CUDA_MODULE_LOADING=EAGER, which reserves everything when the library is
 *     loaded).  That first call should also come before any stream capture.
 *     Later calls reserve nothing.
 *   - The array's device address is looked up on every call, with the calling
 *     thread's current device and context.
 *   - Every call on a device uses the same array, and the array keeps the last
 *     call's contents; each call clears what it needs at zero.  Calls that
 *     overlap on the GPU (other streams, other host threads) race on it and must
 *     be serialized by the caller.
 */
msda_status msda_backward_noalloc(int64_t B, int64_t S, int64_t M, int64_t D, int64_t Lq,
                                  int64_t L, int64_t K, msda_dtype value_dtype,
                                  const void *value, const int64_t *spatial_shapes,
                                  const int64_t *level_start_index,
                                  const float *sampling_locations,
                                  const float *attention_weights,
                                  const float *grad_output, float *grad_value,
                                  float *grad_sampling_locations,
                                  float *grad_attention_weights, void *stream);

/*
 * *failed = 1 if a kernel with bounded waits between its warps (the encoder
 * kernels that stage value windows in shared memory) gave up a wait since the
 * last check, else 0; clears the flag.  Such a kernel leaves some outputs
 * unwritten.  The waits cannot run out unless the library has a bug; the bound
 * exists so that a bug cannot hang the GPU.  Synchronises with the device (it
 * copies the flag to the host).
 */
msda_status msda_wait_check(int *failed);

/*
 * Debug build.  libmsda_debug.so is this library compiled with
 * MSDA_DEBUG_BOUNDS (build.py --debug): the same entry points, in which every
 * gather of a value or grad_output row and every reduction into grad_value
 * (or into the deterministic backward's integer accumulators) first checks
 * that its bytes lie inside a buffer of the current call.  Before it launches,
 * each compute entry point registers its buffers on its stream: readable
 * value and grad_output, writable grad_value and the workspace.  An access
 * outside them is skipped (a read gives zeros) and the first one is recorded.
 * The checks stand in for a memory checker; they make the kernels several
 * times slower.  The registered buffers are process-wide, so the debug build
 * expects one call in flight at a time and is not for CUDA graph capture.
 *
 * msda_debug_bounds_check: *kind = 0 if no access has been refused since the
 * last check, 1 for a read, 2 for a write, and *address = the first refused
 * access's device address (0 when *kind is 0); clears the record.
 * Synchronises with the device.  The release library returns
 * MSDA_ERR_UNSUPPORTED (with *kind = 0, *address = 0).
 *
 * msda_debug_bounds_clip: from the next call on, the registered `value`
 * buffer is taken as its first value_bytes bytes and `grad_value` as its first
 * grad_value_bytes bytes (0: the whole buffer).  Memory past the clip stays
 * valid; accesses there are refused as if it were not.  This lets a caller
 * check that the checks fire, without any access outside real buffers.
 * Release library: MSDA_ERR_UNSUPPORTED.
 */
msda_status msda_debug_bounds_check(int *kind, uint64_t *address);
msda_status msda_debug_bounds_clip(uint64_t value_bytes, uint64_t grad_value_bytes);

/*
 * Host-side metadata check, for callers that hold host copies of the metadata
 * (the pages' layer asserts sum_l H_l * W_l == S before calling the op;
 * "Deformable DETR模型解读", MultiScaleDeformableAttention.forward).
 * Returns MSDA_OK if every H_l, W_l >= 1, level_start_index is the exclusive
 * prefix sum of H_l * W_l and the total is S; MSDA_ERR_BAD_SHAPE otherwise;
 * MSDA_ERR_NULL_POINTER for NULL arrays with L > 0.  Reads host memory only.
 */
msda_status msda_check_metadata(int64_t S, int64_t L,
                                const int64_t *spatial_shapes_host,
                                const int64_t *level_start_index_host);

/* Static, NUL-terminated description of a status code. */
const char *msda_status_string(int status);

/* ABI version: major * 10000 + minor * 100 + patch. */
int msda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MSDA_H */
