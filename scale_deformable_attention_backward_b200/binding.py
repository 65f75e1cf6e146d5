"""Thin PyTorch binding of the C ABI in ``include/msda.h`` (``libmsda.so``).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, their device pointers and the current CUDA stream are passed to
``msda_forward`` / ``msda_backward``, and the status code is turned into an
exception.  Every step of the operator runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback, and a missing library is an error.

Interface as in "Deformable DETR模型解读（附源码+论文）",
MultiScaleDeformableAttention.forward: ``MSDeformAttnFunction.apply(value,
spatial_shapes, level_start_index, sampling_locations, attention_weights,
im2col_step)``; ``im2col_step`` is accepted and ignored (it only batches the
work in that implementation and does not change the result).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
RELEASE_LIBRARY_PATH = os.path.join(_HERE, "libmsda.so")
# MSDA_DEBUG_BOUNDS=1 in the environment selects the debug build, whose kernels
# check every gather and scatter address against the call's buffers
# (debug_bounds_check below); it is read once, when the library is loaded.
DEBUG_LIBRARY_PATH = os.path.join(_HERE, "libmsda_debug.so")
LIBRARY_PATH = (DEBUG_LIBRARY_PATH if os.environ.get("MSDA_DEBUG_BOUNDS", "0") not in ("", "0")
                else RELEASE_LIBRARY_PATH)

MSDA_F32, MSDA_BF16 = 0, 1
_STATUS = {0: "MSDA_OK", 1: "MSDA_ERR_NULL_POINTER", 2: "MSDA_ERR_BAD_SHAPE",
           3: "MSDA_ERR_UNSUPPORTED", 4: "MSDA_ERR_MISALIGNED", 5: "MSDA_ERR_CUDA",
           6: "MSDA_ERR_WORKSPACE"}

# Every symbol include/msda.h declares, with its ctypes signature.
_I64, _VP, _I32, _SZ = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "msda_forward": (_I32, [_I64] * 7 + [_I32] + [_VP] * 7),
    "msda_backward": (_I32, [_I64] * 7 + [_I32] + [_VP] * 10 + [_SZ, _VP]),
    "msda_backward_workspace_size": (_I32, [_I64] * 7 + [ctypes.POINTER(_SZ)]),
    "msda_backward_noalloc": (_I32, [_I64] * 7 + [_I32] + [_VP] * 10),
    "msda_backward_deterministic": (_I32, [_I64] * 7 + [_I32] + [_VP] * 10 + [_SZ, _VP]),
    "msda_backward_deterministic_workspace_size": (_I32, [_I64] * 7 + [ctypes.POINTER(_SZ)]),
    "msda_fused_forward": (_I32, [_I64] * 8 + [_I32] + [_VP] * 8),
    "msda_fused_backward": (_I32, [_I64] * 8 + [_I32] + [_VP] * 12),
    "msda_output_projection": (_I32, [_I64] * 3 + [_VP] * 5),
    "msda_output_projection_f32": (_I32, [_I64] * 3 + [_VP] * 5),
    "msda_output_projection_check": (_I32, [ctypes.POINTER(_I32)]),
    "msda_wait_check": (_I32, [ctypes.POINTER(_I32)]),
    "msda_debug_bounds_check": (_I32, [ctypes.POINTER(_I32), ctypes.POINTER(ctypes.c_uint64)]),
    "msda_debug_bounds_clip": (_I32, [ctypes.c_uint64, ctypes.c_uint64]),
    "msda_check_metadata": (_I32, [_I64, _I64, _VP, _VP]),
    "msda_status_string": (ctypes.c_char_p, [_I32]),
    "msda_version": (_I32, []),
}


class MSDAError(RuntimeError):
    """A non-OK status from the C ABI, or a missing library."""

    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = _STATUS.get(status, str(status))
        msg = f"{name}"
        if _LIB is not None:
            msg += f" ({_LIB.msda_status_string(status).decode()})"
        super().__init__(f"{what}: {msg}" if what else msg)


_LIB = None


def library() -> ctypes.CDLL:
    """Load ``libmsda.so`` (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIBRARY_PATH):
            flag = " --debug" if LIBRARY_PATH == DEBUG_LIBRARY_PATH else ""
            raise RuntimeError(
                f"{LIBRARY_PATH} is missing: build it with "
                f"`python scale_deformable_attention_backward_b200/csrc/build.py{flag}` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(LIBRARY_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def _check(status: int, what: str):
    if status != 0:
        raise MSDAError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _metadata(spatial_shapes, level_start_index, S, device):
    """Metadata as contiguous int64 device tensors.  Host tensors are checked on
    the host (sum of H*W == S, exclusive prefix sum) before the copy."""
    ss = torch.as_tensor(spatial_shapes)
    st = torch.as_tensor(level_start_index)
    if ss.dtype != torch.int64 or st.dtype != torch.int64:
        ss, st = ss.to(torch.int64), st.to(torch.int64)
    if ss.device.type == "cpu" and st.device.type == "cpu":
        ss, st = ss.contiguous(), st.contiguous()
        _check(library().msda_check_metadata(S, st.numel(), _ptr(ss), _ptr(st)),
               "spatial_shapes / level_start_index")
    return ss.to(device).contiguous(), st.to(device).contiguous()


def _dims(value, sampling_locations, attention_weights):
    if value.dim() != 4:
        raise ValueError("value must be [B, S, M, D]")
    B, S, M, D = value.shape
    if sampling_locations.dim() != 6 or sampling_locations.shape[-1] != 2:
        raise ValueError("sampling_locations must be [B, Lq, M, L, K, 2]")
    Bq, Lq, Mq, L, K, _ = sampling_locations.shape
    if (Bq, Mq) != (B, M):
        raise ValueError("sampling_locations batch / head dims do not match value")
    if tuple(attention_weights.shape) != (B, Lq, M, L, K):
        raise ValueError("attention_weights must be [B, Lq, M, L, K]")
    return B, S, M, D, Lq, L, K


def _require(t: torch.Tensor, name: str, dtype, device):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, value on {device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _value_code(value: torch.Tensor) -> int:
    if value.dtype == torch.float32:
        return MSDA_F32
    if value.dtype == torch.bfloat16:
        return MSDA_BF16
    raise ValueError(f"value dtype {value.dtype} is not supported (float32 or bfloat16)")


def forward(value: torch.Tensor, spatial_shapes, level_start_index,
            sampling_locations: torch.Tensor, attention_weights: torch.Tensor,
            im2col_step: Optional[int] = None,
            output: Optional[torch.Tensor] = None) -> torch.Tensor:
    """MSDeformAttn forward: returns ``[B, Lq, M*D]`` in value's dtype."""
    del im2col_step
    dev = value.device
    B, S, M, D, Lq, L, K = _dims(value, sampling_locations, attention_weights)
    _require(value, "value", None, dev)
    code = _value_code(value)
    _require(sampling_locations, "sampling_locations", torch.float32, dev)
    _require(attention_weights, "attention_weights", torch.float32, dev)
    ss, st = _metadata(spatial_shapes, level_start_index, S, dev)
    if ss.shape != (L, 2) or st.shape != (L,):
        raise ValueError("spatial_shapes must be [L, 2] and level_start_index [L]")
    if output is None:
        output = torch.empty((B, Lq, M * D), dtype=value.dtype, device=dev)
    else:
        _require(output, "output", value.dtype, dev)
        if tuple(output.shape) != (B, Lq, M * D):
            raise ValueError("output must be [B, Lq, M*D]")
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev).cuda_stream
        _check(library().msda_forward(B, S, M, D, Lq, L, K, code, _ptr(value), _ptr(ss),
                                      _ptr(st), _ptr(sampling_locations),
                                      _ptr(attention_weights), _ptr(output),
                                      ctypes.c_void_p(stream)), "msda_forward")
    return output


def backward(value: torch.Tensor, spatial_shapes, level_start_index,
             sampling_locations: torch.Tensor, attention_weights: torch.Tensor,
             grad_output: torch.Tensor,
             grad_value: Optional[torch.Tensor] = None,
             grad_sampling_locations: Optional[torch.Tensor] = None,
             grad_attention_weights: Optional[torch.Tensor] = None,
             workspace=None, deterministic: bool = False,
             ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """MSDeformAttn backward: (grad_value, grad_sampling_locations,
    grad_attention_weights), all float32.

    ``value`` and ``grad_output`` are float32, or both bfloat16 (scratch-free
    path only; the arithmetic and the gradients stay float32).
    ``workspace``: ``None`` (default) selects the scratch-free path (one vector
    atomic per point corner), the faster one on the encoder workloads;
    ``"auto"`` takes scratch for the cell-sorted path from torch's caching
    allocator, and a uint8 CUDA tensor supplies that scratch.

    ``deterministic=True`` selects ``msda_backward_deterministic`` (bit-identical
    results run to run); its scratch is ``workspace`` if that is a uint8 CUDA
    tensor, else taken from torch's caching allocator."""
    dev = value.device
    B, S, M, D, Lq, L, K = _dims(value, sampling_locations, attention_weights)
    _require(value, "value", None, dev)
    code = _value_code(value)
    _require(sampling_locations, "sampling_locations", torch.float32, dev)
    _require(attention_weights, "attention_weights", torch.float32, dev)
    _require(grad_output, "grad_output", value.dtype, dev)
    if tuple(grad_output.shape) != (B, Lq, M * D):
        raise ValueError("grad_output must be [B, Lq, M*D]")
    ss, st = _metadata(spatial_shapes, level_start_index, S, dev)
    if ss.shape != (L, 2) or st.shape != (L,):
        raise ValueError("spatial_shapes must be [L, 2] and level_start_index [L]")
    out = []
    for t, shape, name in ((grad_value, (B, S, M, D), "grad_value"),
                           (grad_sampling_locations, (B, Lq, M, L, K, 2),
                            "grad_sampling_locations"),
                           (grad_attention_weights, (B, Lq, M, L, K), "grad_attention_weights")):
        if t is None:
            t = torch.empty(shape, dtype=torch.float32, device=dev)
        else:
            _require(t, name, torch.float32, dev)
            if tuple(t.shape) != shape:
                raise ValueError(f"{name} must be {list(shape)}")
        out.append(t)
    gv, gl, ga = out
    ws, ws_bytes = None, 0
    if deterministic:
        if isinstance(workspace, torch.Tensor):
            _require(workspace, "workspace", torch.uint8, dev)
            ws = workspace
        else:
            ws = torch.empty(deterministic_workspace_size(B, S, M, D, Lq, L, K),
                             dtype=torch.uint8, device=dev)
        with torch.cuda.device(dev):
            stream = torch.cuda.current_stream(dev).cuda_stream
            _check(library().msda_backward_deterministic(
                B, S, M, D, Lq, L, K, code, _ptr(value), _ptr(ss), _ptr(st),
                _ptr(sampling_locations), _ptr(attention_weights), _ptr(grad_output), _ptr(gv),
                _ptr(gl), _ptr(ga), _ptr(ws), ws.numel(), ctypes.c_void_p(stream)),
                "msda_backward_deterministic")
        return gv, gl, ga
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a uint8 CUDA tensor")
        need = workspace_size(B, S, M, D, Lq, L, K)
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_bytes = need
    elif workspace is not None:
        _require(workspace, "workspace", torch.uint8, dev)
        ws, ws_bytes = workspace, workspace.numel()
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev).cuda_stream
        _check(library().msda_backward(B, S, M, D, Lq, L, K, code, _ptr(value), _ptr(ss),
                                       _ptr(st), _ptr(sampling_locations),
                                       _ptr(attention_weights), _ptr(grad_output), _ptr(gv),
                                       _ptr(gl), _ptr(ga), _ptr(ws), ws_bytes,
                                       ctypes.c_void_p(stream)),
               "msda_backward")
    return gv, gl, ga


def deterministic_workspace_size(B, S, M, D, Lq, L, K) -> int:
    """Bytes of scratch the deterministic backward needs (host computation)."""
    n = ctypes.c_size_t(0)
    _check(library().msda_backward_deterministic_workspace_size(B, S, M, D, Lq, L, K,
                                                                ctypes.byref(n)),
           "msda_backward_deterministic_workspace_size")
    return int(n.value)


def workspace_size(B, S, M, D, Lq, L, K) -> int:
    """Bytes of scratch the cell-sorted backward needs (host computation)."""
    n = ctypes.c_size_t(0)
    _check(library().msda_backward_workspace_size(B, S, M, D, Lq, L, K, ctypes.byref(n)),
           "msda_backward_workspace_size")
    return int(n.value)


class MSDeformAttnFunction(torch.autograd.Function):
    """Autograd wrapper: forward and backward both run in libmsda.so."""

    @staticmethod
    def forward(ctx, value, spatial_shapes, level_start_index, sampling_locations,
                attention_weights, im2col_step=None):
        out = forward(value, spatial_shapes, level_start_index, sampling_locations,
                      attention_weights)
        ctx.save_for_backward(value, sampling_locations, attention_weights)
        ctx.meta = (spatial_shapes, level_start_index)
        return out

    @staticmethod
    def backward(ctx, grad_output):
        value, loc, attn = ctx.saved_tensors
        ss, st = ctx.meta
        gv, gl, ga = backward(value, ss, st, loc, attn,
                              grad_output.to(value.dtype).contiguous())
        # The op returns float32 gradients; autograd wants value's dtype.
        return gv.to(value.dtype), None, None, gl, ga, None


def ms_deform_attn(value, spatial_shapes, level_start_index, sampling_locations,
                   attention_weights, im2col_step=None):
    """Differentiable MSDeformAttn core (value float32 or bfloat16)."""
    return MSDeformAttnFunction.apply(value, spatial_shapes, level_start_index,
                                      sampling_locations, attention_weights, im2col_step)


def _fused_dims(value, reference_points, sampling_offsets, attention_logits):
    if value.dim() != 4:
        raise ValueError("value must be [B, S, M, D]")
    B, S, M, D = value.shape
    if sampling_offsets.dim() != 6 or sampling_offsets.shape[-1] != 2:
        raise ValueError("sampling_offsets must be [B, Lq, M, L, K, 2]")
    Bq, Lq, Mq, L, K, _ = sampling_offsets.shape
    if (Bq, Mq) != (B, M):
        raise ValueError("sampling_offsets batch / head dims do not match value")
    if reference_points.dim() != 4 or tuple(reference_points.shape[:3]) != (B, Lq, L):
        raise ValueError("reference_points must be [B, Lq, L, R]")
    R = reference_points.shape[3]
    if tuple(attention_logits.shape) != (B, Lq, M, L * K):
        raise ValueError("attention_logits must be [B, Lq, M, L*K]")
    return B, S, M, D, Lq, L, K, R


def fused_forward(value: torch.Tensor, spatial_shapes, level_start_index,
                  reference_points: torch.Tensor, sampling_offsets: torch.Tensor,
                  attention_logits: torch.Tensor,
                  output: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The op fed with raw reference points ([B, Lq, L, 2] or box [B, Lq, L, 4]),
    sampling offsets and attention logits (``msda_fused_forward``): returns
    ``[B, Lq, M*D]`` in value's dtype."""
    dev = value.device
    B, S, M, D, Lq, L, K, R = _fused_dims(value, reference_points, sampling_offsets,
                                          attention_logits)
    _require(value, "value", None, dev)
    code = _value_code(value)
    for t, name in ((reference_points, "reference_points"), (sampling_offsets, "sampling_offsets"),
                    (attention_logits, "attention_logits")):
        _require(t, name, torch.float32, dev)
    ss, st = _metadata(spatial_shapes, level_start_index, S, dev)
    if ss.shape != (L, 2) or st.shape != (L,):
        raise ValueError("spatial_shapes must be [L, 2] and level_start_index [L]")
    if output is None:
        output = torch.empty((B, Lq, M * D), dtype=value.dtype, device=dev)
    else:
        _require(output, "output", value.dtype, dev)
        if tuple(output.shape) != (B, Lq, M * D):
            raise ValueError("output must be [B, Lq, M*D]")
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev).cuda_stream
        _check(library().msda_fused_forward(B, S, M, D, Lq, L, K, R, code, _ptr(value), _ptr(ss),
                                            _ptr(st), _ptr(reference_points),
                                            _ptr(sampling_offsets), _ptr(attention_logits),
                                            _ptr(output), ctypes.c_void_p(stream)),
               "msda_fused_forward")
    return output


def fused_backward(value: torch.Tensor, spatial_shapes, level_start_index,
                   reference_points: torch.Tensor, sampling_offsets: torch.Tensor,
                   attention_logits: torch.Tensor, grad_output: torch.Tensor,
                   reference_grad: bool = True):
    """Backward of :func:`fused_forward` (``msda_fused_backward``): returns
    (grad_value, grad_sampling_offsets, grad_attention_logits,
    grad_reference_points or None), all float32.  value and grad_output are both
    float32 or both bfloat16."""
    dev = value.device
    B, S, M, D, Lq, L, K, R = _fused_dims(value, reference_points, sampling_offsets,
                                          attention_logits)
    _require(value, "value", None, dev)
    code = _value_code(value)
    for t, name in ((reference_points, "reference_points"), (sampling_offsets, "sampling_offsets"),
                    (attention_logits, "attention_logits")):
        _require(t, name, torch.float32, dev)
    _require(grad_output, "grad_output", value.dtype, dev)
    if tuple(grad_output.shape) != (B, Lq, M * D):
        raise ValueError("grad_output must be [B, Lq, M*D]")
    ss, st = _metadata(spatial_shapes, level_start_index, S, dev)
    if ss.shape != (L, 2) or st.shape != (L,):
        raise ValueError("spatial_shapes must be [L, 2] and level_start_index [L]")
    gv = torch.empty((B, S, M, D), dtype=torch.float32, device=dev)
    goff = torch.empty((B, Lq, M, L, K, 2), dtype=torch.float32, device=dev)
    gz = torch.empty((B, Lq, M, L * K), dtype=torch.float32, device=dev)
    gref = torch.empty((B, Lq, L, R), dtype=torch.float32, device=dev) if reference_grad else None
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev).cuda_stream
        _check(library().msda_fused_backward(B, S, M, D, Lq, L, K, R, code, _ptr(value),
                                             _ptr(ss), _ptr(st), _ptr(reference_points),
                                             _ptr(sampling_offsets), _ptr(attention_logits),
                                             _ptr(grad_output), _ptr(gv), _ptr(goff), _ptr(gz),
                                             _ptr(gref), ctypes.c_void_p(stream)),
               "msda_fused_backward")
    return gv, goff, gz, gref


class MSDeformAttnFusedFunction(torch.autograd.Function):
    """Autograd wrapper of the fused op: forward and backward run in libmsda.so."""

    @staticmethod
    def forward(ctx, value, spatial_shapes, level_start_index, reference_points,
                sampling_offsets, attention_logits):
        out = fused_forward(value, spatial_shapes, level_start_index, reference_points,
                            sampling_offsets, attention_logits)
        ctx.save_for_backward(value, reference_points, sampling_offsets, attention_logits)
        ctx.meta = (spatial_shapes, level_start_index)
        return out

    @staticmethod
    def backward(ctx, grad_output):
        value, ref, off, logits = ctx.saved_tensors
        ss, st = ctx.meta
        gv, goff, gz, gref = fused_backward(value, ss, st, ref, off, logits,
                                            grad_output.to(value.dtype).contiguous(),
                                            reference_grad=ctx.needs_input_grad[3])
        # The op returns float32 gradients; autograd wants value's dtype.
        return gv.to(value.dtype), None, None, gref, goff, gz


def ms_deform_attn_fused(value, spatial_shapes, level_start_index, reference_points,
                         sampling_offsets, attention_logits):
    """Differentiable op fed with raw reference points, offsets and logits."""
    return MSDeformAttnFusedFunction.apply(value, spatial_shapes, level_start_index,
                                           reference_points, sampling_offsets,
                                           attention_logits)


def output_projection(x: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None, precise: bool = False) -> torch.Tensor:
    """The Linear layer after the op on the tensor cores (``msda_output_projection``):
    ``x [..., c_in] @ weight[c_out, c_in].T + bias``, float32 in and out (TF32
    products, float32 sums).  ``precise=True`` calls ``msda_output_projection_f32``:
    float32 accuracy from three TF32 products per step."""
    dev = x.device
    if x.dim() < 1 or weight.dim() != 2:
        raise ValueError("x must be [..., c_in] and weight [c_out, c_in]")
    c_in = x.shape[-1]
    c_out = weight.shape[0]
    if tuple(weight.shape) != (c_out, c_in):
        raise ValueError("weight must be [c_out, c_in]")
    _require(x, "x", torch.float32, dev)
    _require(weight, "weight", torch.float32, dev)
    if bias is not None:
        _require(bias, "bias", torch.float32, dev)
        if tuple(bias.shape) != (c_out,):
            raise ValueError("bias must be [c_out]")
    rows = x.numel() // c_in if c_in else 0
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (c_out,), dtype=torch.float32, device=dev)
    else:
        _require(out, "out", torch.float32, dev)
        if tuple(out.shape) != tuple(x.shape[:-1]) + (c_out,):
            raise ValueError("out must be [..., c_out]")
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev).cuda_stream
        fn = library().msda_output_projection_f32 if precise else library().msda_output_projection
        _check(fn(rows, c_in, c_out, _ptr(x), _ptr(weight), _ptr(bias), _ptr(out),
                  ctypes.c_void_p(stream)),
               "msda_output_projection_f32" if precise else "msda_output_projection")
    return out


def output_projection_failed() -> bool:
    """Whether a projection since the last call gave up waiting (for a TMA copy,
    an MMA or its epilogue) and left rows unwritten; clears the flag
    (synchronises with the device)."""
    f = ctypes.c_int(0)
    _check(library().msda_output_projection_check(ctypes.byref(f)), "msda_output_projection_check")
    return bool(f.value)


def wait_failed() -> bool:
    """Whether a kernel with bounded waits between its warps (the encoder
    kernels that stage value windows in shared memory) gave up a wait since the
    last call and left outputs unwritten; clears the flag (synchronises with the
    device)."""
    f = ctypes.c_int(0)
    _check(library().msda_wait_check(ctypes.byref(f)), "msda_wait_check")
    return bool(f.value)


def debug_bounds_check() -> Tuple[int, int]:
    """Debug build: (kind, address) of the first gather (kind 1) or scatter
    (kind 2) whose address fell outside the call's buffers since the last check,
    (0, 0) if none; clears the record (synchronises with the device).  The
    release library raises MSDAError(MSDA_ERR_UNSUPPORTED)."""
    kind, address = ctypes.c_int(0), ctypes.c_uint64(0)
    _check(library().msda_debug_bounds_check(ctypes.byref(kind), ctypes.byref(address)),
           "msda_debug_bounds_check")
    return kind.value, address.value


def debug_bounds_clip(value_bytes: int = 0, grad_value_bytes: int = 0) -> None:
    """Debug build: take the registered value / grad_value buffers of the
    following calls as their first value_bytes / grad_value_bytes bytes (0: the
    whole buffer), so that accesses past the clip are refused and recorded."""
    _check(library().msda_debug_bounds_clip(value_bytes, grad_value_bytes),
           "msda_debug_bounds_clip")
