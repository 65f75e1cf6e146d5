"""Float64 CPU oracle for the MSDeformAttn core, forward and backward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product path (the CUDA library and its binding) never imports or calls it.

The arithmetic lives in ``msda_oracle.c`` (plain nested loops in float64; see
its header for the pages and readings it follows).  This module only
marshals numpy arrays into it.  Inputs of any float dtype are widened to
float64, which is exact for float32 and bfloat16 values.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_I64 = ctypes.c_int64
_PD = ctypes.POINTER(ctypes.c_double)
_PI = ctypes.POINTER(ctypes.c_int64)


class Oracle:
    """Handle on one compiled oracle library (the real one, or a test build)."""

    def __init__(self, library_path: str):
        lib = ctypes.CDLL(library_path)
        lib.msda_oracle_forward.restype = ctypes.c_int
        lib.msda_oracle_forward.argtypes = [_I64] * 7 + [_PD, _PI, _PI, _PD, _PD, _PD]
        lib.msda_oracle_backward.restype = ctypes.c_int
        lib.msda_oracle_backward.argtypes = [_I64] * 7 + [_PD, _PI, _PI, _PD, _PD, _PD,
                                                          _PD, _PD, _PD]
        if hasattr(lib, "msda_oracle_fused_forward"):
            lib.msda_oracle_fused_forward.restype = ctypes.c_int
            lib.msda_oracle_fused_forward.argtypes = ([_I64] * 8 + [ctypes.c_int] +
                                                      [_PD, _PI, _PI, _PD, _PD, _PD, _PD])
            lib.msda_oracle_fused_backward.restype = ctypes.c_int
            lib.msda_oracle_fused_backward.argtypes = ([_I64] * 8 + [ctypes.c_int] +
                                                       [_PD, _PI, _PI, _PD, _PD, _PD, _PD,
                                                        _PD, _PD, _PD, _PD])
        self.lib = lib
        self.path = library_path

    @staticmethod
    def _dims(value, spatial_shapes, level_start_index, sampling_locations,
              attention_weights):
        B, S, M, D = value.shape
        Bq, Lq, Mq, L, K, two = sampling_locations.shape
        if (Bq, Mq, two) != (B, M, 2):
            raise ValueError("sampling_locations must be [B, Lq, M, L, K, 2]")
        if attention_weights.shape != (B, Lq, M, L, K):
            raise ValueError("attention_weights must be [B, Lq, M, L, K]")
        if spatial_shapes.shape != (L, 2) or level_start_index.shape != (L,):
            raise ValueError("spatial_shapes must be [L, 2], level_start_index [L]")
        return B, S, M, D, Lq, L, K

    @staticmethod
    def _f64(a):
        return np.ascontiguousarray(np.asarray(a, dtype=np.float64))

    @staticmethod
    def _i64(a):
        return np.ascontiguousarray(np.asarray(a, dtype=np.int64))

    @staticmethod
    def _p(a, kind):
        return a.ctypes.data_as(kind)

    def forward(self, value, spatial_shapes, level_start_index,
                sampling_locations, attention_weights):
        """Return output [B, Lq, M*D] float64."""
        v, sh, st = self._f64(value), self._i64(spatial_shapes), self._i64(level_start_index)
        loc, att = self._f64(sampling_locations), self._f64(attention_weights)
        B, S, M, D, Lq, L, K = self._dims(v, sh, st, loc, att)
        out = np.empty((B, Lq, M * D), dtype=np.float64)
        rc = self.lib.msda_oracle_forward(B, S, M, D, Lq, L, K, self._p(v, _PD),
                                          self._p(sh, _PI), self._p(st, _PI),
                                          self._p(loc, _PD), self._p(att, _PD),
                                          self._p(out, _PD))
        if rc != 0:
            raise ValueError(f"oracle forward rejected the shapes (rc={rc})")
        return out

    def backward(self, value, spatial_shapes, level_start_index,
                 sampling_locations, attention_weights, grad_output):
        """Return (grad_value [B,S,M,D], grad_sampling_locations [B,Lq,M,L,K,2],
        grad_attention_weights [B,Lq,M,L,K]), all float64."""
        v, sh, st = self._f64(value), self._i64(spatial_shapes), self._i64(level_start_index)
        loc, att = self._f64(sampling_locations), self._f64(attention_weights)
        B, S, M, D, Lq, L, K = self._dims(v, sh, st, loc, att)
        go = self._f64(grad_output).reshape(B, Lq, M * D)
        gv = np.empty((B, S, M, D), dtype=np.float64)
        gl = np.empty((B, Lq, M, L, K, 2), dtype=np.float64)
        ga = np.empty((B, Lq, M, L, K), dtype=np.float64)
        rc = self.lib.msda_oracle_backward(B, S, M, D, Lq, L, K, self._p(v, _PD),
                                           self._p(sh, _PI), self._p(st, _PI),
                                           self._p(loc, _PD), self._p(att, _PD),
                                           self._p(go, _PD), self._p(gv, _PD),
                                           self._p(gl, _PD), self._p(ga, _PD))
        if rc != 0:
            raise ValueError(f"oracle backward rejected the shapes (rc={rc})")
        return gv, gl, ga


    @staticmethod
    def _fused_dims(value, spatial_shapes, reference_points, sampling_offsets,
                    attention_logits):
        B, S, M, D = value.shape
        Bq, Lq, Mq, L, K, two = sampling_offsets.shape
        if (Bq, Mq, two) != (B, M, 2):
            raise ValueError("sampling_offsets must be [B, Lq, M, L, K, 2]")
        if reference_points.ndim != 4 or reference_points.shape[:3] != (B, Lq, L):
            raise ValueError("reference_points must be [B, Lq, L, R]")
        R = reference_points.shape[3]
        if R not in (2, 4):
            raise ValueError("reference_points must have 2 or 4 components")
        if attention_logits.shape != (B, Lq, M, L * K):
            raise ValueError("attention_logits must be [B, Lq, M, L*K]")
        if spatial_shapes.shape != (L, 2):
            raise ValueError("spatial_shapes must be [L, 2]")
        return B, S, M, D, Lq, L, K, R

    def fused_forward(self, value, spatial_shapes, level_start_index, reference_points,
                      sampling_offsets, attention_logits, round_f32=True):
        """Output [B, Lq, M*D] float64 of the op fed with raw reference points,
        offsets and logits (locations in float32 when ``round_f32``)."""
        v, sh, st = self._f64(value), self._i64(spatial_shapes), self._i64(level_start_index)
        ref, off = self._f64(reference_points), self._f64(sampling_offsets)
        z = self._f64(attention_logits)
        B, S, M, D, Lq, L, K, R = self._fused_dims(v, sh, ref, off, z)
        out = np.empty((B, Lq, M * D), dtype=np.float64)
        rc = self.lib.msda_oracle_fused_forward(
            B, S, M, D, Lq, L, K, R, int(bool(round_f32)), self._p(v, _PD), self._p(sh, _PI),
            self._p(st, _PI), self._p(ref, _PD), self._p(off, _PD), self._p(z, _PD),
            self._p(out, _PD))
        if rc != 0:
            raise ValueError(f"oracle fused forward failed (rc={rc})")
        return out

    def fused_backward(self, value, spatial_shapes, level_start_index, reference_points,
                       sampling_offsets, attention_logits, grad_output, round_f32=True):
        """Return (grad_value, grad_sampling_offsets, grad_attention_logits,
        grad_reference_points), all float64."""
        v, sh, st = self._f64(value), self._i64(spatial_shapes), self._i64(level_start_index)
        ref, off = self._f64(reference_points), self._f64(sampling_offsets)
        z = self._f64(attention_logits)
        B, S, M, D, Lq, L, K, R = self._fused_dims(v, sh, ref, off, z)
        go = self._f64(grad_output).reshape(B, Lq, M * D)
        gv = np.empty((B, S, M, D), dtype=np.float64)
        goff = np.empty((B, Lq, M, L, K, 2), dtype=np.float64)
        gz = np.empty((B, Lq, M, L * K), dtype=np.float64)
        gref = np.empty((B, Lq, L, R), dtype=np.float64)
        rc = self.lib.msda_oracle_fused_backward(
            B, S, M, D, Lq, L, K, R, int(bool(round_f32)), self._p(v, _PD), self._p(sh, _PI),
            self._p(st, _PI), self._p(ref, _PD), self._p(off, _PD), self._p(z, _PD),
            self._p(go, _PD), self._p(gv, _PD), self._p(goff, _PD), self._p(gz, _PD),
            self._p(gref, _PD))
        if rc != 0:
            raise ValueError(f"oracle fused backward failed (rc={rc})")
        return gv, goff, gz, gref


def project(x, weight, bias=None):
    """The output projection after the op, a Linear layer ("Deformable DETR模型解读",
    MultiScaleDeformableAttention.forward, output_proj): y = x @ weight.T + bias in
    float64 (numpy's matmul serves as the step).  x [rows, c_in], weight
    [c_out, c_in], bias [c_out] or None."""
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(weight, dtype=np.float64)
    y = x64 @ w64.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


_DEFAULT = None


def default() -> Oracle:
    """The oracle built from ``msda_oracle.c`` (compiled on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle(_build.build())
    return _DEFAULT


def forward(*args, **kwargs):
    return default().forward(*args, **kwargs)


def backward(*args, **kwargs):
    return default().backward(*args, **kwargs)


def fused_forward(*args, **kwargs):
    return default().fused_forward(*args, **kwargs)


def fused_backward(*args, **kwargs):
    return default().fused_backward(*args, **kwargs)


__all__ = ["Oracle", "default", "forward", "backward", "fused_forward", "fused_backward",
           "project"]
