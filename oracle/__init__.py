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


__all__ = ["Oracle", "default", "forward", "backward"]
