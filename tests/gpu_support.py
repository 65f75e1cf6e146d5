"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
CUDA path through the binding (and so the C ABI), run the oracle on the same
inputs, and compare with the tolerances the method's arithmetic allows.

Tolerances (per element unless stated):
  * float32 forward:   |gpu - oracle| <= 1e-6 + 1e-5 * |oracle|
  * float32 backward:  |gpu - oracle| <= 1e-4 * |oracle| + 1e-5 * max|oracle|  (per
    tensor; the absolute floor covers sums whose float32 atomic order cancels)
  * bfloat16 forward:  max|gpu - oracle| <= 2e-2 * max|oracle|, and per element
    |gpu - oracle| <= 2^-8 * |oracle| + 1e-5 * max|oracle| (one bfloat16 rounding
    of a float32 sum)
The oracle consumes exactly the values the GPU sees (float32, or the bfloat16
values widened exactly).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from scale_deformable_attention_backward_b200 import binding


def device_inputs(inp, device="cuda"):
    d = {}
    if inp.value_bf16_bits is not None:
        d["value"] = torch.from_numpy(inp.value_bf16_bits.view(np.int16)).view(
            torch.bfloat16).to(device)
    else:
        d["value"] = torch.from_numpy(inp.value).to(device)
    d["spatial_shapes"] = torch.from_numpy(inp.spatial_shapes).to(device)
    d["level_start_index"] = torch.from_numpy(inp.level_start_index).to(device)
    d["sampling_locations"] = torch.from_numpy(inp.sampling_locations).to(device)
    d["attention_weights"] = torch.from_numpy(inp.attention_weights).to(device)
    if inp.grad_output_bf16_bits is not None:
        d["grad_output"] = torch.from_numpy(inp.grad_output_bf16_bits.view(np.int16)).view(
            torch.bfloat16).to(device)
    elif inp.grad_output is not None:
        d["grad_output"] = torch.from_numpy(inp.grad_output).to(device)
    return d


def gpu_forward(d):
    out = binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                          d["sampling_locations"], d["attention_weights"])
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


BACKWARD_PATHS = ("sorted", "direct")


def backward_paths(d):
    """The paths a call supports: the cell-sorted path is float32 only."""
    return BACKWARD_PATHS if d["value"].dtype == torch.float32 else ("direct",)


def gpu_backward(d, path="sorted"):
    """Backward through the C ABI: ``sorted`` passes a workspace (cell-sorted
    kernels), ``direct`` passes none (one atomic per point corner)."""
    gv, gl, ga = binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                                  d["sampling_locations"], d["attention_weights"],
                                  d["grad_output"],
                                  workspace="auto" if path == "sorted" else None)
    torch.cuda.synchronize()
    return tuple(t.cpu().numpy().astype(np.float64) for t in (gv, gl, ga))


def check_backward_paths(d, inp, what=""):
    """Both backward paths against one oracle backward."""
    rv, rl, ra = oracle_backward(inp)
    for path in backward_paths(d):
        gv, gl, ga = gpu_backward(d, path)
        tag = f" {what} ({path})"
        assert_backward_f32(gv, rv, "grad_value" + tag)
        assert_backward_f32(gl, rl, "grad_sampling_locations" + tag)
        assert_backward_f32(ga, ra, "grad_attention_weights" + tag)


def oracle_forward(inp):
    return oracle.forward(inp.value, inp.spatial_shapes, inp.level_start_index,
                          inp.sampling_locations, inp.attention_weights)


def oracle_backward(inp):
    return oracle.backward(inp.value, inp.spatial_shapes, inp.level_start_index,
                           inp.sampling_locations, inp.attention_weights, inp.grad_output)


def _report(err, bound, what):
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of "
                             f"tolerance; worst at {i}: err {err[i]:.3e} > bound {bound[i]:.3e}")


def assert_forward_f32(got, ref, what="forward"):
    assert got.shape == ref.shape
    assert np.array_equal(np.isnan(got), np.isnan(ref)), f"{what}: NaN pattern differs"
    keep = ~np.isnan(ref)
    err = np.abs(got[keep] - ref[keep])
    _report(err, 1e-6 + 1e-5 * np.abs(ref[keep]), what)


def assert_backward_f32(got, ref, what="backward"):
    assert got.shape == ref.shape
    assert np.array_equal(np.isnan(got), np.isnan(ref)), f"{what}: NaN pattern differs"
    keep = ~np.isnan(ref)
    g, r = got[keep], ref[keep]
    scale = np.abs(r).max() if r.size else 0.0
    _report(np.abs(g - r), 1e-4 * np.abs(r) + 1e-5 * scale, what)


def assert_forward_bf16(got, ref, what="bf16 forward"):
    assert got.shape == ref.shape
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    assert err.max() <= 2e-2 * scale, f"{what}: max err {err.max():.3e} > 2e-2 * {scale:.3e}"
    _report(err, 2.0 ** -8 * np.abs(ref) + 1e-5 * scale, what)
