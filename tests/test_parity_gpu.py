"""GPU parity with the float64 oracle on the five named workloads, at their full
sizes, element by element (forward output; backward grad_value,
grad_sampling_locations and grad_attention_weights).  The CUDA path runs
through the binding and the C ABI, in the same launch configuration the
benchmark times."""
import numpy as np
import pytest

import gpu_support as G
from scale_deformable_attention_backward_b200 import binding, workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", list(W.CONFIGS))
def test_forward_matches_oracle_full_size(name):
    cfg = W.CONFIGS[name]
    inp = W.make_inputs(cfg, seed=0)
    got = G.gpu_forward(G.device_inputs(inp))
    ref = G.oracle_forward(inp)
    if cfg.dtype == "bf16":
        G.assert_forward_bf16(got, ref, f"{name} forward")
    else:
        G.assert_forward_f32(got, ref, f"{name} forward")


@pytest.mark.parametrize("name", [n for n, c in W.CONFIGS.items() if c.backward])
def test_backward_matches_oracle_full_size(name):
    cfg = W.CONFIGS[name]
    inp = W.make_inputs(cfg, seed=0)
    d = G.device_inputs(inp)
    rv, rl, ra = G.oracle_backward(inp)
    for path in G.backward_paths(d):
        gv, gl, ga = G.gpu_backward(d, path)
        G.assert_backward_f32(gv, rv, f"{name} grad_value ({path})")
        G.assert_backward_f32(gl, rl, f"{name} grad_sampling_locations ({path})")
        G.assert_backward_f32(ga, ra, f"{name} grad_attention_weights ({path})")


def test_sorted_backward_location_gradients_are_deterministic():
    """Per-point gradients of the cell-sorted path do not depend on the order
    the atomics give the points inside a cell."""
    inp = W.make_inputs(W.CONFIGS["encoder_train_fp32"].with_batch(1), seed=2)
    d = G.device_inputs(inp)
    first = G.gpu_backward(d, "sorted")
    for _ in range(2):
        again = G.gpu_backward(d, "sorted")
        assert np.array_equal(first[1], again[1]) and np.array_equal(first[2], again[2])


@pytest.mark.parametrize("name", ["encoder_fp32", "decoder_fp32"])
def test_backward_on_forward_workloads(name):
    """The forward-only workloads' geometry through the backward as well (with a
    seeded grad_output), so every geometry is covered by both passes."""
    cfg = W.CONFIGS[name]
    inp = W.make_inputs(cfg, seed=3, with_grad=True)
    gv, gl, ga = G.gpu_backward(G.device_inputs(inp))
    rv, rl, ra = G.oracle_backward(inp)
    G.assert_backward_f32(gv, rv, f"{name} grad_value")
    G.assert_backward_f32(gl, rl, f"{name} grad_sampling_locations")
    G.assert_backward_f32(ga, ra, f"{name} grad_attention_weights")


def test_forward_is_deterministic():
    inp = W.make_inputs(W.CONFIGS["encoder_fp32"].with_batch(1), seed=1)
    d = G.device_inputs(inp)
    a, b = G.gpu_forward(d), G.gpu_forward(d)
    assert np.array_equal(a, b)


def test_bf16_backward_refuses_a_workspace():
    """The cell-sorted path is float32 only: a bfloat16 call with a workspace is
    refused before any launch."""
    inp = W.make_inputs(W.CONFIGS["encoder_train_bf16"].with_batch(1), seed=4)
    d = G.device_inputs(inp)
    with pytest.raises(binding.MSDAError, match="UNSUPPORTED"):
        binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                         d["sampling_locations"], d["attention_weights"], d["grad_output"],
                         workspace="auto")
