"""The C ABI under CUDA graph capture: a training step (forward, then the backward
with its zeroing of grad_value and its programmatic dependent launch) and the
output projection, captured once and replayed, give the eager results.  The
replays start from garbage in every output, so the graph must rewrite all of
them (grad_value included)."""
import numpy as np
import pytest
import torch

import gpu_support as G
from scale_deformable_attention_backward_b200 import binding
from scale_deformable_attention_backward_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()                                # module loading and host caches, outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    return graph


@pytest.mark.parametrize("name", ["tiny_fp32", "decoder_box_train_fp32", "encoder_train_fp32",
                                  "encoder_train_bf16"])
def test_training_step_in_a_graph(name):
    inp = W.make_inputs(W.CONFIGS[name], seed=0, with_grad=True)
    d = G.device_inputs(inp)
    B, S, M, D = inp.value.shape
    Lq = inp.sampling_locations.shape[1]
    out = torch.empty((B, Lq, M * D), dtype=d["value"].dtype, device="cuda")
    gv = torch.empty((B, S, M, D), dtype=torch.float32, device="cuda")
    gl = torch.empty_like(d["sampling_locations"])
    ga = torch.empty_like(d["attention_weights"])

    def step():
        binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                        d["sampling_locations"], d["attention_weights"], output=out)
        binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                         d["sampling_locations"], d["attention_weights"], d["grad_output"],
                         grad_value=gv, grad_sampling_locations=gl, grad_attention_weights=ga)

    step()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (out, gv, gl, ga)]
    graph = _capture(step)
    for _ in range(2):
        for t in (out, gv, gl, ga):
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        # Forward output, grad_loc and grad_attn do not depend on the order of
        # atomics: bit for bit.  grad_value: the float32 backward tolerance.
        assert torch.equal(out, ref[0])
        assert torch.equal(gl, ref[2])
        assert torch.equal(ga, ref[3])
        G.assert_backward_f32(gv.double().cpu().numpy(), ref[1].double().cpu().numpy(),
                              f"{name} grad_value replayed")


@pytest.mark.parametrize("precise", [False, True])
def test_output_projection_in_a_graph(precise):
    rng = np.random.default_rng(5)
    rows, c = 4099, 256
    x = torch.from_numpy(rng.standard_normal((rows, c)).astype(np.float32)).cuda()
    w = torch.from_numpy((rng.standard_normal((c, c)) / 16).astype(np.float32)).cuda()
    b = torch.from_numpy(rng.standard_normal(c).astype(np.float32)).cuda()
    y = torch.empty((rows, c), dtype=torch.float32, device="cuda")

    def proj():
        binding.output_projection(x, w, b, out=y, precise=precise)

    proj()
    torch.cuda.synchronize()
    ref = y.clone()
    graph = _capture(proj)
    y.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert not binding.output_projection_failed()
    assert torch.equal(y, ref)
