"""The debug build's bounds checks on the GPU, run by test_debug_bounds_gpu.py as
a child process with MSDA_DEBUG_BOUNDS=1, so that the binding loads
libmsda_debug.so.

1. With every buffer registered whole, each entry point (forward, the three
   backward paths, the fused op) matches the oracle and no access is refused.
2. With the value buffer clipped (msda_debug_bounds_clip) at a pixel boundary
   inside the last image, the gathers past the clip are refused and read as
   zeros: the forward, and the backward's location and weight gradients, match
   the oracle run on a value whose pixels past the clip are zero, and the first
   refused address lies past the clip.
3. With grad_value clipped the same way, the reductions past the clip are
   refused: grad_value matches the oracle's with those pixels zeroed.

The clip narrows what the checks accept; every access still falls inside real
buffers, so no case reads or writes outside memory that the test owns."""
import dataclasses
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path[:0] = [HERE, os.path.dirname(HERE)]

import numpy as np  # noqa: E402
import torch  # noqa: E402

import gpu_support as G  # noqa: E402
import oracle  # noqa: E402
from scale_deformable_attention_backward_b200 import binding  # noqa: E402
from scale_deformable_attention_backward_b200 import workloads as W  # noqa: E402

RAGGED_F32 = W.Config("ragged_f32", 2, 3, 12, 3, ((7, 9), (4, 5), (2, 3)), "uniform", "f32",
                      True, 37)
RAGGED_BF16 = W.Config("ragged_bf16", 2, 2, 16, 4, ((6, 5), (3, 3)), "uniform", "bf16", True, 29)
WIDE_F32 = W.Config("wide_f32", 1, 2, 192, 2, ((5, 6), (3, 2)), "uniform", "f32", True, 11)


def refusal():
    torch.cuda.synchronize()
    return binding.debug_bounds_check()


def expect_none(what):
    kind, address = refusal()
    assert kind == 0, f"{what}: access refused (kind {kind}) at {address:#x}"


def backward(d, path):
    if path == "deterministic":
        res = binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                               d["sampling_locations"], d["attention_weights"], d["grad_output"],
                               deterministic=True)
        torch.cuda.synchronize()
        return tuple(t.cpu().numpy().astype(np.float64) for t in res)
    return G.gpu_backward(d, path)


def check_whole_buffers():
    for cfg in (W.CONFIGS["tiny_fp32"], RAGGED_F32, RAGGED_BF16, WIDE_F32):
        inp = W.make_inputs(cfg, seed=3)
        d = G.device_inputs(inp)
        got = G.gpu_forward(d)
        ref = G.oracle_forward(inp)
        if cfg.dtype == "bf16":
            G.assert_forward_bf16(got, ref, f"{cfg.name} forward")
        else:
            G.assert_forward_f32(got, ref, f"{cfg.name} forward")
        expect_none(f"{cfg.name} forward")
        rv, rl, ra = G.oracle_backward(inp)
        paths = ["direct"]
        if cfg.D <= 128:
            paths.append("deterministic")
            if cfg.dtype == "f32":
                paths.append("sorted")
        for path in paths:
            gv, gl, ga = backward(d, path)
            G.assert_backward_f32(gv, rv, f"{cfg.name} grad_value ({path})")
            G.assert_backward_f32(gl, rl, f"{cfg.name} grad_sampling_locations ({path})")
            G.assert_backward_f32(ga, ra, f"{cfg.name} grad_attention_weights ({path})")
            expect_none(f"{cfg.name} backward ({path})")

    fz = W.make_fused_inputs(RAGGED_F32, seed=5)
    fd = {k: torch.from_numpy(getattr(fz, k)).cuda() for k in
          ("value", "spatial_shapes", "level_start_index", "reference_points",
           "sampling_offsets", "attention_logits", "grad_output")}
    args = [fd[k] for k in ("value", "spatial_shapes", "level_start_index", "reference_points",
                            "sampling_offsets", "attention_logits")]
    out = binding.fused_forward(*args)
    ref = oracle.fused_forward(fz.value, fz.spatial_shapes, fz.level_start_index,
                               fz.reference_points, fz.sampling_offsets, fz.attention_logits)
    G.assert_forward_f32(out.double().cpu().numpy(), ref, "fused forward")
    expect_none("fused forward")
    got = binding.fused_backward(*args, fd["grad_output"])
    want = oracle.fused_backward(fz.value, fz.spatial_shapes, fz.level_start_index,
                                 fz.reference_points, fz.sampling_offsets, fz.attention_logits,
                                 fz.grad_output)
    for g, r, name in zip(got, want, ("grad_value", "grad_sampling_offsets",
                                      "grad_attention_logits", "grad_reference_points")):
        G.assert_backward_f32(g.double().cpu().numpy(), r, f"fused {name}")
    expect_none("fused backward")


def check_clipped():
    cfg = RAGGED_F32
    inp = W.make_inputs(cfg, seed=7)
    d = G.device_inputs(inp)
    B, S, M, D = inp.value.shape
    row = M * D * 4                       # bytes of one pixel (all heads)
    keep = (B - 1) * S + S // 2           # pixels accepted: all but the last image's upper half
    clip = keep * row
    total = B * S * row

    zeroed = inp.value.copy()
    zeroed[B - 1, S // 2:] = 0.0
    inp0 = dataclasses.replace(inp, value=zeroed)

    def past_clip(address, base):
        return base + clip <= address < base + total

    # 2. value clipped: gathers past the clip read zeros.
    binding.debug_bounds_clip(clip, 0)
    got = G.gpu_forward(d)
    kind, address = refusal()
    G.assert_forward_f32(got, G.oracle_forward(inp0), "clipped-value forward")
    assert kind == 1 and past_clip(address, d["value"].data_ptr()), (kind, hex(address))
    rv, rl0, ra0 = G.oracle_backward(inp0)
    for path in ("direct", "sorted"):
        gv, gl, ga = G.gpu_backward(d, path)
        kind, address = refusal()
        G.assert_backward_f32(gv, rv, f"clipped-value grad_value ({path})")
        G.assert_backward_f32(gl, rl0, f"clipped-value grad_sampling_locations ({path})")
        G.assert_backward_f32(ga, ra0, f"clipped-value grad_attention_weights ({path})")
        assert kind == 1 and past_clip(address, d["value"].data_ptr()), (path, kind, hex(address))

    # 3. grad_value clipped: reductions past the clip are dropped.
    binding.debug_bounds_clip(0, clip)
    rv, rl, ra = G.oracle_backward(inp)
    rv = rv.copy()
    rv[B - 1, S // 2:] = 0.0
    for path in ("direct", "sorted"):
        gv_t = torch.empty(inp.value.shape, dtype=torch.float32, device="cuda")
        gl_t = torch.empty_like(d["sampling_locations"])
        ga_t = torch.empty_like(d["attention_weights"])
        binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                         d["sampling_locations"], d["attention_weights"], d["grad_output"],
                         workspace="auto" if path == "sorted" else None, grad_value=gv_t,
                         grad_sampling_locations=gl_t, grad_attention_weights=ga_t)
        kind, address = refusal()
        G.assert_backward_f32(gv_t.double().cpu().numpy(), rv, f"clipped grad_value ({path})")
        G.assert_backward_f32(gl_t.double().cpu().numpy(), rl, f"grad_sampling_locations ({path})")
        G.assert_backward_f32(ga_t.double().cpu().numpy(), ra, f"grad_attention_weights ({path})")
        assert kind == 2 and past_clip(address, gv_t.data_ptr()), (path, kind, hex(address))

    binding.debug_bounds_clip(0, 0)
    G.gpu_forward(d)
    expect_none("after the clip is lifted")


def main():
    assert binding.LIBRARY_PATH == binding.DEBUG_LIBRARY_PATH, binding.LIBRARY_PATH
    check_whole_buffers()
    check_clipped()
    print("debug bounds: ok")


if __name__ == "__main__":
    main()
