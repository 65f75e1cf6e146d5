"""The output projection on the tensor cores against the oracle's float64
x W^T + b.

msda_output_projection (TF32): TF32 operands (10 explicit mantissa bits each)
and float32 sums give |y - exact| <= 2^-9 sum_k |x w| (products) + float32
summation, so the test allows 2^-8 sum_k |x w| + 1e-6 |b| per element.

msda_output_projection_f32 (3 x TF32, float32 accuracy): each product is within
about 3 * 2^-20 |x w| and the float32 accumulation of 3 c_in terms adds its
rounding; the test allows 1e-5 sum_k |x w| + 1e-6 |b| per element, the float32
backward's relative bound."""
import numpy as np
import pytest
import torch

import gpu_support as G
import oracle
from scale_deformable_attention_backward_b200 import binding, workloads as W

pytestmark = pytest.mark.gpu


def check(x, w, b, what, precise=False):
    dev = torch.device("cuda")
    xt = torch.from_numpy(x).to(dev)
    wt = torch.from_numpy(w).to(dev)
    bt = None if b is None else torch.from_numpy(b).to(dev)
    y = binding.output_projection(xt, wt, bt, precise=precise)
    torch.cuda.synchronize()
    assert not binding.output_projection_failed(), f"{what}: an MMA wait ran out"
    got = y.cpu().numpy().astype(np.float64)
    ref = oracle.project(x, w, b)
    rel = 1e-5 if precise else 2.0 ** -8
    bound = rel * (np.abs(x.astype(np.float64)) @ np.abs(w.astype(np.float64)).T)
    if b is not None:
        bound += 1e-6 * np.abs(b.astype(np.float64))[None, :]
    bound += 1e-30
    err = np.abs(got - ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} out of tolerance, "
                           f"worst {float((err - bound).max()):.3e}")


@pytest.mark.parametrize("rows,c_in,c_out", [
    (1, 8, 16), (127, 32, 16), (128, 256, 256), (129, 256, 256), (300, 40, 48),
    (1000, 256, 128), (4096, 264, 256), (333, 4096, 32),
    # several row tiles per CTA (both accumulators reused), ragged last tile
    (40000, 96, 80), (80000, 256, 256)])
def test_projection_random(rows, c_in, c_out):
    rng = np.random.default_rng(rows + c_in + c_out)
    x = rng.standard_normal((rows, c_in)).astype(np.float32)
    w = (rng.standard_normal((c_out, c_in)) / np.sqrt(c_in)).astype(np.float32)
    b = rng.standard_normal(c_out).astype(np.float32)
    check(x, w, b, f"rows={rows} c_in={c_in} c_out={c_out}")
    check(x, w, None, f"rows={rows} c_in={c_in} c_out={c_out} no bias")
    check(x, w, b, f"rows={rows} c_in={c_in} c_out={c_out} precise", precise=True)
    check(x, w, None, f"rows={rows} c_in={c_in} c_out={c_out} no bias, precise", precise=True)


def test_precise_projection_beats_tf32():
    """The 3 x TF32 mode is not the TF32 mode in disguise: on data whose
    low mantissa bits matter, its worst error relative to sum_k |x w| is far
    below the TF32 mode's (about 2^-11 there), and below 2^-17."""
    rng = np.random.default_rng(17)
    x = (1.0 + rng.uniform(0, 1, size=(512, 256))).astype(np.float32)  # all bits used
    w = (rng.standard_normal((256, 256)) / 16.0).astype(np.float32)
    dev = torch.device("cuda")
    xt, wt = torch.from_numpy(x).to(dev), torch.from_numpy(w).to(dev)
    scale = np.abs(x.astype(np.float64)) @ np.abs(w.astype(np.float64)).T
    ref = oracle.project(x, w)
    errs = {}
    for precise in (False, True):
        y = binding.output_projection(xt, wt, None, precise=precise)
        torch.cuda.synchronize()
        errs[precise] = float((np.abs(y.cpu().numpy().astype(np.float64) - ref) / scale).max())
    assert not binding.output_projection_failed()
    assert errs[True] < 2.0 ** -17, errs
    assert errs[True] * 64 < errs[False], errs


def test_projection_of_the_encoder_forward():
    """The Linear layer after the op on the encoder workload (B=2, 39,894 rows of
    256 channels): GPU forward then GPU projection, against the oracle's forward
    and projection in float64 (the forward's own float32 error is far below the
    projection's tolerance)."""
    inp = W.make_inputs(W.CONFIGS["encoder_fp32"], seed=0)
    d = G.device_inputs(inp)
    out = binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                          d["sampling_locations"], d["attention_weights"])
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((256, 256)) / 16.0).astype(np.float32)
    b = rng.standard_normal(256).astype(np.float32)
    y = binding.output_projection(out.reshape(-1, 256), torch.from_numpy(w).cuda(),
                                  torch.from_numpy(b).cuda())
    torch.cuda.synchronize()
    assert not binding.output_projection_failed()
    ref_out = G.oracle_forward(inp).reshape(-1, 256)
    ref = oracle.project(ref_out, w, b)
    bound = 2.0 ** -8 * (np.abs(ref_out) @ np.abs(w.astype(np.float64)).T) + 1e-5
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    assert (err <= bound).all(), f"max excess {float((err - bound).max()):.3e}"
    # Precise mode on the same rows: the forward's own float32 error (rel 1e-5 of
    # |out| per element, abs 1e-6) passes through the Linear layer as well.
    yp = binding.output_projection(out.reshape(-1, 256), torch.from_numpy(w).cuda(),
                                   torch.from_numpy(b).cuda(), precise=True)
    torch.cuda.synchronize()
    assert not binding.output_projection_failed()
    absw = np.abs(w.astype(np.float64))
    bound = (1e-5 * (np.abs(ref_out) @ absw.T) + (1e-5 * np.abs(ref_out) + 1e-6) @ absw.T
             + 1e-6 * np.abs(b.astype(np.float64))[None, :])
    err = np.abs(yp.cpu().numpy().astype(np.float64) - ref)
    assert (err <= bound).all(), f"precise: max excess {float((err - bound).max()):.3e}"
