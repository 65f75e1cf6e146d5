"""GPU parity of the fused op (locations and weights formed in the kernels from
raw reference points, offsets and logits) with the oracle's fused entry points,
element by element, through the binding and the C ABI.

The oracle forms the locations in float32 exactly as the kernels do (the pages'
order of operations), so both take the same bilinear cell; tolerances are those
of the core (see gpu_support)."""
import numpy as np
import pytest
import torch

import gpu_support as G
import oracle
from scale_deformable_attention_backward_b200 import binding, workloads as W

pytestmark = pytest.mark.gpu


def fused_device(inp, device="cuda"):
    d = {}
    if inp.value_bf16_bits is not None:
        d["value"] = torch.from_numpy(inp.value_bf16_bits.view(np.int16)).view(
            torch.bfloat16).to(device)
    else:
        d["value"] = torch.from_numpy(inp.value).to(device)
    for k in ("spatial_shapes", "level_start_index", "reference_points", "sampling_offsets",
              "attention_logits"):
        d[k] = torch.from_numpy(getattr(inp, k)).to(device)
    if inp.grad_output is not None:
        d["grad_output"] = torch.from_numpy(inp.grad_output).to(device)
    return d


def gpu_fused_forward(d):
    out = binding.fused_forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                                d["reference_points"], d["sampling_offsets"],
                                d["attention_logits"])
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


def gpu_fused_backward(d, reference_grad=True):
    res = binding.fused_backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                                 d["reference_points"], d["sampling_offsets"],
                                 d["attention_logits"], d["grad_output"],
                                 reference_grad=reference_grad)
    torch.cuda.synchronize()
    return tuple(None if t is None else t.cpu().numpy().astype(np.float64) for t in res)


def oracle_fused_forward(inp):
    return oracle.fused_forward(inp.value, inp.spatial_shapes, inp.level_start_index,
                                inp.reference_points, inp.sampling_offsets,
                                inp.attention_logits)


def oracle_fused_backward(inp):
    return oracle.fused_backward(inp.value, inp.spatial_shapes, inp.level_start_index,
                                 inp.reference_points, inp.sampling_offsets,
                                 inp.attention_logits, inp.grad_output)


def check_fused_backward(inp, d, what):
    rv, roff, rz, rref = oracle_fused_backward(inp)
    gv, goff, gz, gref = gpu_fused_backward(d)
    G.assert_backward_f32(gv, rv, f"{what} grad_value")
    G.assert_backward_f32(goff, roff, f"{what} grad_sampling_offsets")
    G.assert_backward_f32(gz, rz, f"{what} grad_attention_logits")
    G.assert_backward_f32(gref, rref, f"{what} grad_reference_points")


@pytest.mark.parametrize("name", list(W.CONFIGS))
def test_fused_forward_matches_oracle_full_size(name):
    cfg = W.CONFIGS[name]
    inp = W.make_fused_inputs(cfg, seed=0)
    got = gpu_fused_forward(fused_device(inp))
    ref = oracle_fused_forward(inp)
    if cfg.dtype == "bf16":
        G.assert_forward_bf16(got, ref, f"{name} fused forward")
    else:
        G.assert_forward_f32(got, ref, f"{name} fused forward")


@pytest.mark.parametrize("name", [n for n, c in W.CONFIGS.items()
                                  if c.backward and c.dtype == "f32"])
def test_fused_backward_matches_oracle_full_size(name):
    inp = W.make_fused_inputs(W.CONFIGS[name], seed=0)
    check_fused_backward(inp, fused_device(inp), f"{name} fused")


def test_fused_backward_bf16_matches_oracle_full_size():
    """The bf16 training workload through the fused backward: bfloat16 value and
    grad_output (the oracle reads the same values widened exactly), float32
    arithmetic and gradients, so the float32 backward tolerances apply."""
    import dataclasses
    inp = W.make_fused_inputs(W.CONFIGS["encoder_train_bf16"], seed=0)
    bits = W.bf16_round_bits(inp.grad_output)
    inp = dataclasses.replace(inp, grad_output=W.bf16_bits_to_f32(bits))
    d = fused_device(inp)
    d["grad_output"] = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    check_fused_backward(inp, d, "encoder_train_bf16 fused")


def _random_fused(rng, B, Lq, M, D, K, shapes, R):
    ss, st = W.level_metadata(shapes)
    S = int((ss[:, 0] * ss[:, 1]).sum())
    L = len(shapes)
    if R == 2:
        ref = rng.uniform(-0.1, 1.1, size=(B, Lq, L, 2))
        off = rng.standard_normal((B, Lq, M, L, K, 2)) * 2.0
    else:
        ref = np.concatenate([rng.uniform(0.0, 1.0, size=(B, Lq, L, 2)),
                              rng.uniform(0.02, 0.8, size=(B, Lq, L, 2))], -1)
        off = rng.standard_normal((B, Lq, M, L, K, 2)) * K / 2.0
    f32 = lambda a: np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return W.FusedInputs(
        config=W.CONFIGS["tiny_fp32"], value=f32(rng.standard_normal((B, S, M, D))),
        value_bf16_bits=None, spatial_shapes=ss, level_start_index=st,
        reference_points=f32(ref), sampling_offsets=f32(off),
        attention_logits=f32(rng.standard_normal((B, Lq, M, L * K)) * 2.0),
        grad_output=f32(rng.standard_normal((B, Lq, M * D))))


@pytest.mark.parametrize("case", [
    # (B, Lq, M, D, K, shapes, R): several tiles, ragged query / channel / point counts
    (2, 37, 3, 4, 3, ((7, 5), (3, 4), (2, 2)), 2),
    (1, 129, 5, 12, 5, ((9, 11), (4, 6)), 4),
    (3, 50, 8, 32, 4, ((20, 30), (10, 15), (5, 8), (3, 4)), 2),
    (2, 65, 2, 64, 8, ((12, 16), (6, 8)), 4),
    (1, 23, 4, 128, 2, ((6, 6),), 2),
    (2, 41, 3, 20, 1, ((5, 9), (3, 5), (2, 3)), 4),
], ids=lambda c: f"B{c[0]}Lq{c[1]}M{c[2]}D{c[3]}K{c[4]}L{len(c[5])}R{c[6]}")
def test_fused_random_shapes(case):
    B, Lq, M, D, K, shapes, R = case
    inp = _random_fused(np.random.default_rng(B * 1000 + Lq), B, Lq, M, D, K, list(shapes), R)
    d = fused_device(inp)
    G.assert_forward_f32(gpu_fused_forward(d), oracle_fused_forward(inp), f"{case} forward")
    check_fused_backward(inp, d, str(case))


def test_fused_nan_logit_poisons_its_group():
    """A NaN logit makes every weight of its (b, q, m) NaN, as the softmax does;
    the NaN pattern of every output matches the oracle's."""
    inp = _random_fused(np.random.default_rng(5), 2, 9, 3, 8, 2, [(6, 7), (3, 4)], 2)
    inp.attention_logits[1, 4, 2, 3] = np.nan
    d = fused_device(inp)
    out = gpu_fused_forward(d)
    assert np.isnan(out[1, 4, 2 * 8:3 * 8]).all()
    G.assert_forward_f32(out, oracle_fused_forward(inp), "NaN-logit forward")
    check_fused_backward(inp, d, "NaN-logit")


def test_fused_reference_gradient_is_optional():
    inp = _random_fused(np.random.default_rng(6), 2, 33, 4, 16, 3, [(9, 8), (4, 5)], 4)
    d = fused_device(inp)
    gv, goff, gz, gref = gpu_fused_backward(d, reference_grad=False)
    assert gref is None
    rv, roff, rz, _ = oracle_fused_backward(inp)
    G.assert_backward_f32(gv, rv, "grad_value without reference gradient")
    G.assert_backward_f32(goff, roff, "grad_sampling_offsets without reference gradient")
    G.assert_backward_f32(gz, rz, "grad_attention_logits without reference gradient")


def test_fused_autograd():
    """ms_deform_attn_fused under torch autograd gives the oracle's gradients."""
    inp = _random_fused(np.random.default_rng(7), 1, 20, 2, 8, 2, [(6, 5), (3, 3)], 2)
    d = fused_device(inp)
    v = d["value"].clone().requires_grad_(True)
    r = d["reference_points"].clone().requires_grad_(True)
    o = d["sampling_offsets"].clone().requires_grad_(True)
    z = d["attention_logits"].clone().requires_grad_(True)
    out = binding.ms_deform_attn_fused(v, d["spatial_shapes"], d["level_start_index"], r, o, z)
    out.backward(d["grad_output"])
    torch.cuda.synchronize()
    rv, roff, rz, rref = oracle_fused_backward(inp)
    G.assert_backward_f32(v.grad.cpu().numpy().astype(np.float64), rv, "autograd grad_value")
    G.assert_backward_f32(o.grad.cpu().numpy().astype(np.float64), roff, "autograd grad_offsets")
    G.assert_backward_f32(z.grad.cpu().numpy().astype(np.float64), rz, "autograd grad_logits")
    G.assert_backward_f32(r.grad.cpu().numpy().astype(np.float64), rref, "autograd grad_reference")


def test_offset_init_grid():
    """The pages' initial sampling pattern: point k of head m at (k + 1) pixels
    along the head's compass direction from pixel-centre reference points, on
    maps whose sides are powers of two.  On a token's own level every sample
    lands exactly on a pixel centre, so three of its four corner weights are
    exactly zero, and neighbouring points share corners where one side's weight
    is zero (which the backward's corner merge must leave unmerged).  The fused
    op, and the core on the same float32 locations and weights, against the
    oracle."""
    import dataclasses
    from oracle_pins import load_offset_init_directions

    shapes = ((16, 32), (8, 16), (4, 8), (2, 4))
    cfg = W.Config("init_grid", 1, 8, 32, 4, shapes, "encoder", "f32", True)
    fz = W.make_fused_inputs(cfg, seed=3)
    B, Lq, M, L, K = 1, cfg.queries, 8, 4, 4
    dirs = load_offset_init_directions().astype(np.float32)         # [8, (dx, dy)]
    off = np.empty((B, Lq, M, L, K, 2), dtype=np.float32)
    for k in range(K):
        off[:, :, :, :, k, :] = (k + 1) * dirs[None, None, :, None, :]
    fz = dataclasses.replace(fz, sampling_offsets=off)
    d = fused_device(fz)
    G.assert_forward_f32(gpu_fused_forward(d), oracle_fused_forward(fz), "init grid fused forward")
    check_fused_backward(fz, d, "init grid fused")

    # The core on the locations and weights the pages form (float32, their order).
    wh = fz.spatial_shapes[:, ::-1].astype(np.float32)              # [L, (W, H)]
    loc = (fz.reference_points[:, :, None, :, None, :] + off / wh[None, None, None, :, None, :])
    z = fz.attention_logits.astype(np.float64)
    a = np.exp(z - z.max(-1, keepdims=True))
    a = (a / a.sum(-1, keepdims=True)).astype(np.float32).reshape(B, Lq, M, L, K)
    inp = W.Inputs(cfg, fz.value, None, fz.spatial_shapes, fz.level_start_index,
                   np.ascontiguousarray(loc.astype(np.float32)), np.ascontiguousarray(a),
                   fz.grad_output)
    x = loc[..., 0].astype(np.float64) * wh[None, None, None, :, None, 0] - 0.5
    assert np.mean(x == np.floor(x)) > 0.2, "too few samples on pixel centres"
    cd = G.device_inputs(inp)
    G.assert_forward_f32(G.gpu_forward(cd), G.oracle_forward(inp), "init grid forward")
    G.check_backward_paths(cd, inp, "init grid")
