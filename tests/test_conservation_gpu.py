"""Conservation of grad_value on a batch four times the training workload's, for
every backward path: no reduction may be lost or doubled.

Each point scatters A * w_c * gO into its corners inside the map, so summed over
all pixels, for every (b, m, d),
    sum_s grad_value[b, s, m, d] = sum_q gO[b, q, m, d] * sum_{l,k} A * mass,
where mass is the bilinear weight of the point's corners inside the map
(1 for an interior point).  The right side is computed here in float64 from the
inputs; it holds at any size, so the oracle need not run on all 79,788 x 4
queries ("Deformable DETR模型解读（附源码+论文）", ms_deform_attn_core_pytorch:
bilinear sampling with zeros padding, whose adjoint spreads each sample's
gradient over the same corners with the same weights)."""
import numpy as np
import pytest
import torch

import gpu_support as G
from scale_deformable_attention_backward_b200 import binding
from scale_deformable_attention_backward_b200 import workloads as W

pytestmark = pytest.mark.gpu


def in_map_mass(loc, shapes):
    """[B, Lq, M, L, K] bilinear weight of the corners inside each level."""
    mass = np.zeros(loc.shape[:-1])
    for l, (H, Wd) in enumerate(shapes):
        x = loc[..., l, :, 0].astype(np.float64) * Wd - 0.5
        y = loc[..., l, :, 1].astype(np.float64) * H - 0.5
        x0, y0 = np.floor(x), np.floor(y)
        fx, fy = x - x0, y - y0
        ok = lambda v, n: (v >= 0) & (v < n)
        wx = [np.where(ok(x0, Wd), 1 - fx, 0.0), np.where(ok(x0 + 1, Wd), fx, 0.0)]
        wy = [np.where(ok(y0, H), 1 - fy, 0.0), np.where(ok(y0 + 1, H), fy, 0.0)]
        mass[..., l, :] = (wx[0] + wx[1]) * (wy[0] + wy[1])
    return mass


@pytest.fixture(scope="module")
def problem():
    cfg = W.CONFIGS["encoder_train_fp32"].with_batch(16)
    inp = W.make_inputs(cfg, seed=21)
    B, S, M, D = inp.value.shape
    Lq = inp.sampling_locations.shape[1]
    mass = in_map_mass(inp.sampling_locations, [tuple(s) for s in inp.spatial_shapes])
    per_query = (inp.attention_weights.astype(np.float64) * mass).sum(axis=(3, 4))  # [B, Lq, M]
    go = inp.grad_output.astype(np.float64).reshape(B, Lq, M, D)
    want = np.einsum("bqm,bqmd->bmd", per_query, go)
    scale = np.einsum("bqm,bqmd->bmd", np.abs(per_query), np.abs(go))
    return G.device_inputs(inp), want, scale


@pytest.mark.parametrize("path", ["direct", "sorted", "deterministic"])
def test_grad_value_conserves_the_scattered_mass(problem, path):
    d, want, scale = problem
    kw = {"workspace": "auto"} if path == "sorted" else {}
    if path == "deterministic":
        kw = {"deterministic": True}
    gv, _, _ = binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                                d["sampling_locations"], d["attention_weights"], d["grad_output"],
                                **kw)
    got = gv.sum(dim=1, dtype=torch.float64).cpu().numpy()          # [B, M, D]
    err = np.abs(got - want)
    worst = np.unravel_index(err.argmax(), err.shape)
    assert np.all(err <= 1e-5 * scale + 1e-6), \
        f"{path}: worst {err[worst]:.3e} against scale {scale[worst]:.3e}"
