"""Pins of the oracle's fused entry points (locations and weights formed from
raw reference points, sampling offsets and attention logits), each checked
against something other than the oracle itself.

What the fused step computes ("Deformable DETR模型解读（附源码+论文）",
MultiScaleDeformableAttention.forward, and the MSDeformAttn.forward printed on
the phdsky.com notes of "Deformable DETR: Deformable Transformers for
End-to-End Object Detection"):
  - attention weights are a softmax over the L*K logits of each (b, q, m);
  - 2-component reference points: loc = ref + off / (W_l, H_l);
  - 4-component (box) reference points: loc = ref[:2] + off / K * ref[2:] * 0.5.

Each pin function takes an ``oracle.Oracle`` and raises AssertionError on a
mismatch.  ``FIRST_PRINCIPLES_PINS`` are those that do not call torch.
"""
from __future__ import annotations

import numpy as np

from oracle_pins import _close, _meta, grid_sample_core, load_offset_init_directions


def _f32(a):
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _fused_case(rng, B, M, D, K, shapes, Lq, R):
    """Random inputs; reference points, offsets and logits are float32 values."""
    ss, start, S = _meta(shapes)
    L = len(shapes)
    value = rng.standard_normal((B, S, M, D))
    if R == 2:
        ref = rng.uniform(0.02, 0.98, size=(B, Lq, L, 2))
        off = rng.standard_normal((B, Lq, M, L, K, 2)) * 2.0      # pixels of level l
    else:
        ref = np.concatenate([rng.uniform(0.1, 0.9, size=(B, Lq, L, 2)),
                              rng.uniform(0.05, 0.7, size=(B, Lq, L, 2))], axis=-1)
        off = rng.standard_normal((B, Lq, M, L, K, 2)) * 1.5      # box units
    logits = rng.standard_normal((B, Lq, M, L * K)) * 2.0
    grad = rng.standard_normal((B, Lq, M * D))
    return value, ss, start, _f32(ref), _f32(off), _f32(logits), grad


def torch_fused(value, ss, start, ref, off, logits, grad=None, f32_locations=False):
    """The pages' formulation in torch: softmax of the logits, locations from the
    reference points and offsets (float32 arithmetic when ``f32_locations``, as the
    pages' float32 tensors compute it), then the grid_sample core in float64.
    With ``grad`` it also returns the autograd gradients (float64 locations only)."""
    import torch

    req = grad is not None
    v = torch.tensor(value, dtype=torch.float64, requires_grad=req)
    r = torch.tensor(ref, dtype=torch.float64, requires_grad=req)
    o = torch.tensor(off, dtype=torch.float64, requires_grad=req)
    z = torch.tensor(logits, dtype=torch.float64, requires_grad=req)
    B, Lq, M, LK = z.shape
    L = ss.shape[0]
    K = LK // L
    A = torch.softmax(z, -1).reshape(B, Lq, M, L, K)
    R = r.shape[-1]
    dt = torch.float32 if f32_locations else torch.float64
    rr, oo = r.to(dt), o.to(dt)
    if R == 2:
        norm = torch.tensor(np.stack([ss[:, 1], ss[:, 0]], -1), dtype=dt)   # (W, H)
        loc = rr[:, :, None, :, None, :] + oo / norm[None, None, None, :, None, :]
    else:
        loc = rr[:, :, None, :, None, :2] + oo / K * rr[:, :, None, :, None, 2:] * 0.5
    loc = loc.to(torch.float64)
    out = grid_sample_core(v, loc, A, ss, start)
    if grad is None:
        return out.detach().numpy()
    out.backward(torch.tensor(grad, dtype=torch.float64).reshape(out.shape))
    return (out.detach().numpy(), v.grad.numpy(), o.grad.numpy(), z.grad.numpy(),
            r.grad.numpy())


# ----------------------------------------------------------------------------
# torch: the pages' formulation with autograd
# ----------------------------------------------------------------------------

def pin_fused_torch(orc):
    """Forward with float32-formed locations, and forward plus every gradient
    with float64 locations, agree with torch (softmax, the offset normaliser or
    the box formula, grid_sample, autograd) for both kinds of reference points."""
    for R, seed in ((2, 31), (4, 32)):
        rng = np.random.default_rng(seed)
        shapes = [(6, 9), (3, 5), (2, 3)]
        v, ss, st, ref, off, z, g = _fused_case(rng, 2, 3, 5, 3, shapes, 11, R)
        _close(orc.fused_forward(v, ss, st, ref, off, z, round_f32=True),
               torch_fused(v, ss, st, ref, off, z, f32_locations=True), 1e-12, 1e-12,
               f"fused forward, float32 locations, R={R}")
        t_out, t_gv, t_goff, t_gz, t_gref = torch_fused(v, ss, st, ref, off, z, grad=g)
        _close(orc.fused_forward(v, ss, st, ref, off, z, round_f32=False), t_out,
               1e-12, 1e-12, f"fused forward, R={R}")
        gv, goff, gz, gref = orc.fused_backward(v, ss, st, ref, off, z, g, round_f32=False)
        _close(gv, t_gv, 1e-12, 1e-12, f"grad_value, R={R}")
        _close(goff, t_goff, 1e-10, 1e-11, f"grad_sampling_offsets, R={R}")
        _close(gz, t_gz, 1e-10, 1e-11, f"grad_attention_logits, R={R}")
        _close(gref, t_gref, 1e-10, 1e-11, f"grad_reference_points, R={R}")


# ----------------------------------------------------------------------------
# softmax: shift invariance and zero-sum logit gradients
# ----------------------------------------------------------------------------

def pin_fused_softmax_invariants(orc):
    """A softmax ignores a constant added to a group's logits -- even one large
    enough to overflow exp without the max subtraction -- and its Jacobian maps
    any upstream gradient to logit gradients that sum to zero over the group."""
    rng = np.random.default_rng(33)
    shapes = [(5, 7), (3, 4)]
    v, ss, st, ref, off, z, g = _fused_case(rng, 2, 2, 4, 3, shapes, 6, 2)
    shift = rng.choice([-800.0, 800.0], size=z.shape[:3] + (1,))
    base = orc.fused_backward(v, ss, st, ref, off, z, g)
    moved = orc.fused_backward(v, ss, st, ref, off, z + shift, g)
    _close(orc.fused_forward(v, ss, st, ref, off, z + shift),
           orc.fused_forward(v, ss, st, ref, off, z), 1e-10, 1e-12, "output under a logit shift")
    for a, b, what in zip(moved, base, ("grad_value", "grad_offsets", "grad_logits", "grad_ref")):
        _close(a, b, 1e-9, 1e-12, f"{what} under a logit shift")
    gz = base[2]
    assert np.all(np.abs(gz.sum(-1)) <= 1e-12 * np.abs(gz).sum(-1) + 1e-300), \
        "logit gradients do not sum to zero over a group"


# ----------------------------------------------------------------------------
# constant field: the softmax weights sum to one; every location gradient is 0
# ----------------------------------------------------------------------------

def pin_fused_constant_field(orc):
    """A value field constant over the pixels (per head and channel), sampled at
    interior locations, returns that constant: the weights of each (b, q, m)
    sum to one.  Then every point has the same grad_attn, so the logit gradients
    vanish, and the field has no slope, so the offset and reference-point
    gradients vanish too."""
    rng = np.random.default_rng(34)
    shapes = [(8, 12), (6, 5)]
    ss, st, S = _meta(shapes)
    B, M, D, K, Lq = 2, 3, 4, 2, 5
    L = len(shapes)
    c = rng.standard_normal((M, D))
    v = np.broadcast_to(c, (B, S, M, D)).copy()
    for R in (2, 4):
        if R == 2:
            ref = _f32(rng.uniform(0.35, 0.65, size=(B, Lq, L, 2)))
            off = _f32(rng.uniform(-0.4, 0.4, size=(B, Lq, M, L, K, 2)))
        else:
            ref = _f32(np.concatenate([rng.uniform(0.35, 0.65, size=(B, Lq, L, 2)),
                                       rng.uniform(0.05, 0.2, size=(B, Lq, L, 2))], -1))
            off = _f32(rng.uniform(-1.0, 1.0, size=(B, Lq, M, L, K, 2)))
        z = _f32(rng.standard_normal((B, Lq, M, L * K)))
        g = rng.standard_normal((B, Lq, M * D))
        out = orc.fused_forward(v, ss, st, ref, off, z)
        _close(out, np.broadcast_to(c.reshape(-1), out.shape), 1e-13, 1e-13,
               f"constant field, R={R}")
        gv, goff, gz, gref = orc.fused_backward(v, ss, st, ref, off, z, g)
        scale = np.abs(g).max() * np.abs(c).max()
        assert np.abs(gz).max() <= 1e-13 * scale, f"logit gradients on a constant field, R={R}"
        assert np.abs(goff).max() <= 1e-13 * scale, f"offset gradients on a constant field, R={R}"
        assert np.abs(gref).max() <= 1e-13 * scale, f"reference gradients on a constant field, R={R}"


# ----------------------------------------------------------------------------
# the pages' offset initialisation lands on pixel centres (both reference kinds)
# ----------------------------------------------------------------------------

def pin_fused_offset_init(orc):
    """Offsets from the pages' initialisation -- point k of head m at (k + 1)
    pixels along the head's compass direction -- around a pixel-centre reference
    point sample whole pixels, so out = sum A * value[that pixel] exactly.  The
    same holds for a box reference of size (2K / W_l, 2K / H_l), for which
    off / K * size * 0.5 = off / (W_l, H_l).  Levels are non-square powers of
    two, so float32 arithmetic is exact and a swapped normaliser or box term
    moves the samples."""
    dirs = load_offset_init_directions()                          # [8, (dx, dy)]
    rng = np.random.default_rng(35)
    shapes = [(16, 8), (8, 32), (8, 16)]
    ss, st, S = _meta(shapes)
    B, M, D, K, Lq = 2, 8, 3, 2, 2
    L = len(shapes)
    v = rng.standard_normal((B, S, M, D))
    centres = [(7, 3), (4, 20), (3, 9)]                          # (row, col) per level
    z = _f32(rng.standard_normal((B, Lq, M, L * K)))
    e = np.exp(z - z.max(-1, keepdims=True))
    A = (e / e.sum(-1, keepdims=True)).reshape(B, Lq, M, L, K)
    off = np.empty((B, Lq, M, L, K, 2))
    expect = np.zeros((B, Lq, M, D))
    ref2 = np.empty((B, Lq, L, 2))
    ref4 = np.empty((B, Lq, L, 4))
    for l, (h, w) in enumerate(shapes):
        r0, c0 = centres[l]
        ref2[:, :, l] = ((c0 + 0.5) / w, (r0 + 0.5) / h)
        ref4[:, :, l] = ((c0 + 0.5) / w, (r0 + 0.5) / h, 2.0 * K / w, 2.0 * K / h)
        for m in range(M):
            for k in range(K):
                dx, dy = (k + 1) * dirs[m, 0], (k + 1) * dirs[m, 1]
                off[:, :, m, l, k] = (dx, dy)
                pix = st[l] + (r0 + dy) * w + (c0 + dx)
                expect[:, :, m, :] += A[:, :, m, l, k, None] * v[:, None, pix, m, :]
    for R, ref in ((2, ref2), (4, ref4)):
        out = orc.fused_forward(v, ss, st, ref, off, z).reshape(B, Lq, M, D)
        _close(out, expect, 1e-14, 1e-14, f"offset-initialisation grid, R={R}")


# ----------------------------------------------------------------------------
# boxes of zero size ignore the offsets
# ----------------------------------------------------------------------------

def pin_fused_zero_box(orc):
    """A box reference of zero size puts every sample at the box centre, so the
    output does not depend on the offsets and their gradient is exactly 0."""
    rng = np.random.default_rng(36)
    shapes = [(6, 9), (3, 5)]
    v, ss, st, ref, off, z, g = _fused_case(rng, 2, 2, 4, 3, shapes, 5, 4)
    ref = ref.copy()
    ref[..., 2:] = 0.0
    out1 = orc.fused_forward(v, ss, st, ref, off, z)
    out2 = orc.fused_forward(v, ss, st, ref, off * -3.0 + 1.0, z)
    assert np.array_equal(out1, out2), "zero-size boxes depend on the offsets"
    goff = orc.fused_backward(v, ss, st, ref, off, z, g)[1]
    assert np.all(goff == 0.0), "offset gradient of zero-size boxes"


# ----------------------------------------------------------------------------
# central finite differences (float64 locations)
# ----------------------------------------------------------------------------

def _pixel_coords(ss, ref, off, K, R):
    """Float64 pixel coordinates x = loc * W - 0.5 of every point, [B,Lq,M,L,K,2]."""
    L = ss.shape[0]
    W = ss[:, 1].astype(np.float64)
    H = ss[:, 0].astype(np.float64)
    r = ref[:, :, None, :, None, :]
    if R == 2:
        loc = r + off / np.stack([W, H], -1)[None, None, None, :, None, :]
    else:
        loc = r[..., :2] + off / K * r[..., 2:] * 0.5
    return loc * np.stack([W, H], -1)[None, None, None, :, None, :] - 0.5


def pin_fused_finite_differences(orc):
    """Every gradient of J = <grad_output, output> w.r.t. offsets, logits and
    reference points matches central differences (step 1e-6) in float64, away
    from integer pixel coordinates where the bilinear derivative jumps."""
    for R, seed in ((2, 37), (4, 38)):
        rng = np.random.default_rng(seed)
        shapes = [(5, 7), (3, 4)]
        v, ss, st, ref, off, z, g = _fused_case(rng, 1, 2, 3, 2, shapes, 4, R)
        K = off.shape[4]
        _, goff, gz, gref = orc.fused_backward(v, ss, st, ref, off, z, g, round_f32=False)
        J = lambda r_, o_, z_: float(np.sum(g * orc.fused_forward(v, ss, st, r_, o_, z_,
                                                                  round_f32=False)))
        h = 1e-6
        px = _pixel_coords(ss, ref, off, K, R)
        frac = np.abs(px - np.round(px))
        near = frac < 1e-3                                       # [B,Lq,M,L,K,2]
        checked = 0
        for idx in np.ndindex(off.shape):
            if near[idx]:
                continue
            d = np.zeros_like(off)
            d[idx] = h
            fd = (J(ref, off + d, z) - J(ref, off - d, z)) / (2 * h)
            assert abs(fd - goff[idx]) <= 1e-5 * abs(fd) + 1e-7, f"d/d offset {idx}, R={R}"
            checked += 1
        for idx in np.ndindex(z.shape):
            d = np.zeros_like(z)
            d[idx] = h
            fd = (J(ref, off, z + d) - J(ref, off, z - d)) / (2 * h)
            assert abs(fd - gz[idx]) <= 1e-5 * abs(fd) + 1e-7, f"d/d logit {idx}, R={R}"
        for idx in np.ndindex(ref.shape):
            b, q, l, c = idx
            if near[b, q, :, l, :, :].any():
                continue
            d = np.zeros_like(ref)
            d[idx] = h
            fd = (J(ref + d, off, z) - J(ref - d, off, z)) / (2 * h)
            assert abs(fd - gref[idx]) <= 1e-5 * abs(fd) + 1e-7, f"d/d reference {idx}, R={R}"
            checked += 1
        assert checked > 20, "too few finite-difference checks"


ALL_PINS = [
    pin_fused_torch,
    pin_fused_softmax_invariants,
    pin_fused_constant_field,
    pin_fused_offset_init,
    pin_fused_zero_box,
    pin_fused_finite_differences,
]

FIRST_PRINCIPLES_PINS = [p for p in ALL_PINS if p is not pin_fused_torch]
