"""Pins that tie the float64 oracle to what the pages and mathematics fix.

Each ``pin_*`` function takes an :class:`oracle.Oracle` handle and raises
``AssertionError`` if the oracle disagrees.  They run against the real oracle in
``test_oracle_pins.py`` and against deliberately broken copies of it in
``test_oracle_mutants.py`` (every planted mistake must fail at least one pin).

No pin re-types the oracle's formula.  Expected values come from:
  * exact special cases of the pages' sampling rule ("Deformable DETR模型解读",
    ms_deform_attn_core_pytorch: grid = 2*loc - 1, bilinear, zeros padding,
    align_corners=False), e.g. a pixel-centre location returns that pixel;
  * closed forms (bilinear interpolation reproduces affine fields exactly, so
    outputs and location gradients of an affine field are known analytically);
  * invariants (constant field, linearity, the adjoint identity between the
    forward and grad_value, finite differences of the forward);
  * the library routine the pages build on, ``torch.nn.functional.grid_sample``
    in float64 on the CPU, with its autograd gradients.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------
# helpers (input construction only)
# ----------------------------------------------------------------------------

def _meta(shapes):
    ss = np.asarray(shapes, dtype=np.int64).reshape(-1, 2)
    sizes = ss[:, 0] * ss[:, 1]
    start = np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64)
    return ss, start, int(sizes.sum())


def _random_case(rng, B, M, D, K, shapes, Lq, loc_lo=-0.15, loc_hi=1.15):
    ss, start, S = _meta(shapes)
    L = len(shapes)
    value = rng.standard_normal((B, S, M, D))
    loc = rng.uniform(loc_lo, loc_hi, size=(B, Lq, M, L, K, 2))
    attn = rng.uniform(0.0, 1.0, size=(B, Lq, M, L, K))
    attn /= attn.sum(axis=(3, 4), keepdims=True)
    grad = rng.standard_normal((B, Lq, M * D))
    return value, ss, start, loc, attn, grad


def _interior_locations(rng, shapes, size):
    """Locations whose four bilinear corners all lie inside their level's map,
    i.e. pixel coordinates x = loc_x*W - 0.5 in [0, W-1] (same for y), kept
    a margin away from integer pixel coordinates."""
    L = len(shapes)
    loc = np.empty(size + (L, 1, 2))
    for l, (h, w) in enumerate(shapes):
        for comp, n in ((0, w), (1, h)):
            cells = rng.integers(0, n - 1, size=size)
            frac = rng.uniform(0.05, 0.95, size=size)
            loc[..., l, 0, comp] = (cells + frac + 0.5) / n
    return loc


def _close(a, b, rtol, atol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.abs(a - b)
    bound = atol + rtol * np.abs(b)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} differ, "
                           f"max err {err.max():.3e}")


# ----------------------------------------------------------------------------
# P-1: a location at a pixel centre returns that pixel (coordinate convention)
# ----------------------------------------------------------------------------

def pin_pixel_centre(orc):
    """M=L=K=1 (and a second level selected by a one-hot weight): the location
    ((j + 0.5)/W, (i + 0.5)/H) -- the encoder reference points of
    get_reference_points -- returns value[start + i*W + j] exactly.  Shapes are
    powers of two and deliberately not square, so the float arithmetic is exact
    and a swap of W and H, of x and y, or of the level start cannot pass."""
    rng = np.random.default_rng(1)
    shapes = [(4, 8), (2, 16)]
    ss, start, S = _meta(shapes)
    D = 3
    value = rng.standard_normal((1, S, 1, D))
    for lvl, (h, w) in enumerate(shapes):
        ii, jj = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
        ii, jj = ii.reshape(-1), jj.reshape(-1)
        Lq = ii.size
        loc = np.zeros((1, Lq, 1, 2, 1, 2))
        loc[0, :, 0, :, 0, 0] = ((jj + 0.5) / w)[:, None]
        loc[0, :, 0, :, 0, 1] = ((ii + 0.5) / h)[:, None]
        attn = np.zeros((1, Lq, 1, 2, 1))
        attn[:, :, :, lvl, :] = 1.0
        out = orc.forward(value, ss, start, loc, attn)
        expect = value[0, start[lvl] + ii * w + jj, 0, :]
        assert np.array_equal(out[0], expect), f"pixel-centre sample wrong on level {lvl}"


def load_offset_init_directions():
    """The 8 head directions of the sampling-offset initialisation (golden
    fixture ``tests/golden/offset_init_directions.txt``, cited there)."""
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                        "offset_init_directions.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    return np.array([[int(r[1]), int(r[2])] for r in rows], dtype=np.int64)


def pin_offset_init_grid(orc):
    """The pages' initial sampling pattern: head m samples point k of every level
    at (k + 1) pixels along its compass direction from a pixel-centre reference
    point.  Offsets are whole pixels, so every sample lands on a pixel centre and
    returns that pixel exactly: out = sum_{l,k} A * value[that pixel]."""
    dirs = load_offset_init_directions()                          # [8, (dx, dy)]
    rng = np.random.default_rng(11)
    shapes = [(16, 16), (8, 16), (16, 8)]
    ss, start, S = _meta(shapes)
    B, M, D, K = 2, 8, 3, 3
    L = len(shapes)
    value = rng.standard_normal((B, S, M, D))
    refs = [(7, 8), (4, 9), (8, 3)]                               # (row, col) per level
    Lq = 2
    loc = np.empty((B, Lq, M, L, K, 2))
    expect = np.zeros((B, Lq, M, D))
    attn = rng.uniform(size=(B, Lq, M, L, K))
    for l, (h, w) in enumerate(shapes):
        r0, c0 = refs[l]
        for m in range(M):
            for k in range(K):
                col, row = c0 + (k + 1) * dirs[m, 0], r0 + (k + 1) * dirs[m, 1]
                loc[:, :, m, l, k, 0] = (col + 0.5) / w
                loc[:, :, m, l, k, 1] = (row + 0.5) / h
                pix = start[l] + row * w + col
                expect[:, :, m, :] += attn[:, :, m, l, k, None] * value[:, None, pix, m, :]
    out = orc.forward(value, ss, start, loc, attn).reshape(B, Lq, M, D)
    _close(out, expect, 1e-14, 1e-14, "offset-initialisation grid samples")


# ----------------------------------------------------------------------------
# P-1b / P-2: the half-pixel shift and zero padding
# ----------------------------------------------------------------------------

def pin_half_pixel_and_padding(orc):
    """loc_x = j/W puts the sample on the border between pixels j-1 and j, so it
    returns their mean; at j = 0 the left neighbour is outside the map and
    contributes zero (zeros padding), leaving half of pixel 0."""
    rng = np.random.default_rng(2)
    h, w = 4, 8
    ss, start, S = _meta([(h, w)])
    value = rng.standard_normal((1, S, 1, 2))
    grid = value[0, :, 0, :].reshape(h, w, 2)
    rows = np.arange(h)
    cols = np.arange(w)
    ii, jj = np.meshgrid(rows, cols, indexing="ij")
    ii, jj = ii.reshape(-1), jj.reshape(-1)
    loc = np.zeros((1, ii.size, 1, 1, 1, 2))
    loc[0, :, 0, 0, 0, 0] = jj / w
    loc[0, :, 0, 0, 0, 1] = (ii + 0.5) / h
    attn = np.ones((1, ii.size, 1, 1, 1))
    out = orc.forward(value, ss, start, loc, attn)[0]
    left = np.where((jj > 0)[:, None], grid[ii, np.maximum(jj - 1, 0)], 0.0)
    expect = 0.5 * left + 0.5 * grid[ii, jj]
    _close(out, expect, 1e-15, 1e-15, "half-pixel sample")

    # Same along y: loc_y = i/H is the border between rows i-1 and i.
    loc2 = np.zeros_like(loc)
    loc2[0, :, 0, 0, 0, 0] = (jj + 0.5) / w
    loc2[0, :, 0, 0, 0, 1] = ii / h
    out2 = orc.forward(value, ss, start, loc2, attn)[0]
    up = np.where((ii > 0)[:, None], grid[np.maximum(ii - 1, 0), jj], 0.0)
    _close(out2, 0.5 * up + 0.5 * grid[ii, jj], 1e-15, 1e-15, "half-pixel sample (y)")


def pin_fully_outside(orc):
    """Locations whose every corner lies outside the map (x < -1, x >= W, or the
    same for y) read nothing: output, and all gradients, are exactly zero."""
    rng = np.random.default_rng(3)
    shapes = [(5, 7), (3, 4)]
    ss, start, S = _meta(shapes)
    B, M, D, K, Lq = 2, 2, 3, 3, 6
    value = rng.standard_normal((B, S, M, D))
    loc = np.empty((B, Lq, M, 2, K, 2))
    choices = np.array([[-0.6, 0.5], [1.5, 0.5], [0.5, -0.7], [0.5, 1.8], [-2.0, -3.0],
                        [4.0, 9.0]])
    for q in range(Lq):
        loc[:, q] = choices[q]
    # x = loc*W - 0.5 < -1  <=>  loc < -0.5/W; x >= W  <=>  loc >= (W + 0.5)/W.
    attn = rng.uniform(0.1, 1.0, size=(B, Lq, M, 2, K))
    grad = rng.standard_normal((B, Lq, M * D))
    out = orc.forward(value, ss, start, loc, attn)
    assert np.all(out == 0.0), "a sample outside the map must be zero"
    gv, gl, ga = orc.backward(value, ss, start, loc, attn, grad)
    assert np.all(gv == 0.0) and np.all(gl == 0.0) and np.all(ga == 0.0), \
        "gradients of samples outside the map must be zero"


# ----------------------------------------------------------------------------
# P-3: constant field; P-4: linearity
# ----------------------------------------------------------------------------

def pin_constant_field(orc):
    """A value field constant over each level's pixels (per head and channel),
    sampled where all four corners are inside, returns the constant times the sum
    of the weights (here 1), and its location gradient is zero."""
    rng = np.random.default_rng(4)
    shapes = [(6, 9), (4, 5), (3, 3)]
    ss, start, S = _meta(shapes)
    B, M, D, K, Lq = 2, 3, 4, 2, 7
    c = rng.standard_normal((M, D))
    value = np.broadcast_to(c, (B, S, M, D)).copy()
    loc = np.repeat(_interior_locations(rng, shapes, (B, Lq, M)), K, axis=4)
    loc += rng.uniform(-1e-3, 1e-3, size=loc.shape) / 50.0
    attn = rng.uniform(0.0, 1.0, size=(B, Lq, M, len(shapes), K))
    attn /= attn.sum(axis=(3, 4), keepdims=True)
    out = orc.forward(value, ss, start, loc, attn).reshape(B, Lq, M, D)
    _close(out, np.broadcast_to(c, out.shape), 1e-13, 1e-13, "constant field")
    grad = rng.standard_normal((B, Lq, M * D))
    _, gl, _ = orc.backward(value, ss, start, loc, attn, grad)
    _close(gl, np.zeros_like(gl), 0.0, 1e-11, "location gradient of a constant field")


def pin_linearity(orc):
    """The output is linear in value and in the attention weights."""
    rng = np.random.default_rng(5)
    shapes = [(5, 6), (3, 2)]
    v1, ss, start, loc, a1, _ = _random_case(rng, 2, 2, 3, 3, shapes, 9)
    v2 = rng.standard_normal(v1.shape)
    a2 = rng.uniform(size=a1.shape)
    f = lambda v, a: orc.forward(v, ss, start, loc, a)
    _close(f(2.0 * v1 - 3.0 * v2, a1), 2.0 * f(v1, a1) - 3.0 * f(v2, a1), 1e-12, 1e-12,
           "linearity in value")
    _close(f(v1, 0.5 * a1 + 1.5 * a2), 0.5 * f(v1, a1) + 1.5 * f(v1, a2), 1e-12, 1e-12,
           "linearity in attention weights")


# ----------------------------------------------------------------------------
# P-5 / P-6: affine fields (closed forms for output, grad_loc and grad_attn)
# ----------------------------------------------------------------------------

def _affine_case(rng, shapes, B, M, D, K, Lq):
    """value(level l, pixel (col x, row y), head m, channel d) =
    alpha[l,m,d]*x + beta[l,m,d]*y + gamma[l,m,d]."""
    ss, start, S = _meta(shapes)
    L = len(shapes)
    alpha = rng.standard_normal((L, M, D))
    beta = rng.standard_normal((L, M, D))
    gamma = rng.standard_normal((L, M, D))
    value = np.empty((B, S, M, D))
    for l, (h, w) in enumerate(shapes):
        ys, xs = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
        xs, ys = xs.reshape(-1), ys.reshape(-1)
        field = (alpha[l][None] * xs[:, None, None] + beta[l][None] * ys[:, None, None]
                 + gamma[l][None])
        value[:, start[l]:start[l] + h * w] = field[None]
    loc = np.concatenate([_interior_locations(rng, shapes, (B, Lq, M)) for _ in range(K)],
                         axis=4)
    attn = rng.uniform(0.0, 1.0, size=(B, Lq, M, L, K))
    attn /= attn.sum(axis=(3, 4), keepdims=True)
    return value, ss, start, loc, attn, alpha, beta, gamma


def pin_affine_field(orc):
    """Bilinear interpolation reproduces an affine field exactly, so a sample at
    pixel coordinate (X, Y) = (loc_x*W - 0.5, loc_y*H - 0.5) is
    alpha*X + beta*Y + gamma.  Then, in closed form:
      out[b,q,m,d]      = sum_{l,k} A * (alpha X + beta Y + gamma)
      grad_attn[..l,k]  = sum_d gO * (alpha X + beta Y + gamma)
      grad_loc[..l,k]   = A * (W * sum_d gO*alpha, H * sum_d gO*beta)."""
    rng = np.random.default_rng(6)
    shapes = [(7, 11), (4, 6), (2, 3)]
    B, M, D, K, Lq = 2, 3, 4, 3, 5
    value, ss, start, loc, attn, alpha, beta, gamma = _affine_case(rng, shapes, B, M, D, K, Lq)
    W = ss[:, 1].astype(np.float64)[None, None, None, :, None]
    H = ss[:, 0].astype(np.float64)[None, None, None, :, None]
    X = loc[..., 0] * W - 0.5                              # [B,Lq,M,L,K]
    Y = loc[..., 1] * H - 0.5
    # samples[b,q,m,l,k,d]
    samp = (np.transpose(alpha, (1, 0, 2))[None, None, :, :, None, :] * X[..., None]
            + np.transpose(beta, (1, 0, 2))[None, None, :, :, None, :] * Y[..., None]
            + np.transpose(gamma, (1, 0, 2))[None, None, :, :, None, :])
    expect = (attn[..., None] * samp).sum(axis=(3, 4)).reshape(B, Lq, M * D)
    out = orc.forward(value, ss, start, loc, attn)
    _close(out, expect, 1e-12, 1e-12, "affine field output")

    grad = rng.standard_normal((B, Lq, M * D))
    gO = grad.reshape(B, Lq, M, 1, 1, D)
    _, gl, ga = orc.backward(value, ss, start, loc, attn, grad)
    _close(ga, (gO * samp).sum(-1), 1e-12, 1e-12, "affine field grad_attn")
    ga_x = (gO * np.transpose(alpha, (1, 0, 2))[None, None, :, :, None, :]).sum(-1)
    ga_y = (gO * np.transpose(beta, (1, 0, 2))[None, None, :, :, None, :]).sum(-1)
    _close(gl[..., 0], attn * W * ga_x, 1e-11, 1e-12, "affine field grad_loc x")
    _close(gl[..., 1], attn * H * ga_y, 1e-11, 1e-12, "affine field grad_loc y")


# ----------------------------------------------------------------------------
# P-7: adjoint identity for grad_value;  conservation of weight mass
# ----------------------------------------------------------------------------

def pin_adjoint_identity(orc):
    """For fixed locations and weights the forward is linear in value, and
    grad_value is its transpose applied to grad_output:
    <gO, fwd(V)> = <grad_value(gO), V> for every V.  Checked for several V,
    with locations that also fall partly or fully outside the maps."""
    rng = np.random.default_rng(7)
    shapes = [(5, 7), (3, 4), (2, 2)]
    v, ss, start, loc, attn, grad = _random_case(rng, 2, 3, 5, 3, shapes, 11, -0.4, 1.4)
    gv, _, _ = orc.backward(v, ss, start, loc, attn, grad)
    for _ in range(4):
        probe = rng.standard_normal(v.shape)
        lhs = float((grad * orc.forward(probe, ss, start, loc, attn)).sum())
        rhs = float((gv * probe).sum())
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs)), f"adjoint: {lhs} vs {rhs}"
    # Unit basis vectors: grad_value entry (b,s,m,d) equals <gO, fwd(e_bsmd)>.
    for _ in range(6):
        idx = tuple(int(rng.integers(0, n)) for n in v.shape)
        e = np.zeros_like(v)
        e[idx] = 1.0
        lhs = float((grad * orc.forward(e, ss, start, loc, attn)).sum())
        assert abs(lhs - gv[idx]) <= 1e-13 * max(1.0, abs(lhs)), \
            f"grad_value{idx}: {gv[idx]} vs {lhs}"


def pin_conservation(orc):
    """With value-independent bookkeeping: summing grad_value over all tokens of
    a level gives sum over points of A * (weight mass of its in-map corners) *
    gO.  With every corner inside the map the mass is 1, so the level sums are
    sum_{q,k} A[...,l,k] * gO."""
    rng = np.random.default_rng(8)
    shapes = [(6, 5), (3, 4)]
    ss, start, S = _meta(shapes)
    B, M, D, K, Lq = 2, 2, 3, 4, 9
    value = rng.standard_normal((B, S, M, D))
    loc = np.concatenate([_interior_locations(rng, shapes, (B, Lq, M)) for _ in range(K)], axis=4)
    attn = rng.uniform(size=(B, Lq, M, 2, K))
    grad = rng.standard_normal((B, Lq, M * D))
    gv, _, _ = orc.backward(value, ss, start, loc, attn, grad)
    gO = grad.reshape(B, Lq, M, D)
    for l, (h, w) in enumerate(shapes):
        got = gv[:, start[l]:start[l] + h * w].sum(axis=1)                  # [B,M,D]
        expect = np.einsum("bqmk,bqmd->bmd", attn[:, :, :, l, :], gO)
        _close(got, expect, 1e-12, 1e-12, f"grad_value mass on level {l}")


# ----------------------------------------------------------------------------
# P-8: finite differences of the forward
# ----------------------------------------------------------------------------

def pin_finite_differences(orc):
    """grad_sampling_locations and grad_attention_weights equal central finite
    differences of <gO, forward> (float64, step 1e-6 pixel; points within 1e-4
    pixel of an integer coordinate -- where the bilinear weights have kinks --
    are left out)."""
    rng = np.random.default_rng(9)
    shapes = [(5, 6), (3, 4)]
    B, M, D, K, Lq = 1, 2, 3, 2, 4
    v, ss, start, loc, attn, grad = _random_case(rng, B, M, D, K, shapes, Lq, -0.2, 1.2)
    _, gl, ga = orc.backward(v, ss, start, loc, attn, grad)
    f = lambda lo, at: float((grad * orc.forward(v, ss, start, lo, at)).sum())
    L = len(shapes)
    checked = 0
    for idx in np.ndindex(B, Lq, M, L, K):
        l = idx[3]
        h, w = shapes[l]
        for comp, n in ((0, w), (1, h)):
            px = loc[idx + (comp,)] * n - 0.5
            if abs(px - np.round(px)) < 1e-4:
                continue
            step = 1e-6 / n
            lp, lm = loc.copy(), loc.copy()
            lp[idx + (comp,)] += step
            lm[idx + (comp,)] -= step
            fd = (f(lp, attn) - f(lm, attn)) / (2 * step)
            an = gl[idx + (comp,)]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), \
                f"grad_loc{idx + (comp,)}: analytic {an} vs fd {fd}"
            checked += 1
        ap, am = attn.copy(), attn.copy()
        ap[idx] += 1e-4
        am[idx] -= 1e-4
        fd = (f(loc, ap) - f(loc, am)) / 2e-4
        assert abs(fd - ga[idx]) <= 1e-8 * max(1.0, abs(fd)), \
            f"grad_attn{idx}: analytic {ga[idx]} vs fd {fd}"
    assert checked > 20


# ----------------------------------------------------------------------------
# P-9: the library routine the pages build on (torch grid_sample, float64, CPU)
# ----------------------------------------------------------------------------

def grid_sample_core(v, lo, at, shapes, start):
    """The core on torch float64 CPU tensors (differentiable): value [B,S,M,D],
    locations [B,Lq,M,L,K,2], weights [B,Lq,M,L,K] -> output [B,Lq,M*D], written
    with ``torch.nn.functional.grid_sample(mode='bilinear', padding_mode='zeros',
    align_corners=False)``, one call per level with grid = 2*loc - 1 -- the
    formulation of ms_deform_attn_core_pytorch ("Deformable DETR模型解读")."""
    import torch
    import torch.nn.functional as F

    B, S, M, D = v.shape
    _, Lq, _, L, K, _ = lo.shape
    acc = torch.zeros(B * M, D, Lq, dtype=torch.float64)
    for l, (h, w) in enumerate(np.asarray(shapes).reshape(-1, 2)):
        h, w, s0 = int(h), int(w), int(start[l])
        img = v[:, s0:s0 + h * w].permute(0, 2, 3, 1).reshape(B * M, D, h, w)
        grid = lo[:, :, :, l].permute(0, 2, 1, 3, 4).reshape(B * M, Lq, K, 2) * 2.0 - 1.0
        smp = F.grid_sample(img, grid, mode="bilinear", padding_mode="zeros",
                            align_corners=False)                     # [B*M, D, Lq, K]
        wts = at[:, :, :, l].permute(0, 2, 1, 3).reshape(B * M, 1, Lq, K)
        acc = acc + (smp * wts).sum(-1)
    return acc.reshape(B, M, D, Lq).permute(0, 3, 1, 2).reshape(B, Lq, M * D)


def grid_sample_reference(value, shapes, start, loc, attn, grad=None):
    """Forward (and, with ``grad``, autograd gradients) of :func:`grid_sample_core`
    on float64 CPU tensors.  Test-only cross-check of the oracle."""
    import torch

    v = torch.tensor(value, dtype=torch.float64, requires_grad=grad is not None)
    lo = torch.tensor(loc, dtype=torch.float64, requires_grad=grad is not None)
    at = torch.tensor(attn, dtype=torch.float64, requires_grad=grad is not None)
    B, S, M, D = v.shape
    Lq = lo.shape[1]
    out = grid_sample_core(v, lo, at, shapes, start)
    if grad is None:
        return out.detach().numpy()
    out.backward(torch.tensor(grad, dtype=torch.float64).reshape(B, Lq, M * D))
    return (out.detach().numpy(), v.grad.numpy(), lo.grad.numpy(), at.grad.numpy())


def pin_grid_sample(orc):
    """Forward and all three gradients agree with torch grid_sample + autograd in
    float64 (to 1e-12) on random multi-level, multi-head, non-square inputs whose
    locations spill outside the maps on every side."""
    rng = np.random.default_rng(10)
    shapes = [(6, 9), (3, 5), (2, 3)]
    v, ss, start, loc, attn, grad = _random_case(rng, 2, 3, 5, 3, shapes, 13, -0.3, 1.3)
    ref_out, ref_gv, ref_gl, ref_ga = grid_sample_reference(v, ss, start, loc, attn, grad)
    out = orc.forward(v, ss, start, loc, attn)
    gv, gl, ga = orc.backward(v, ss, start, loc, attn, grad)
    _close(out, ref_out, 1e-12, 1e-12, "forward vs grid_sample")
    _close(gv, ref_gv, 1e-12, 1e-12, "grad_value vs grid_sample autograd")
    _close(gl, ref_gl, 1e-11, 1e-11, "grad_loc vs grid_sample autograd")
    _close(ga, ref_ga, 1e-12, 1e-12, "grad_attn vs grid_sample autograd")

    # Non-finite locations: grid_sample turns the sample into NaN and gives
    # grad_value nothing from it; the oracle must agree on where NaN appears.
    loc = loc.copy()
    loc[0, 1, 0, 0, 0, 0] = np.nan
    loc[1, 2, 2, 1, 1, 1] = np.inf
    loc[0, 5, 1, 2, 0, 0] = -np.inf
    ref_out, ref_gv, ref_gl, ref_ga = grid_sample_reference(v, ss, start, loc, attn, grad)
    out = orc.forward(v, ss, start, loc, attn)
    gv, gl, ga = orc.backward(v, ss, start, loc, attn, grad)
    for got, ref, what in ((out, ref_out, "output"), (gv, ref_gv, "grad_value"),
                           (gl, ref_gl, "grad_loc"), (ga, ref_ga, "grad_attn")):
        assert np.array_equal(np.isnan(got), np.isnan(ref)), f"NaN pattern of {what}"
        keep = ~np.isnan(ref)
        _close(got[keep], ref[keep], 1e-11, 1e-11, f"{what} with non-finite locations")
    assert np.isnan(out).any() and not np.isnan(gv).any()


ALL_PINS = [
    pin_pixel_centre,
    pin_offset_init_grid,
    pin_half_pixel_and_padding,
    pin_fully_outside,
    pin_constant_field,
    pin_linearity,
    pin_affine_field,
    pin_adjoint_identity,
    pin_conservation,
    pin_finite_differences,
    pin_grid_sample,
]

# The pins that do not lean on a library routine: a planted mistake must fail
# at least one of these too, so the oracle is pinned without grid_sample.
FIRST_PRINCIPLES_PINS = [p for p in ALL_PINS if p is not pin_grid_sample]
