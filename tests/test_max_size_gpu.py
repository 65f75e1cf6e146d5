"""The largest value block the C ABI accepts, checked against closed forms.

One image's value block is addressed with 32-bit element offsets, so the ABI
takes S*M*D < 2^31.  Here M = 1, D = 4 and four levels of 2^13, 2^12, 2^11 and
2^10 rows by 2^15 columns give S = 2^29 - 2^25 pixels: S*M*D = 2^31 - 2^27, and
with B = 2 the second image starts past element 2^31 (64-bit image base).  The
value tensor is 16 GiB, grad_value another 16 GiB, the deterministic backward's
workspace 32 GiB; the float64 oracle cannot hold that, so the check uses
properties that hold at any size:

* value is an affine field of the pixel coordinates on every level: channel 0
  is x, channel 1 is y, channel 2 is x + 512 y, channel 3 the constant
  3 + l + 10 b, all integers below 2^24 and so exact in float32;
* bilinear interpolation reproduces an affine field exactly inside the map
  ("Deformable DETR模型解读（附源码+论文）", ms_deform_attn_core_pytorch: the
  sample is the bilinear blend of the four corners), so a point at pixel
  coordinate (x, y) samples (x, y, x + 512 y, c);
* every location is (x + 0.5) / W with x a multiple of 1/16 and W a power of
  two, so loc * W - 0.5 is exact in float32 and the kernels see the same x as
  the float64 closed form; all four corners lie inside the map.

Then, per point with weight A and per-query gO:
  output  = sum over points of A * sample;
  grad_attention_weights = gO . sample;
  grad_sampling_locations = (A W gO . (1, 0, 1, 0), A H gO . (0, 1, 512, 0));
  grad_value at each corner pixel = sum of A * bilinear weight * gO over the
  points that touch it, and zero everywhere else (checked through the sum of
  |grad_value| over the whole tensor).
Level 3's points sit in its last rows, so their corner offsets reach
S*M*D - 4, the largest element offset an image can have."""
import numpy as np
import pytest
import torch

import gpu_support as G
from scale_deformable_attention_backward_b200 import binding

pytestmark = pytest.mark.gpu

SHAPES = [(1 << 13, 1 << 15), (1 << 12, 1 << 15), (1 << 11, 1 << 15), (1 << 10, 1 << 15)]
B, M, D, K, LQ = 2, 1, 4, 4, 256
COEF = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 512.0], [0.0, 0.0]])  # (a_d, b_d) per channel


def constant(l, b):
    return 3.0 + l + 10.0 * b


def build_value(starts):
    S = starts[-1] + SHAPES[-1][0] * SHAPES[-1][1]
    assert S * M * D == (1 << 31) - (1 << 27)
    value = torch.empty((B, S, M, D), dtype=torch.float32, device="cuda")
    for b in range(B):
        for l, (H, W) in enumerate(SHAPES):
            v = value[b, starts[l]:starts[l] + H * W, 0, :].view(H, W, D)
            x = torch.arange(W, dtype=torch.float32, device="cuda")
            y = torch.arange(H, dtype=torch.float32, device="cuda")
            v[..., 0] = x[None, :]
            v[..., 1] = y[:, None]
            v[..., 2] = x[None, :] + 512.0 * y[:, None]
            v[..., 3] = constant(l, b)
    return value


def make_points(rng):
    """Pixel coordinates (x, y) on a 1/16 grid with all four corners inside each
    level, locations (x + 0.5) / (W, H), and weights A."""
    xy = np.empty((B, LQ, M, len(SHAPES), K, 2))
    for l, (H, W) in enumerate(SHAPES):
        ix = rng.integers(0, W - 1, size=(B, LQ, M, K))
        if l == len(SHAPES) - 1:
            iy = rng.integers(H - 3, H - 1, size=(B, LQ, M, K))  # the last rows
        else:
            iy = rng.integers(0, H - 1, size=(B, LQ, M, K))
        xy[:, :, :, l, :, 0] = ix + rng.integers(0, 16, size=ix.shape) / 16.0
        xy[:, :, :, l, :, 1] = iy + rng.integers(0, 16, size=iy.shape) / 16.0
    wh = np.array([[W, H] for H, W in SHAPES], dtype=np.float64)[None, None, None, :, None, :]
    loc = ((xy + 0.5) / wh).astype(np.float32)
    assert np.array_equal(loc.astype(np.float64) * wh - 0.5, xy)  # exact in float32
    attn = rng.uniform(0.05, 1.0, size=(B, LQ, M, len(SHAPES), K)).astype(np.float32)
    return xy, loc, attn


def samples(xy):
    """[B, LQ, M, L, K, D] affine value at each point (the exact bilinear sample)."""
    s = xy[..., 0:1] * COEF[:, 0] + xy[..., 1:2] * COEF[:, 1]
    c = np.array([[constant(l, b) for l in range(len(SHAPES))] for b in range(B)])
    s[..., 3] = c[:, None, None, :, None]
    return s


def corner_contributions(xy, attn, go, starts):
    """(flat pixel index per image, b, weight * gO [.., D]) of every point corner."""
    pix, bs, contrib = [], [], []
    for l, (H, W) in enumerate(SHAPES):
        x, y = xy[:, :, :, l, :, 0], xy[:, :, :, l, :, 1]
        x0, y0 = np.floor(x), np.floor(y)
        fx, fy = x - x0, y - y0
        a = attn[:, :, :, l, :].astype(np.float64)
        for dx, dy, w in ((0, 0, (1 - fx) * (1 - fy)), (1, 0, fx * (1 - fy)),
                          (0, 1, (1 - fx) * fy), (1, 1, fx * fy)):
            p = starts[l] + (y0 + dy) * W + (x0 + dx)
            pix.append(p.astype(np.int64).ravel())
            bs.append(np.broadcast_to(np.arange(B)[:, None, None, None], p.shape).ravel())
            g = (a * w)[..., None] * go[:, :, None, None, :]      # [B, LQ, M, K, D]
            contrib.append(g.reshape(-1, D))
    return np.concatenate(pix), np.concatenate(bs), np.concatenate(contrib)


def test_largest_value_block_against_closed_forms():
    free, _ = torch.cuda.mem_get_info()
    if free < (80 << 30):
        pytest.skip("needs 80 GiB of free device memory")
    rng = np.random.default_rng(11)
    starts = np.concatenate([[0], np.cumsum([h * w for h, w in SHAPES])[:-1]]).astype(np.int64)
    value = build_value(starts)
    S = value.shape[1]
    shapes_t = torch.tensor(SHAPES, dtype=torch.int64, device="cuda")
    starts_t = torch.from_numpy(starts).cuda()
    xy, loc, attn = make_points(rng)
    go = rng.standard_normal((B, LQ, M * D)).astype(np.float32)
    loc_t, attn_t = torch.from_numpy(loc).cuda(), torch.from_numpy(attn).cuda()
    go_t = torch.from_numpy(go).cuda()
    sm = samples(xy)
    go64 = go.astype(np.float64)

    # Forward.
    out = binding.forward(value, shapes_t, starts_t, loc_t, attn_t)
    want = (attn.astype(np.float64)[..., None] * sm).sum(axis=(3, 4)).reshape(B, LQ, M * D)
    G.assert_forward_f32(out.double().cpu().numpy(), want, "forward at the largest block")

    # Backward closed forms.
    want_ga = (sm * go64[:, :, None, None, None, :]).sum(-1)
    a64 = attn.astype(np.float64)
    Ws = np.array([w for _, w in SHAPES], dtype=np.float64)[None, None, None, :, None]
    Hs = np.array([h for h, _ in SHAPES], dtype=np.float64)[None, None, None, :, None]
    gx = (go64 @ COEF[:, 0])[:, :, None, None, None] * a64 * Ws
    gy = (go64 @ COEF[:, 1])[:, :, None, None, None] * a64 * Hs
    want_gl = np.stack([gx, gy], axis=-1)
    pix, bs, contrib = corner_contributions(xy, attn, go64, starts)
    keys, inv = np.unique(bs * S + pix, return_inverse=True)
    want_gv = np.zeros((keys.size, D))
    np.add.at(want_gv, inv, contrib)
    kb = torch.from_numpy(keys // S).cuda()
    kp = torch.from_numpy(keys % S).cuda()
    assert (keys % S).max() * M * D >= (1 << 31) - (1 << 27) - (1 << 17)  # near the largest offset

    for deterministic in (False, True):
        tag = "deterministic" if deterministic else "direct"
        gv, gl, ga = binding.backward(value, shapes_t, starts_t, loc_t, attn_t, go_t,
                                      deterministic=deterministic)
        torch.cuda.synchronize()
        G.assert_backward_f32(ga.double().cpu().numpy(), want_ga, f"grad_attention_weights ({tag})")
        G.assert_backward_f32(gl.double().cpu().numpy(), want_gl, f"grad_sampling_locations ({tag})")
        got_gv = gv[kb, kp, 0, :].double().cpu().numpy()
        G.assert_backward_f32(got_gv, want_gv, f"grad_value at the touched pixels ({tag})")
        # Nothing written anywhere else: |grad_value| sums to the touched pixels' total.
        total = float(gv.abs().sum(dtype=torch.float64))
        touched = float(np.abs(got_gv).sum())
        assert abs(total - touched) <= 1e-9 * touched, (tag, total, touched)
        del gv, gl, ga
        torch.cuda.empty_cache()
    del value, out
    torch.cuda.empty_cache()                 # hand the 16 GiB back to the tests that follow
