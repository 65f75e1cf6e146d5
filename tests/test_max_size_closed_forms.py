"""The closed forms that test_max_size_gpu.py checks the kernels against, checked
here against the float64 oracle on a small geometry of the same construction
(affine value field, locations on a 1/16 pixel grid, every corner inside the
map, the last level's points in its last rows)."""
import numpy as np

import gpu_support as G
import oracle
import test_max_size_gpu as T

SMALL = [(1 << 4, 1 << 5), (1 << 3, 1 << 5), (1 << 3, 1 << 4), (1 << 2, 1 << 5)]


def test_closed_forms_match_the_oracle(monkeypatch):
    monkeypatch.setattr(T, "SHAPES", SMALL)
    monkeypatch.setattr(T, "LQ", 7)
    rng = np.random.default_rng(11)
    starts = np.concatenate([[0], np.cumsum([h * w for h, w in SMALL])[:-1]]).astype(np.int64)
    S = int(starts[-1] + SMALL[-1][0] * SMALL[-1][1])
    B, M, D = T.B, T.M, T.D
    value = np.zeros((B, S, M, D), np.float32)
    for b in range(B):
        for l, (H, W) in enumerate(SMALL):
            v = value[b, starts[l]:starts[l] + H * W, 0, :].reshape(H, W, D)
            x = np.arange(W, dtype=np.float32)
            y = np.arange(H, dtype=np.float32)
            v[..., 0] = x[None, :]
            v[..., 1] = y[:, None]
            v[..., 2] = x[None, :] + 512.0 * y[:, None]
            v[..., 3] = T.constant(l, b)
    xy, loc, attn = T.make_points(rng)
    go = rng.standard_normal((B, T.LQ, M * D)).astype(np.float32)
    shapes = np.array(SMALL, np.int64)
    sm = T.samples(xy)
    a64, go64 = attn.astype(np.float64), go.astype(np.float64)

    out = oracle.forward(value, shapes, starts, loc, attn)
    want = (a64[..., None] * sm).sum(axis=(3, 4)).reshape(B, T.LQ, M * D)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-9)

    gv, gl, ga = oracle.backward(value, shapes, starts, loc, attn, go)
    np.testing.assert_allclose(ga, (sm * go64[:, :, None, None, None, :]).sum(-1),
                               rtol=1e-12, atol=1e-9)
    Ws = np.array([w for _, w in SMALL], dtype=np.float64)[None, None, None, :, None]
    Hs = np.array([h for h, _ in SMALL], dtype=np.float64)[None, None, None, :, None]
    want_gl = np.stack([(go64 @ T.COEF[:, 0])[:, :, None, None, None] * a64 * Ws,
                        (go64 @ T.COEF[:, 1])[:, :, None, None, None] * a64 * Hs], axis=-1)
    np.testing.assert_allclose(gl, want_gl, rtol=1e-9, atol=1e-9)
    pix, bs, contrib = T.corner_contributions(xy, attn, go64, starts)
    keys, inv = np.unique(bs * S + pix, return_inverse=True)
    want_gv = np.zeros((keys.size, D))
    np.add.at(want_gv, inv, contrib)
    got = gv[keys // S, keys % S, 0, :]
    np.testing.assert_allclose(got, want_gv, rtol=1e-12, atol=1e-12)
    assert np.abs(gv).sum() == np.abs(got).sum()       # nothing outside the touched pixels
    assert (keys % S).max() == S - 1                     # the last pixel is reached
    G.assert_forward_f32(out, want)                      # the GPU test's own tolerance holds
