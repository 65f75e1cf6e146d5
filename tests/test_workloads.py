"""The seeded input generators (CPU only): geometry against the pages' printed
numbers, and the properties each recipe promises."""
import os

import numpy as np
import pytest

from scale_deformable_attention_backward_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    path = os.path.join(GOLDEN, name)
    return [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]


def test_level_token_counts_match_pages():
    rows = _rows("level_token_counts.txt")
    shapes = [(int(r[1]), int(r[2])) for r in rows]
    assert shapes == W.ENCODER_608x848
    ss, start = W.level_metadata(shapes)
    sizes = ss[:, 0] * ss[:, 1]
    assert sizes.tolist() == [int(r[3]) for r in rows]
    assert start.tolist() == [0, 8056, 8056 + 2014, 8056 + 2014 + 513]
    assert W.CONFIGS["encoder_bf16"].S == 10687


def test_encoder_geometry():
    cfg = W.CONFIGS["encoder_fp32"]
    assert cfg.S == 19947 and cfg.queries == 19947 and cfg.L == 4
    # strides 8/16/32/64 of an 800x1200 image (rounded up)
    for (h, w), stride in zip(cfg.shapes, (8, 16, 32, 64)):
        assert h == -(-800 // stride) and w == -(-1200 // stride)


@pytest.mark.parametrize("name", ["tiny_fp32", "decoder_fp32"])
def test_shapes_and_softmax(name):
    cfg = W.CONFIGS[name]
    inp = W.make_inputs(cfg, seed=0)
    d = inp.dims
    assert inp.value.shape == (cfg.B, cfg.S, cfg.M, cfg.D)
    assert inp.sampling_locations.shape == (cfg.B, cfg.queries, cfg.M, cfg.L, cfg.K, 2)
    assert inp.sampling_locations.dtype == np.float32
    assert inp.attention_weights.dtype == np.float32
    s = inp.attention_weights.astype(np.float64).sum(axis=(3, 4))
    assert np.allclose(s, 1.0, atol=1e-6)
    assert d["Lq"] == cfg.queries
    assert (inp.grad_output is not None) == cfg.backward


def test_seed_is_deterministic():
    cfg = W.CONFIGS["tiny_fp32"]
    a, b = W.make_inputs(cfg, seed=0), W.make_inputs(cfg, seed=0)
    c = W.make_inputs(cfg, seed=1)
    assert np.array_equal(a.sampling_locations, b.sampling_locations)
    assert np.array_equal(a.value, b.value)
    assert not np.array_equal(a.value, c.value)


def test_encoder_reference_is_pixel_centre():
    cfg = W.CONFIGS["encoder_fp32"].with_batch(1)
    inp = W.make_inputs(cfg, seed=0)
    loc = inp.sampling_locations.astype(np.float64)
    # mean over heads, points of the offset (N(0, 2 px)) is ~0: the mean location
    # of a token is its own pixel centre on every level.
    mean = loc.mean(axis=(2, 4))                                      # [1, Lq, L, 2]
    ss, start = W.level_metadata(cfg.shapes)
    h0, w0 = cfg.shapes[0]
    q = np.arange(h0 * w0)
    cx, cy = (q % w0 + 0.5) / w0, (q // w0 + 0.5) / h0
    for l, (h, w) in enumerate(cfg.shapes):
        err_x = mean[0, q, l, 0] - cx
        # std of the mean of 32 offsets of 2/W_l each
        assert np.abs(err_x).mean() < 3 * 2.0 / w / np.sqrt(32)
        assert np.abs(mean[0, q, l, 1] - cy).mean() < 3 * 2.0 / h / np.sqrt(32)


def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * 10.0).astype(np.float32)
    bits = W.bf16_round_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)


def test_valid_ratio_recipe():
    cfg = W.CONFIGS["encoder_bf16"].with_batch(2)
    inp = W.make_inputs(cfg, seed=0)
    assert inp.value_bf16_bits is not None
    assert np.array_equal(W.bf16_bits_to_f32(inp.value_bf16_bits), inp.value)
    # Reference points of a token are its pixel centre over its own level's valid
    # extent, times each target level's valid ratio: the mean location (over heads
    # and points, which averages the offsets away) of a level-0 token on level l
    # is its level-0 location times vr_l / vr_0 -- one ratio per image and level.
    loc = inp.sampling_locations.astype(np.float64)
    h0, w0 = cfg.shapes[0]
    q = np.arange(h0 * w0)
    q = q[(q % w0) > w0 // 2]                                  # right half: large x
    mean = loc[:, q].mean(axis=(2, 4))                         # [B, nq, L, 2]
    ratios = mean[:, :, :, 0] / mean[:, :, :1, 0]              # [B, nq, L]
    spread = ratios.std(axis=1)
    assert np.all(spread < 0.08)          # offsets of 2 px average out to ~2/sqrt(32) px
    assert np.abs(ratios.mean(axis=1)[:, 1:] - 1.0).max() > 1e-3


def test_select_queries():
    cfg = W.CONFIGS["tiny_fp32"]
    inp = W.make_inputs(cfg, seed=0)
    sub = W.select_queries(inp, np.array([3, 1, 7]))
    assert sub.sampling_locations.shape[1] == 3
    assert np.array_equal(sub.sampling_locations[:, 1], inp.sampling_locations[:, 1])
    assert np.array_equal(sub.grad_output[:, 2], inp.grad_output[:, 7])


@pytest.mark.parametrize("name", ["tiny_fp32", "encoder_fp32", "decoder_fp32",
                                  "decoder_box_train_fp32"])
def test_fused_inputs_reproduce_locations_and_weights(name):
    """The raw inputs of the fused op, pushed through the pages' formulas in
    float64, give the locations and weights make_inputs draws (up to their
    float32 storage)."""
    cfg = W.CONFIGS[name]
    f = W.make_fused_inputs(cfg, seed=0)
    c = W.make_inputs(cfg, seed=0)
    assert np.array_equal(f.value, c.value)
    if cfg.recipe == "uniform":
        return  # the uniform recipe draws locations directly
    ref = f.reference_points.astype(np.float64)[:, :, None, :, None, :]
    off = f.sampling_offsets.astype(np.float64)
    if ref.shape[-1] == 2:
        wh = f.spatial_shapes[:, ::-1].astype(np.float64)[None, None, None, :, None, :]
        loc = ref + off / wh
    else:
        loc = ref[..., :2] + off / cfg.K * ref[..., 2:] * 0.5
    assert np.abs(loc - c.sampling_locations).max() < 1e-6
    z = f.attention_logits.astype(np.float64)
    e = np.exp(z - z.max(-1, keepdims=True))
    A = (e / e.sum(-1, keepdims=True)).reshape(c.attention_weights.shape)
    assert np.abs(A - c.attention_weights).max() < 1e-6
