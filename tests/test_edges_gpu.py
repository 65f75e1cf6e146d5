"""GPU parity on shapes and inputs chosen to break things: every lane width and
channel chunking, ragged query counts, levels of height or width 1, locations
far outside the maps or within one float32 ulp of a pixel boundary, non-finite
locations, empty calls, inconsistent metadata, misaligned pointers, and guard
bands around every output."""
import dataclasses

import numpy as np
import pytest
import torch

import gpu_support as G
from scale_deformable_attention_backward_b200 import binding
from scale_deformable_attention_backward_b200 import workloads as W

pytestmark = pytest.mark.gpu


def random_inputs(seed, B, M, D, K, shapes, Lq, lo=-0.3, hi=1.3, dtype="f32", grad=True):
    rng = np.random.default_rng(seed)
    ss, start = W.level_metadata(shapes)
    S = int((ss[:, 0] * ss[:, 1]).sum())
    L = len(shapes)
    value = rng.standard_normal((B, S, M, D)).astype(np.float32)
    bits = None
    if dtype == "bf16":
        bits = W.bf16_round_bits(value)
        value = W.bf16_bits_to_f32(bits)
    loc = rng.uniform(lo, hi, size=(B, Lq, M, L, K, 2)).astype(np.float32)
    attn = rng.uniform(0, 1, size=(B, Lq, M, L, K))
    attn = (attn / attn.sum(axis=(3, 4), keepdims=True)).astype(np.float32)
    go = rng.standard_normal((B, Lq, M * D)).astype(np.float32) if grad else None
    go_bits = None
    if go is not None and dtype == "bf16":
        go_bits = W.bf16_round_bits(go)
        go = W.bf16_bits_to_f32(go_bits)
    cfg = W.Config("random", B, M, D, K, tuple(shapes), "uniform", dtype, grad, Lq)
    return W.Inputs(cfg, np.ascontiguousarray(value), bits, ss, start, loc, attn, go, go_bits)


SHAPES = [[(5, 7)], [(1, 9), (6, 1), (3, 4)], [(16, 3), (8, 2), (4, 1), (2, 1)],
          [(11, 13), (1, 1)]]


@pytest.mark.parametrize("D", [4, 8, 12, 16, 20, 32, 64, 128])
@pytest.mark.parametrize("shapes_id", range(len(SHAPES)))
def test_random_shapes_f32(D, shapes_id):
    shapes = SHAPES[shapes_id]
    inp = random_inputs(100 + D + shapes_id, B=2, M=3, D=D, K=3, shapes=shapes, Lq=37)
    d = G.device_inputs(inp)
    G.assert_forward_f32(G.gpu_forward(d), G.oracle_forward(inp), f"forward D={D}")
    G.check_backward_paths(d, inp)


@pytest.mark.parametrize("offset", [100.0, -1000.0])
def test_value_with_large_common_offset(offset):
    """value = offset + N(0, 1): the backward forms grad_loc from differences of
    corner dot products (G10 - G00 ...), whose common part cancels.  The result
    must still meet the float32 backward tolerance against the oracle, on every
    backward path."""
    inp = random_inputs(31, B=2, M=4, D=32, K=4, shapes=SHAPES[2], Lq=45)
    inp = dataclasses.replace(inp, value=np.ascontiguousarray(inp.value + np.float32(offset)))
    d = G.device_inputs(inp)
    G.assert_forward_f32(G.gpu_forward(d), G.oracle_forward(inp), f"forward offset={offset}")
    G.check_backward_paths(d, inp)


@pytest.mark.parametrize("D", [132, 192, 256])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_channel_passes(D, dtype):
    """Heads wider than 128 channels: the scratch-free backward runs two channel
    passes (the second adds its share of grad_loc and grad_attn); against the
    oracle (bfloat16 too: its backward lanes move 4 channels, so D % 4 == 0
    suffices).  The cell-sorted path (a workspace) refuses them."""
    inp = random_inputs(400 + D, B=2, M=2, D=D, K=4, shapes=SHAPES[2], Lq=41, dtype=dtype)
    d = G.device_inputs(inp)
    rv, rl, ra = G.oracle_backward(inp)
    gv, gl, ga = G.gpu_backward(d, "direct")
    G.assert_backward_f32(gv, rv, f"{dtype} D={D} grad_value")
    G.assert_backward_f32(gl, rl, f"{dtype} D={D} grad_sampling_locations")
    G.assert_backward_f32(ga, ra, f"{dtype} D={D} grad_attention_weights")
    if dtype == "f32":
        with pytest.raises(RuntimeError, match="UNSUPPORTED|unsupported"):
            G.gpu_backward(d, "sorted")


@pytest.mark.parametrize("D", [256, 384])
def test_forward_channel_chunks_f32(D):
    """More than 32 lanes' worth of channels: several chunks per head."""
    inp = random_inputs(7 + D, B=1, M=2, D=D, K=2, shapes=SHAPES[1], Lq=19, grad=False)
    G.assert_forward_f32(G.gpu_forward(G.device_inputs(inp)), G.oracle_forward(inp))


@pytest.mark.parametrize("D", [8, 16, 24, 32, 64, 256, 512])
def test_random_shapes_bf16(D):
    inp = random_inputs(200 + D, B=2, M=2, D=D, K=4, shapes=SHAPES[2], Lq=29, dtype="bf16",
                        grad=False)
    G.assert_forward_bf16(G.gpu_forward(G.device_inputs(inp)), G.oracle_forward(inp))


@pytest.mark.parametrize("D", [4, 8, 12, 20, 32, 64, 128])
@pytest.mark.parametrize("shapes_id", [1, 2])
def test_random_shapes_bf16_backward(D, shapes_id):
    """bfloat16 value and grad_output through the scratch-free backward (float32
    arithmetic and gradients): the oracle sees the same bfloat16 values widened,
    so the float32 backward tolerances apply."""
    inp = random_inputs(400 + D + shapes_id, B=2, M=3, D=D, K=3, shapes=SHAPES[shapes_id],
                        Lq=41, dtype="bf16")
    G.check_backward_paths(G.device_inputs(inp), inp, f"bf16 D={D}")


def test_bf16_autograd():
    """ms_deform_attn with a bfloat16 value: autograd gets grad_value in bfloat16
    (rounded from the float32 result) and the location / weight gradients."""
    inp = random_inputs(77, B=1, M=2, D=16, K=2, shapes=SHAPES[1], Lq=17, dtype="bf16")
    d = G.device_inputs(inp)
    v = d["value"].clone().requires_grad_(True)
    loc = d["sampling_locations"].clone().requires_grad_(True)
    att = d["attention_weights"].clone().requires_grad_(True)
    out = binding.ms_deform_attn(v, d["spatial_shapes"], d["level_start_index"], loc, att)
    out.backward(d["grad_output"])
    torch.cuda.synchronize()
    rv, rl, ra = G.oracle_backward(inp)
    assert v.grad.dtype == torch.bfloat16
    G.assert_forward_bf16(v.grad.float().cpu().numpy().astype(np.float64), rv, "bf16 grad_value")
    G.assert_backward_f32(loc.grad.cpu().numpy().astype(np.float64), rl, "bf16 grad_loc")
    G.assert_backward_f32(att.grad.cpu().numpy().astype(np.float64), ra, "bf16 grad_attn")


@pytest.mark.parametrize("L,K", [(1, 1), (3, 5), (16, 1), (1, 64), (16, 4)])
def test_level_and_point_counts(L, K):
    rng = np.random.default_rng(L * 100 + K)
    shapes = [(int(rng.integers(1, 9)), int(rng.integers(1, 9))) for _ in range(L)]
    inp = random_inputs(300 + L + K, B=1, M=2, D=8, K=K, shapes=shapes, Lq=13)
    d = G.device_inputs(inp)
    G.assert_forward_f32(G.gpu_forward(d), G.oracle_forward(inp))
    G.check_backward_paths(d, inp)


def test_locations_at_pixel_boundaries():
    """Pixel coordinates x = loc*W - 0.5 within a few float32 ulps of an integer,
    on maps whose widths are not powers of two.  The cell (floor) must match the
    oracle's exact one, or grad_sampling_locations jumps by a whole corner
    difference."""
    shapes = [(100, 150), (25, 38), (13, 19)]
    ss, start = W.level_metadata(shapes)
    rng = np.random.default_rng(5)
    B, M, D, K, Lq = 1, 2, 8, 4, 256
    L = len(shapes)
    loc = np.empty((B, Lq, M, L, K, 2), dtype=np.float32)
    for l, (h, w) in enumerate(shapes):
        for comp, n in ((0, w), (1, h)):
            pix = rng.integers(0, n, size=(B, Lq, M, K))
            base = ((pix + 0.5) / n).astype(np.float32)
            steps = rng.integers(-3, 4, size=base.shape)
            out = base.copy()
            for s in range(1, 4):
                out = np.where(steps >= s, np.nextafter(out, np.float32(2)), out)
                out = np.where(steps <= -s, np.nextafter(out, np.float32(-1)), out)
            loc[:, :, :, l, :, comp] = out
    inp = random_inputs(6, B, M, D, K, shapes, Lq)
    inp = dataclasses.replace(inp, sampling_locations=loc)
    d = G.device_inputs(inp)
    G.assert_forward_f32(G.gpu_forward(d), G.oracle_forward(inp))
    G.check_backward_paths(d, inp, "at pixel boundaries")


@pytest.mark.parametrize("special", ["finite", "nonfinite"])
def test_points_sharing_corners(special):
    """The four points of one level of one (b, q, m) placed in the same,
    side-by-side and diagonal cells, also across the map's edges, so that their
    corners coincide: the float backward merges such corners' grad_value
    contributions (K = 4) before the scatter.  Every backward path against the
    oracle; in the second case with NaN and Inf weights and an Inf grad_output
    on groups whose corners are shared."""
    shapes = [(6, 7), (3, 5), (1, 4), (2, 1)]
    rng = np.random.default_rng(41)
    B, M, D, K, Lq = 2, 3, 16, 4, 57
    L = len(shapes)
    loc = np.empty((B, Lq, M, L, K, 2), dtype=np.float32)
    for l, (h, w) in enumerate(shapes):
        cx = rng.integers(-1, w, size=(B, Lq, M))
        cy = rng.integers(-1, h, size=(B, Lq, M))
        for k in range(K):
            same = rng.random((B, Lq, M)) < 0.3
            dx = np.where(same, 0, rng.integers(-1, 2, size=(B, Lq, M)))
            dy = np.where(same, 0, rng.integers(-1, 2, size=(B, Lq, M)))
            # pixel coordinate loc * n - 0.5 inside cell c + d
            loc[:, :, :, l, k, 0] = (cx + dx + rng.random((B, Lq, M)) + 0.5) / w
            loc[:, :, :, l, k, 1] = (cy + dy + rng.random((B, Lq, M)) + 0.5) / h
    inp = random_inputs(42, B, M, D, K, shapes, Lq)
    attn = inp.attention_weights.copy()
    go = inp.grad_output.copy()
    if special == "nonfinite":
        attn[0, 3, 1, 0, 2] = np.nan
        attn[1, 5, 0, 1, 1] = np.inf
        attn[1, 6, 2, 0, 0] = -np.inf
        go[0, 7, 1 * D + 3] = np.inf
        # Two points of that group on exact pixel centres of the 1 x 4 level: the
        # corner they share has weight 0 in one of them, and 0 * Inf is NaN.
        loc[0, 7, 1, 2, 0] = (1.5 / 4, 0.5)
        loc[0, 7, 1, 2, 1] = (2.5 / 4, 0.5)
    inp = dataclasses.replace(inp, sampling_locations=loc, attention_weights=attn,
                              grad_output=go)
    d = G.device_inputs(inp)
    got, ref = G.gpu_forward(d), G.oracle_forward(inp)
    if special == "nonfinite":
        # An infinite weight: the pages scale the interpolated value, A * sum_c b_c V_c
        # (+-Inf); the kernels fold A into the corner weights, sum_c (A b_c) V_c, which
        # is NaN when the corner values differ in sign.  Elsewhere the outputs agree.
        inf = np.isinf(ref)
        assert np.all(np.isinf(got[inf]) | np.isnan(got[inf]))
        got, ref = np.where(inf, 0.0, got), np.where(inf, 0.0, ref)
    G.assert_forward_f32(got, ref)
    if special == "finite":
        G.check_backward_paths(d, inp, "shared corners")
        return
    # grad_value is a sum of products A w gO, so its NaN / +-Inf pattern does not
    # depend on the order of the sums.  grad_attn and grad_loc sum over the
    # channels first and combine the corner sums after (P + fx Ex + ...), where an
    # Inf channel can meet Inf - Inf; the oracle combines per channel.  There NaN
    # may stand for the oracle's +-Inf.
    rv, rl, ra = G.oracle_backward(inp)
    for path in G.backward_paths(d):
        gv, gl, ga = G.gpu_backward(d, path)
        for got_t, ref_t, name, relaxed in ((gv, rv, "grad_value", False),
                                            (gl, rl, "grad_sampling_locations", True),
                                            (ga, ra, "grad_attention_weights", True)):
            inf = np.isinf(ref_t)
            what = f"{name} shared corners, non-finite ({path})"
            same = got_t[inf] == ref_t[inf]
            assert np.all(same | np.isnan(got_t[inf]) if relaxed else same), what
            G.assert_backward_f32(got_t[~inf], ref_t[~inf], what)


def test_far_and_nonfinite_locations():
    inp = random_inputs(8, B=2, M=2, D=8, K=3, shapes=SHAPES[1], Lq=11)
    loc = inp.sampling_locations.copy()
    loc[0, 0, 0, 0, 0] = (1e30, 0.5)
    loc[0, 1, 1, 1, 2] = (-1e30, -1e30)
    loc[1, 2, 0, 2, 1] = (3.0e38, 0.2)
    loc[1, 3, 1, 0, 0] = (-7.5, 42.0)
    loc[0, 4, 0, 0, 1] = (np.nan, 0.5)
    loc[1, 5, 1, 2, 2] = (0.5, np.inf)
    loc[0, 6, 0, 1, 0] = (-np.inf, -np.inf)
    inp = dataclasses.replace(inp, sampling_locations=loc)
    d = G.device_inputs(inp)
    G.assert_forward_f32(G.gpu_forward(d), G.oracle_forward(inp))
    G.check_backward_paths(d, inp)



def test_nonfinite_value_pixels():
    """NaN and +-Inf in value, on the first pixel of every level (the pixel a
    point with no corner in the map would stand nearest to) and inside the maps,
    with locations spread over [-0.3, 1.3] so that many points sit partly or
    wholly outside.  Zero padding means a corner outside the map adds nothing,
    so the non-finite pixels reach exactly the outputs whose points touch them:
    the forward matches the oracle element by element, NaN and Inf pattern
    included.  grad_value does not depend on value and matches exactly as in
    the finite case.  grad_attn and grad_loc combine corner differences
    (P + fx Ex + ..., Ex = gO . (V10 - V00)), so an infinite corner may give
    NaN where the oracle's direct sum gives +-Inf; everywhere else they agree."""
    shapes = [(6, 7), (3, 5), (2, 3)]
    inp = random_inputs(77, B=2, M=2, D=8, K=3, shapes=shapes, Lq=61)
    value = inp.value.copy()
    starts = inp.level_start_index
    value[0, starts[0]] = np.nan
    value[0, starts[1], 0] = np.inf
    value[0, starts[2], 1, :4] = -np.inf
    value[1, starts[0] + 17, 1, 2:5] = np.inf
    value[1, starts[0] + 18, 1, 3] = -np.inf
    value[1, starts[1] + 6, 0, :] = np.nan
    inp = dataclasses.replace(inp, value=value)
    d = G.device_inputs(inp)
    ref = G.oracle_forward(inp)
    assert 0 < (~np.isfinite(ref)).mean() < 0.5      # the pixels are reached, not everywhere
    got = G.gpu_forward(d)
    inf = np.isinf(ref)
    assert np.array_equal(got[inf], ref[inf])
    G.assert_forward_f32(np.where(inf, 0.0, got), np.where(inf, 0.0, ref))  # NaN pattern, finite values
    rv, rl, ra = G.oracle_backward(inp)
    assert np.all(np.isfinite(rv))
    for path in G.backward_paths(d):
        gv, gl, ga = G.gpu_backward(d, path)
        G.assert_backward_f32(gv, rv, f"grad_value, non-finite value ({path})")
        for got_t, ref_t, name in ((gl, rl, "grad_sampling_locations"),
                                   (ga, ra, "grad_attention_weights")):
            inf = np.isinf(ref_t)
            what = f"{name}, non-finite value ({path})"
            assert np.all((got_t[inf] == ref_t[inf]) | np.isnan(got_t[inf])), what
            G.assert_backward_f32(got_t[~inf], ref_t[~inf], what)

def test_empty_calls():
    inp = random_inputs(9, B=2, M=2, D=8, K=2, shapes=SHAPES[0], Lq=0)
    d = G.device_inputs(inp)
    out = binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                          d["sampling_locations"], d["attention_weights"])
    assert out.shape == (2, 0, 16)
    gv = torch.full(d["value"].shape, 7.0, device="cuda")
    binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                     d["sampling_locations"], d["attention_weights"], d["grad_output"],
                     grad_value=gv)
    torch.cuda.synchronize()
    assert torch.count_nonzero(gv).item() == 0, "grad_value must be zeroed even with Lq = 0"
    inp0 = random_inputs(9, B=0, M=2, D=8, K=2, shapes=SHAPES[0], Lq=5)
    d0 = G.device_inputs(inp0)
    out = binding.forward(d0["value"], d0["spatial_shapes"], d0["level_start_index"],
                          d0["sampling_locations"], d0["attention_weights"])
    assert out.shape == (0, 5, 16)


def _guarded(shape, fill, dtype=torch.float32, pad=64):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * pad,), fill, dtype=dtype, device="cuda")
    return buf, buf[pad:pad + n].view(shape)


def test_guard_bands_untouched():
    inp = random_inputs(10, B=2, M=3, D=12, K=3, shapes=SHAPES[1], Lq=21)
    d = G.device_inputs(inp)
    B, S, M, D = inp.value.shape
    _, Lq, _, L, K, _ = inp.sampling_locations.shape
    sentinel = 12345.0
    ob, out = _guarded((B, Lq, M * D), sentinel)
    binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                    d["sampling_locations"], d["attention_weights"], output=out)
    torch.cuda.synchronize()
    assert torch.all(ob[:64] == sentinel) and torch.all(ob[-64:] == sentinel)
    G.assert_forward_f32(out.double().cpu().numpy(), G.oracle_forward(inp))
    rv, rl, ra = G.oracle_backward(inp)
    need = binding.workspace_size(B, S, M, D, Lq, L, K)
    for path in G.BACKWARD_PATHS:
        vb, gv = _guarded((B, S, M, D), sentinel)
        lb, gl = _guarded((B, Lq, M, L, K, 2), sentinel)
        ab, ga = _guarded((B, Lq, M, L, K), sentinel)
        # The workspace sits between two guard bands of its own (256-byte aligned).
        wb = torch.full((need + 2 * 512,), 0x5A, dtype=torch.uint8, device="cuda")
        ws = wb[512:512 + need] if path == "sorted" else None
        binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                         d["sampling_locations"], d["attention_weights"], d["grad_output"],
                         grad_value=gv, grad_sampling_locations=gl, grad_attention_weights=ga,
                         workspace=ws)
        torch.cuda.synchronize()
        for buf in (vb, lb, ab):
            assert torch.all(buf[:64] == sentinel) and torch.all(buf[-64:] == sentinel), path
        assert torch.all(wb[:512] == 0x5A) and torch.all(wb[-512:] == 0x5A), path
        G.assert_backward_f32(gv.double().cpu().numpy(), rv, f"grad_value ({path})")
        G.assert_backward_f32(gl.double().cpu().numpy(), rl, f"grad_sampling_locations ({path})")
        G.assert_backward_f32(ga.double().cpu().numpy(), ra, f"grad_attention_weights ({path})")


def test_workspace_too_small_is_rejected():
    inp = random_inputs(15, B=1, M=2, D=8, K=2, shapes=SHAPES[0], Lq=4)
    d = G.device_inputs(inp)
    B, S, M, D = inp.value.shape
    need = binding.workspace_size(B, S, M, D, 4, 1, 2)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.MSDAError) as e:
        binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                         d["sampling_locations"], d["attention_weights"], d["grad_output"],
                         workspace=small)
    assert e.value.status == 6


def test_misaligned_pointer_is_rejected():
    inp = random_inputs(11, B=1, M=2, D=8, K=2, shapes=SHAPES[0], Lq=4)
    d = G.device_inputs(inp)
    flat = torch.zeros(d["value"].numel() + 1, device="cuda")
    shifted = flat[1:].view(d["value"].shape)           # 4 bytes off a 16-byte boundary
    with pytest.raises(binding.MSDAError) as e:
        binding.forward(shifted, d["spatial_shapes"], d["level_start_index"],
                        d["sampling_locations"], d["attention_weights"])
    assert e.value.status == 4


def test_inconsistent_device_metadata_is_memory_safe():
    """A level whose start + H*W reaches past S is treated as empty: the result
    equals the oracle run with that level's weights set to zero, and no memory
    outside the buffers is touched (guard bands)."""
    inp = random_inputs(12, B=1, M=2, D=8, K=2, shapes=SHAPES[1], Lq=9)
    d = G.device_inputs(inp)
    bad = inp.level_start_index.copy()
    bad[2] = inp.value.shape[1] - 3                      # level 2 (3x4) overruns S
    d["level_start_index"] = torch.from_numpy(bad).cuda()
    got = G.gpu_forward(d)
    attn = inp.attention_weights.copy()
    attn[:, :, :, 2, :] = 0.0
    ref = G.oracle_forward(dataclasses.replace(inp, attention_weights=attn))
    G.assert_forward_f32(got, ref, "forward with an overrunning level")
    for path in G.BACKWARD_PATHS:
        gv, gl, ga = G.gpu_backward(d, path)
        assert np.all(gl[:, :, :, 2] == 0.0) and np.all(ga[:, :, :, 2] == 0.0), path


def test_host_metadata_is_checked():
    inp = random_inputs(13, B=1, M=2, D=8, K=2, shapes=SHAPES[1], Lq=3)
    d = G.device_inputs(inp)
    bad = torch.from_numpy(inp.level_start_index.copy())
    bad[1] += 1
    with pytest.raises(binding.MSDAError) as e:
        binding.forward(d["value"], torch.from_numpy(inp.spatial_shapes), bad,
                        d["sampling_locations"], d["attention_weights"])
    assert e.value.status == 2
    out = binding.forward(d["value"], torch.from_numpy(inp.spatial_shapes),
                          torch.from_numpy(inp.level_start_index),
                          d["sampling_locations"], d["attention_weights"])
    torch.cuda.synchronize()
    G.assert_forward_f32(out.double().cpu().numpy(), G.oracle_forward(inp))


def test_autograd_function_and_side_stream():
    from scale_deformable_attention_backward_b200 import ms_deform_attn
    inp = random_inputs(14, B=2, M=2, D=8, K=2, shapes=SHAPES[1], Lq=17)
    d = G.device_inputs(inp)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        v = d["value"].clone().requires_grad_()
        lo = d["sampling_locations"].clone().requires_grad_()
        at = d["attention_weights"].clone().requires_grad_()
        out = ms_deform_attn(v, d["spatial_shapes"], d["level_start_index"], lo, at, 64)
        out.backward(d["grad_output"])
    s.synchronize()
    G.assert_forward_f32(out.detach().double().cpu().numpy(), G.oracle_forward(inp))
    rv, rl, ra = G.oracle_backward(inp)
    G.assert_backward_f32(v.grad.double().cpu().numpy(), rv, "autograd grad_value")
    G.assert_backward_f32(lo.grad.double().cpu().numpy(), rl, "autograd grad_loc")
    G.assert_backward_f32(at.grad.double().cpu().numpy(), ra, "autograd grad_attn")
