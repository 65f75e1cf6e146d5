"""GPU parity of the tiled forward (csrc/msda_forward_tiled.cu), the kernel the
encoder form of the op runs: the queries are the value's own pixels (Lq == S),
and each CTA stages the value windows of a rectangle of queries in shared
memory.

Every case is compared with the float64 oracle, and with the per-point gather
kernel (selected by MSDA_FORWARD_KERNEL=gather) on the same inputs.  The tiled
kernels add the same float32 products as the gather kernel in the same order --
level, point, corner -- so at full size they agree with it bit for bit.  On the
small cases here the gather kernel spreads each query's points over several
sub-warps (too few queries to fill the GPU otherwise) and adds partial sums, so
there the comparison is within the float32 forward tolerance.

The cases cover the three kinds of step the kernel has: windows that fit the
shared buffer (encoder locality), windows that do not (non-local samples: the
step reads value from global memory), and the one-dimensional tiling used when
the level metadata is not a row-major partition of the queries."""
import contextlib
import dataclasses
import os

import numpy as np
import pytest
import torch

import gpu_support as G
from scale_deformable_attention_backward_b200 import binding
from scale_deformable_attention_backward_b200 import workloads as W

pytestmark = pytest.mark.gpu

SMALL_ENCODER = ((24, 40), (12, 20), (6, 10), (3, 5))


TILED_KERNELS = ("staged", "l1")


@contextlib.contextmanager
def forward_kernel(name):
    old = os.environ.get("MSDA_FORWARD_KERNEL")
    os.environ["MSDA_FORWARD_KERNEL"] = name
    try:
        yield
    finally:
        if old is None:
            del os.environ["MSDA_FORWARD_KERNEL"]
        else:
            os.environ["MSDA_FORWARD_KERNEL"] = old


def all_kernels(inp):
    d = G.device_inputs(inp)
    out = {}
    for name in TILED_KERNELS + ("gather",):
        with forward_kernel(name):
            out[name] = G.gpu_forward(d)
    return out


def check(inp, what):
    out = all_kernels(inp)
    assert not binding.wait_failed(), f"{what}: a bounded wait ran out"
    ref = G.oracle_forward(inp)
    for name in TILED_KERNELS:
        if inp.config.dtype == "bf16":
            # Two roundings of float32 sums that differ in their last bits can be
            # one bfloat16 step (2^-7 relative) apart.
            a, b = out[name], out["gather"]
            scale = np.abs(b).max()
            assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.abs(b) + 1e-5 * scale), \
                f"{what} ({name} vs gather)"
        else:
            G.assert_forward_f32(out[name], out["gather"], f"{what} ({name} vs gather)")
        if inp.config.dtype == "bf16":
            G.assert_forward_bf16(out[name], ref, f"{what} ({name})")
        else:
            G.assert_forward_f32(out[name], ref, f"{what} ({name})")


def encoder(name, B, M, D, K, shapes=SMALL_ENCODER, dtype="f32", recipe="encoder", seed=0):
    cfg = W.Config(name, B, M, D, K, tuple(shapes), recipe, dtype, False)
    return W.make_inputs(cfg, seed=seed)


@pytest.mark.parametrize("K", [1, 3, 4, 5, 8])
def test_encoder_point_counts(K):
    """K <= 4 gives 8 x 16 query tiles, 4 < K <= 8 gives 8 x 8."""
    check(encoder("enc", B=2, M=4, D=32, K=K, seed=K), f"encoder K={K}")


@pytest.mark.parametrize("D,dtype", [(16, "f32"), (32, "f32"), (64, "f32"),
                                     (32, "bf16"), (64, "bf16"), (128, "bf16")])
def test_encoder_row_widths(D, dtype):
    """One pixel of one head is 64, 128 or 256 bytes: the copy and gather widths."""
    check(encoder("enc", B=2, M=3, D=D, K=4, dtype=dtype, seed=D), f"encoder D={D} {dtype}")


def test_encoder_valid_ratios_bf16():
    """The bf16 encoder recipe: reference points scaled by per-level valid ratios."""
    check(encoder("enc", B=3, M=2, D=32, K=4, shapes=((19, 27), (10, 14), (5, 7), (3, 4)),
                  dtype="bf16", recipe="encoder_valid_ratio", seed=5), "valid ratios")


def test_nonlocal_samples_take_global_steps():
    """Uniform locations over 1.2x the map: the fine level's window (the whole
    48 x 64 map, 3072 pixels) exceeds the shared buffer and its steps read value
    from global memory, while the coarse levels' windows are staged."""
    check(encoder("uni", B=2, M=2, D=32, K=4, shapes=((48, 64), (24, 32), (12, 16)),
                  recipe="uniform", seed=11), "uniform locations")


def test_outliers_and_nonfinite_locations():
    """Encoder locality with a few points moved far inside the map (their tile's
    window grows past the buffer for that level), far outside it (no corner:
    ignored by the window), to the map's edges, and to NaN / Inf (the output is
    NaN, as grid_sample gives)."""
    inp = encoder("enc", B=2, M=3, D=32, K=4, seed=21)
    loc = inp.sampling_locations.copy()
    rng = np.random.default_rng(22)
    B, Lq, M, L, K, _ = loc.shape
    picks = rng.integers(0, [B, Lq, M, L, K], size=(40, 5))
    for i, (b, q, m, l, k) in enumerate(picks):
        kind = i % 5
        if kind == 0:
            loc[b, q, m, l, k] = rng.uniform(0.0, 1.0, size=2)          # far, inside the map
        elif kind == 1:
            loc[b, q, m, l, k] = (rng.choice([-5.0, 7.0]), 0.5)        # outside the map
        elif kind == 2:
            loc[b, q, m, l, k] = (0.0, 1.0)                             # on the map's edge
        elif kind == 3:
            loc[b, q, m, l, k, 0] = np.nan
        else:
            loc[b, q, m, l, k, 1] = -np.inf
    check(dataclasses.replace(inp, sampling_locations=loc), "outliers")


def test_thin_levels():
    """Levels one pixel high or wide, and a level wider than many tiles."""
    check(encoder("thin", B=2, M=2, D=32, K=4, shapes=((1, 300), (40, 1), (3, 3), (1, 1)),
                  seed=31), "thin levels")


def test_single_level_and_ragged_tiles():
    """One level whose sides are not multiples of the tile's (8 x 16)."""
    check(encoder("one", B=1, M=5, D=32, K=4, shapes=((37, 53),), seed=41), "one level")


def test_one_dimensional_tiling():
    """Lq == S, but the levels are stored in reverse order: level_start_index is
    not the running total, so the queries are tiled as runs of consecutive
    queries instead of rectangles.  The op itself is defined for any start
    offsets; the oracle reads the same ones."""
    inp = encoder("rev", B=2, M=2, D=32, K=4, shapes=((20, 30), (10, 15), (5, 8)), seed=51)
    ss = inp.spatial_shapes
    sizes = ss[:, 0] * ss[:, 1]
    start = np.array([sizes[1] + sizes[2], sizes[2], 0], dtype=np.int64)
    check(dataclasses.replace(inp, level_start_index=start), "reversed levels")


@pytest.mark.parametrize("name", ["encoder_fp32", "encoder_bf16"])
def test_full_size_matches_gather_kernel(name):
    """The full-size encoder workloads (the benchmark's launch configuration):
    the tiled kernel gives exactly the gather kernel's output (both are checked
    against the oracle in test_parity_gpu.py)."""
    inp = W.make_inputs(W.CONFIGS[name], seed=0)
    out = all_kernels(inp)
    for k in TILED_KERNELS:
        assert np.array_equal(out[k], out["gather"], equal_nan=True), k


@pytest.mark.parametrize("kernel", TILED_KERNELS)
def test_guard_bands_untouched(kernel):
    inp = encoder("enc", B=2, M=3, D=32, K=4, seed=61)
    d = G.device_inputs(inp)
    B, S, M, D = inp.value.shape
    sentinel = 12345.0
    n = B * S * M * D
    buf = torch.full((n + 128,), sentinel, device="cuda")
    out = buf[64:64 + n].view(B, S, M * D)
    with forward_kernel(kernel):
        binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                        d["sampling_locations"], d["attention_weights"], output=out)
    torch.cuda.synchronize()
    assert torch.all(buf[:64] == sentinel) and torch.all(buf[-64:] == sentinel)
    G.assert_forward_f32(out.double().cpu().numpy(), G.oracle_forward(inp))


@pytest.mark.parametrize("kernel", TILED_KERNELS)
def test_inconsistent_metadata_is_memory_safe(kernel):
    """A level whose start + H*W reaches past S is treated as empty (its weights
    count as zero), in the tiled kernel as in the others."""
    inp = encoder("enc", B=1, M=2, D=32, K=4, shapes=((6, 9), (3, 5), (2, 2)), seed=71)
    d = G.device_inputs(inp)
    bad = inp.level_start_index.copy()
    bad[1] = inp.value.shape[1] - 3                      # level 1 (3 x 5) overruns S
    d["level_start_index"] = torch.from_numpy(bad).cuda()
    with forward_kernel(kernel):
        got = G.gpu_forward(d)
    attn = inp.attention_weights.copy()
    attn[:, :, :, 1, :] = 0.0
    ref = G.oracle_forward(dataclasses.replace(inp, attention_weights=attn))
    G.assert_forward_f32(got, ref, "forward with an overrunning level")
