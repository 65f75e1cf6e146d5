"""The pins are strong enough: each plausible mistake, planted in a copy of the
oracle's C source and compiled on the CPU, fails at least one pin -- and at
least one pin that does not use grid_sample.

A mutant is a textual edit of ``oracle/msda_oracle.c``; the edit's "before"
text must occur in the source, so a mutant can never silently be a no-op.
Every mutant keeps its memory accesses inside the arrays it is given (index
mistakes are wrapped into the level with a modulo or a smaller stride), so none can crash the
test process.
"""
import pytest

import oracle
from oracle import build as oracle_build
import oracle_pins
import fused_pins

SOURCE = open(oracle_build.SOURCE).read()

# (name, before, after, replace every occurrence?)
MUTANTS = [
    ("shift_sign_x", "loc_x * (double)W - 0.5", "loc_x * (double)W + 0.5", False),
    ("no_shift_y", "loc_y * (double)H - 0.5", "loc_y * (double)H", False),
    ("swap_x_scale", "loc_x * (double)W", "loc_x * (double)H", False),
    ("swap_loc_components", "sampling_locations[2 * p + 0],\n                            sampling_locations[2 * p + 1]",
     "sampling_locations[2 * p + 1],\n                            sampling_locations[2 * p + 0]", False),
    ("edge_last_pixel_dropped", "c <= (double)(n - 1)", "c <= (double)(n - 2)", False),
    ("edge_first_pixel_dropped", "c >= 0.0 &&", "c >= 1.0 &&", False),
    ("swapped_weights", "double wx[2] = {1.0 - c.fx, c.fx};", "double wx[2] = {c.fx, 1.0 - c.fx};", True),
    ("ignore_level_start", "start + yi * W + xi", "yi * W + xi", False),
    ("row_stride_wrong", "b, start, W,", "b, start, (H < W ? H : W),", False),
    ("head_channel_transposed_out", "output[(b * Lq + q) * M * D + m * D + d] += A * sample",
     "output[(b * Lq + q) * M * D + d * M + m] += A * sample", False),
    ("attention_not_applied", "+= A * sample;", "+= sample;", False),
    ("dropped_corner_forward", "for (int i = 0; i < 2; ++i)\n                        sample += wx[i] * wy[j] *",
     "for (int i = 0; i < 1; ++i)\n                        sample += wx[i] * wy[j] *", False),
    ("grad_x_sign", "wy[0] * (v[0][1] - v[0][0])", "wy[0] * (v[0][0] - v[0][1])", False),
    ("grad_y_wrong_diff", "wx[0] * (v[1][0] - v[0][0])", "wx[0] * (v[1][0] - v[0][1])", False),
    ("grad_loc_scale_swapped", "A * (double)W * g_x", "A * (double)H * g_x", False),
    ("grad_loc_no_attention", "= A * (double)H * g_y", "= (double)H * g_y", False),
    ("grad_attn_no_gO", "g_attn += gO * sample;", "g_attn += sample;", False),
    ("grad_value_no_attention", "A * wx[i] * wy[j] * gO;", "wx[i] * wy[j] * gO;", False),
    ("grad_value_column_major", "start + c.yi[j] * W + c.xi[i]", "start + (c.xi[i] * H + c.yi[j]) % (H * W)", False),
    ("grad_value_wrong_corner_weight", "A * wx[i] * wy[j] * gO;", "A * wx[1 - i] * wy[j] * gO;", False),
    ("grad_value_drops_lower_row", "if (c.xi[i] >= 0 && c.yi[j] >= 0)", "if (c.xi[i] >= 0 && c.yi[j] >= 0 && j == 0)", False),
    # The step before the core (fused entry points).
    ("fused_normaliser_swapped", "off[2 * p + 0], W,", "off[2 * p + 0], H,", False),
    ("fused_reference_components_swapped", "form_location(r[0], R == 4 ? r[2] : 0.0",
     "form_location(r[1], R == 4 ? r[2] : 0.0", False),
    ("fused_box_half_dropped_f32", "t = t * 0.5f;", "t = t * 1.0f;", False),
    ("fused_box_size_swapped", "R == 4 ? r[2] : 0.0, off[2 * p + 0]", "R == 4 ? r[3] : 0.0, off[2 * p + 0]", False),
    ("fused_softmax_unnormalised", "A[g * LK + i] = exp(z[i] - zmax) / sum;", "A[g * LK + i] = exp(z[i] - zmax);", False),
    ("fused_softmax_no_max", "sum += exp(z[i] - zmax);", "sum += exp(z[i]);", False),
    ("fused_logit_grad_not_centred", "* (gA[g * LK + i] - s);", "* gA[g * LK + i];", False),
    ("fused_offset_grad_unscaled", "grad_sampling_offsets[2 * p + c] = gl * dloc_doff;",
     "grad_sampling_offsets[2 * p + c] = gl;", False),
    ("fused_offset_grad_wrong_axis", "1.0 / (double)(c == 0 ? W : H)", "1.0 / (double)(c == 0 ? H : W)", False),
    ("fused_box_size_grad_half_dropped", "gl * sampling_offsets[2 * p + c] * 0.5 / (double)K;",
     "gl * sampling_offsets[2 * p + c] / (double)K;", False),
    ("fused_reference_grad_dropped", "gr[c] += gl;", "gr[c] += 0.0 * gl;", False),
]


def _mutate(before, after, every):
    assert before in SOURCE, f"mutant pattern not found: {before!r}"
    return SOURCE.replace(before, after) if every else SOURCE.replace(before, after, 1)


def _failing_pins(orc, pins):
    failed = []
    for pin in pins:
        try:
            pin(orc)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name,before,after,every", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, before, after, every):
    src = tmp_path / f"mutant_{name}.c"
    src.write_text(_mutate(before, after, every))
    lib = oracle_build.compile_source(str(src), str(tmp_path / f"libmutant_{name}.so"))
    orc = oracle.Oracle(lib)
    failed = _failing_pins(orc, oracle_pins.FIRST_PRINCIPLES_PINS + fused_pins.FIRST_PRINCIPLES_PINS)
    assert failed, f"mutant {name} passes every first-principles pin"
