"""Host-side arithmetic behind bench.py's roofline figures (CPU only): the
compulsory-byte counts, the grad_value add count behind the atomic rate, and the
rule that a recorded ncu traffic figure is reported only while the kernel
sources it was taken from are unchanged."""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from scale_deformable_attention_backward_b200 import workloads as W  # noqa: E402


def _shape_only_inputs(cfg, Lq=None):
    """Inputs with the right shapes and zero contents (no random draws)."""
    ss, st = W.level_metadata(cfg.shapes)
    S = int((ss[:, 0] * ss[:, 1]).sum())
    Lq = cfg.queries if Lq is None else Lq
    B, M, D, L, K = cfg.B, cfg.M, cfg.D, cfg.L, cfg.K
    z = np.zeros
    return W.Inputs(cfg, z((B, S, M, D), np.float32), None, ss, st,
                    z((B, Lq, M, L, K, 2), np.float32), z((B, Lq, M, L, K), np.float32),
                    z((B, Lq, M * D), np.float32), None)


def test_forward_bytes_per_query_on_the_encoder():
    """For the encoder (S = Lq, fp32, M=8, D=32, L=K=4) every query owns one
    token of value (1024 B), its locations and weights (8*16*12 = 1536 B) and
    its output row (1024 B): 3584 B per query."""
    cfg = W.CONFIGS["encoder_fp32"]
    inp = _shape_only_inputs(cfg)
    got = bench.algorithmic_bytes(cfg, inp)
    assert got["forward"] == 3584 * cfg.B * cfg.queries == 142_980_096


def test_backward_bytes_on_the_training_workload():
    """The backward reads value, locations, weights and grad_output and writes
    grad_value (float32), grad_loc and grad_attn: 6144 B per query here."""
    cfg = W.CONFIGS["encoder_train_fp32"]
    inp = _shape_only_inputs(cfg)
    got = bench.algorithmic_bytes(cfg, inp)
    per_query = 1024 + 1024 + 1536 + 1024 + 1536
    assert got["backward"] == per_query * cfg.B * cfg.queries == 490_217_472


def test_bf16_value_halves_value_and_output_bytes():
    cfg = W.CONFIGS["encoder_bf16"]
    inp = _shape_only_inputs(cfg)
    B, S, M, D = inp.value.shape
    Lq = inp.sampling_locations.shape[1]
    pts = B * Lq * M * cfg.L * cfg.K
    assert bench.algorithmic_bytes(cfg, inp)["forward"] == (
        B * S * M * D * 2 + pts * 12 + B * Lq * M * D * 2)


def test_grad_value_adds_counts_corners_inside_the_map():
    """Hand-placed points on one 4 x 5 level (H=4, W=5), D=8: an interior point
    has 4 corners in the map; a point on the left edge x = 0.5/W (pixel x = 0,
    cell x0 = 0) also 4; a point left of the first pixel centre (x0 = -1) 2; a
    point in the top-left corner cell (x0 = y0 = -1) 1; one far outside 0."""
    cfg = W.Config("hand", 1, 1, 8, 1, ((4, 5),), "uniform", "f32", True, 5)
    inp = _shape_only_inputs(cfg)
    locs = [(0.5, 0.5), (0.5 / 5, 0.5), (0.05, 0.5), (0.05, 0.05), (3.0, 3.0)]
    for q, (x, y) in enumerate(locs):
        inp.sampling_locations[0, q, 0, 0, 0] = (x, y)
    assert bench.grad_value_adds(inp) == (4 + 4 + 2 + 1 + 0) * 8


def test_recorded_traffic_requires_unchanged_sources(tmp_path, monkeypatch):
    files = ["msda_forward.cu", "msda_device.cuh"]
    rec = {"dram_bytes_per_launch": 1234, "files": files,
           "source_digest": bench.source_digest(files)}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps({"k": rec, "stale": dict(rec, source_digest="0" * 16)}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.recorded_traffic("k") == 1234
    assert bench.recorded_traffic("stale") is None
    assert bench.recorded_traffic("missing") is None


def test_committed_traffic_records_name_existing_sources():
    with open(bench.TRAFFIC_FILE) as f:
        records = json.load(f)
    assert records
    for key, rec in records.items():
        assert rec["dram_bytes_per_launch"] > 0, key
        for name in rec["files"]:
            assert os.path.exists(os.path.join(bench.KERNEL_SOURCES, name)), (key, name)


def test_single_launch_cases_run_on_their_workloads():
    assert bench.case_workload("forward_encoder") == "encoder_fp32"
    assert bench.case_workload("decoder_forward") == "decoder_fp32"
    assert bench.case_workload("decoder_backward") == "decoder_box_train_fp32"
    for case in ("forward", "backward", "backward_sorted", "fused_forward", "fused_backward",
                 "projection", "projection_f32"):
        assert bench.case_workload(case) == "encoder_train_fp32", case
    for case in bench.CASES:
        assert bench.case_workload(case) in W.CONFIGS
