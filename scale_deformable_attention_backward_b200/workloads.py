"""Seeded synthetic inputs for the MSDeformAttn core.

This module is shared by the CUDA path's tests/benchmark and by the oracle's
tests, and it holds none of the operator's own arithmetic: it only draws the
operator's *inputs* (value, sampling locations, attention weights and the
incoming gradient) the way a Deformable DETR layer would produce them.

Geometry and input recipes follow the pages:

* Level shapes come from a ResNet-50 + neck at strides 8/16/32/64 ("Deformable
  DETR Deformable Transformers for End-to-End Object Detection", 方法设计 /
  多尺度特征图构建 table).  The encoder geometry (100,150),(50,75),(25,38),(13,19)
  is an 800x1200 image; the bf16 geometry (76,106),(38,53),(19,27),(8,13) is the
  one the get_reference_points walkthrough prints (its per-level token counts
  8056 / 2014 / 513 / 104).
* Encoder reference points are pixel centres ``(j + 0.5) / W, (i + 0.5) / H`` of
  every token, divided by the image's valid ratio on its own level and then
  multiplied by the valid ratio of each target level (get_reference_points,
  重点知识1).  Without padding the ratios are 1 and the point is shared by all
  levels.
* Sampling locations are ``reference + offset / (W_l, H_l)`` with the offset in
  pixels of level l, and attention weights are a softmax over the L*K points of
  a head ("Deformable DETR模型解读", MultiScaleDeformableAttention.forward).
  Here offsets and logits are drawn at random instead of being predicted by
  linear layers (those layers are outside the core op).

Every draw comes from one ``numpy.random.default_rng(seed)`` in a fixed order:
value, reference points, offsets, logits, grad_output.  Generation runs in
float64 and casts at the end (value to bfloat16 with round-to-nearest-even for
the bf16 workloads, and grad_output too when they include the backward; locations
and weights always float32).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

ENCODER_800x1200 = [(100, 150), (50, 75), (25, 38), (13, 19)]
ENCODER_608x848 = [(76, 106), (38, 53), (19, 27), (8, 13)]


@dataclasses.dataclass(frozen=True)
class Config:
    """One named workload: geometry, input recipe and which passes it covers."""

    name: str
    B: int
    M: int
    D: int
    K: int
    shapes: Tuple[Tuple[int, int], ...]
    recipe: str            # "uniform" | "encoder" | "decoder" | "encoder_valid_ratio"
                           # | "decoder_box"
    dtype: str             # value dtype: "f32" | "bf16"
    backward: bool         # whether the workload includes the training backward
    Lq: Optional[int] = None   # None: one query per value token (self-attention)
    description: str = ""

    @property
    def L(self) -> int:
        return len(self.shapes)

    @property
    def S(self) -> int:
        return sum(h * w for h, w in self.shapes)

    @property
    def queries(self) -> int:
        return self.S if self.Lq is None else self.Lq

    def with_batch(self, B: int) -> "Config":
        return dataclasses.replace(self, B=B)


CONFIGS: Dict[str, Config] = {
    "tiny_fp32": Config(
        "tiny_fp32", B=1, M=2, D=8, K=2, shapes=((8, 8), (4, 4)), recipe="uniform",
        dtype="f32", backward=True,
        description="tiny fp32 fwd+bwd: B=1 M=2 D=8 K=2, levels (8,8),(4,4), S=Lq=80, "
                    "locations U[-0.1,1.1]^2"),
    "encoder_fp32": Config(
        "encoder_fp32", B=2, M=8, D=32, K=4, shapes=tuple(ENCODER_800x1200),
        recipe="encoder", dtype="f32", backward=False,
        description="encoder self-attention fp32 fwd: B=2 M=8 D=32 K=4 L=4, "
                    "levels (100,150),(50,75),(25,38),(13,19), S=Lq=19947"),
    "decoder_fp32": Config(
        "decoder_fp32", B=2, M=8, D=32, K=4, shapes=tuple(ENCODER_800x1200),
        recipe="decoder", dtype="f32", backward=False, Lq=300,
        description="decoder cross-attention fp32 fwd: B=2 Lq=300 M=8 D=32 K=4 L=4, "
                    "value over the 800x1200 encoder levels"),
    "encoder_bf16": Config(
        "encoder_bf16", B=8, M=8, D=32, K=4, shapes=tuple(ENCODER_608x848),
        recipe="encoder_valid_ratio", dtype="bf16", backward=False,
        description="encoder bf16 fwd (fp32 accumulate): B=8 M=8 D=32 K=4 L=4, "
                    "levels (76,106),(38,53),(19,27),(8,13), S=Lq=10687, valid ratios U[0.7,1]"),
    "encoder_train_fp32": Config(
        "encoder_train_fp32", B=4, M=8, D=32, K=4, shapes=tuple(ENCODER_800x1200),
        recipe="encoder", dtype="f32", backward=True,
        description="encoder training fp32 fwd+bwd: B=4 M=8 D=32 K=4 L=4, "
                    "levels (100,150),(50,75),(25,38),(13,19), S=Lq=19947"),
    "decoder_box_train_fp32": Config(
        "decoder_box_train_fp32", B=2, M=8, D=32, K=4, shapes=tuple(ENCODER_800x1200),
        recipe="decoder_box", dtype="f32", backward=True, Lq=300,
        description="decoder cross-attention with box reference points fp32 fwd+bwd: B=2 "
                    "Lq=300 M=8 D=32 K=4 L=4 over the 800x1200 encoder levels; box centre "
                    "U[0.05,0.95]^2, size U[0.05,0.5]^2, offsets N(0,1)*K/2 box units"),
    "encoder_train_bf16": Config(
        "encoder_train_bf16", B=8, M=8, D=32, K=4, shapes=tuple(ENCODER_608x848),
        recipe="encoder_valid_ratio", dtype="bf16", backward=True,
        description="encoder training bf16 fwd+bwd (fp32 arithmetic and gradients): B=8 M=8 "
                    "D=32 K=4 L=4, levels (76,106),(38,53),(19,27),(8,13), S=Lq=10687, "
                    "valid ratios U[0.7,1]")
}


@dataclasses.dataclass
class Inputs:
    """Host arrays for one call of the operator (numpy, C-contiguous)."""

    config: Config
    value: np.ndarray                  # [B,S,M,D] float32 (bf16-representable for bf16)
    value_bf16_bits: Optional[np.ndarray]  # [B,S,M,D] uint16 raw bf16, bf16 workloads only
    spatial_shapes: np.ndarray         # [L,2] int64 (H, W)
    level_start_index: np.ndarray      # [L] int64
    sampling_locations: np.ndarray     # [B,Lq,M,L,K,2] float32
    attention_weights: np.ndarray      # [B,Lq,M,L,K] float32
    grad_output: Optional[np.ndarray]  # [B,Lq,M*D] float32, backward workloads only
    grad_output_bf16_bits: Optional[np.ndarray] = None  # raw bf16 of grad_output (bf16 only)

    @property
    def dims(self) -> Dict[str, int]:
        B, S, M, D = self.value.shape
        _, Lq, _, L, K, _ = self.sampling_locations.shape
        return dict(B=B, S=S, M=M, D=D, Lq=Lq, L=L, K=K)


def level_metadata(shapes) -> Tuple[np.ndarray, np.ndarray]:
    """spatial_shapes [L,2] (H, W) and level_start_index [L] (exclusive prefix sum
    of H*W), the flattening of "Deformable DETR模型解读" pre_transformer."""
    ss = np.asarray(shapes, dtype=np.int64).reshape(-1, 2)
    sizes = ss[:, 0] * ss[:, 1]
    start = np.concatenate([np.zeros(1, dtype=np.int64), np.cumsum(sizes)[:-1]]).astype(np.int64)
    return ss, start


def bf16_round_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); return the raw 16 bits."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _pixel_centres(shapes) -> List[np.ndarray]:
    """Per level, the [H*W, 2] (x, y) normalised pixel centres in row-major order."""
    out = []
    for h, w in shapes:
        ys, xs = np.meshgrid((np.arange(h) + 0.5) / h, (np.arange(w) + 0.5) / w, indexing="ij")
        out.append(np.stack([xs.reshape(-1), ys.reshape(-1)], -1))
    return out


def _reference_points(cfg: Config, rng: np.random.Generator, Lq: int) -> np.ndarray:
    """[B, Lq, L, 2] reference points, per the workload's recipe."""
    B, L = cfg.B, cfg.L
    if cfg.recipe == "encoder":
        ref = np.concatenate(_pixel_centres(cfg.shapes), 0)          # [S, 2]
        return np.broadcast_to(ref[None, :, None, :], (B, Lq, L, 2)).copy()
    if cfg.recipe == "decoder":
        ref = rng.uniform(0.05, 0.95, size=(B, Lq, 2))
        return np.broadcast_to(ref[:, :, None, :], (B, Lq, L, 2)).copy()
    if cfg.recipe == "encoder_valid_ratio":
        # Per image the un-padded fraction r of the padded canvas; on each level the
        # valid ratio is the rounded valid extent over the level's extent, as the
        # downsampled padding mask would give it.
        r = rng.uniform(0.7, 1.0, size=(B, 2))                        # (r_x, r_y)
        hw = np.asarray(cfg.shapes, dtype=np.float64)                 # [L, (H, W)]
        vr = np.empty((B, L, 2))
        vr[:, :, 0] = np.round(r[:, None, 0] * hw[None, :, 1]) / hw[None, :, 1]
        vr[:, :, 1] = np.round(r[:, None, 1] * hw[None, :, 0]) / hw[None, :, 0]
        per_level = []
        for lvl, (h, w) in enumerate(cfg.shapes):
            ys, xs = np.meshgrid(np.arange(h) + 0.5, np.arange(w) + 0.5, indexing="ij")
            ref_x = xs.reshape(-1)[None] / (vr[:, None, lvl, 0] * w)
            ref_y = ys.reshape(-1)[None] / (vr[:, None, lvl, 1] * h)
            per_level.append(np.stack([ref_x, ref_y], -1))            # [B, HW, 2]
        ref = np.concatenate(per_level, 1)                            # [B, S, 2]
        return ref[:, :, None, :] * vr[:, None, :, :]
    raise ValueError(cfg.recipe)


def _box_references(rng: np.random.Generator, B: int, Lq: int, L: int) -> np.ndarray:
    """[B, Lq, L, 4] box reference points (centre x, y, size w, h; normalised),
    one box per query shared by the levels, as a box-refining decoder layer feeds
    them ("Deformable DETR模型解读", MultiScaleDeformableAttention.forward, the
    4-component branch)."""
    centre = rng.uniform(0.05, 0.95, size=(B, Lq, 2))
    size = rng.uniform(0.05, 0.5, size=(B, Lq, 2))
    box = np.concatenate([centre, size], -1)
    return np.broadcast_to(box[:, :, None, :], (B, Lq, L, 4)).copy()


def make_inputs(cfg: Config, seed: int = 0, with_grad: Optional[bool] = None) -> Inputs:
    """Draw one seeded set of inputs for ``cfg``."""
    rng = np.random.default_rng(seed)
    B, M, D, K, L = cfg.B, cfg.M, cfg.D, cfg.K, cfg.L
    shapes = [tuple(s) for s in cfg.shapes]
    ss, start = level_metadata(shapes)
    S, Lq = cfg.S, cfg.queries

    value64 = rng.standard_normal((B, S, M, D))
    value32 = value64.astype(np.float32)
    bits = None
    if cfg.dtype == "bf16":
        bits = bf16_round_bits(value32)
        value32 = bf16_to_f32_exact(bits)

    if cfg.recipe == "uniform":
        loc = rng.uniform(-0.1, 1.1, size=(B, Lq, M, L, K, 2))
    elif cfg.recipe == "decoder_box":
        box = _box_references(rng, B, Lq, L)                            # [B, Lq, L, 4]
        off = rng.standard_normal((B, Lq, M, L, K, 2)) * (K / 2.0)
        loc = box[:, :, None, :, None, :2] + off / K * box[:, :, None, :, None, 2:] * 0.5
    else:
        ref = _reference_points(cfg, rng, Lq)                        # [B, Lq, L, 2]
        if cfg.recipe == "decoder":
            off = rng.standard_normal((B, Lq, M, L, K, 2)) * 0.02
        else:
            px = rng.standard_normal((B, Lq, M, L, K, 2)) * 2.0       # pixels of level l
            wh = ss[:, ::-1].astype(np.float64)                       # [L, (W, H)]
            off = px / wh[None, None, None, :, None, :]
        loc = ref[:, :, None, :, None, :] + off

    logits = rng.standard_normal((B, Lq, M, L * K))
    logits -= logits.max(-1, keepdims=True)
    e = np.exp(logits)
    attn = (e / e.sum(-1, keepdims=True)).reshape(B, Lq, M, L, K)

    want_grad = cfg.backward if with_grad is None else with_grad
    grad = rng.standard_normal((B, Lq, M * D)).astype(np.float32) if want_grad else None
    grad_bits = None
    if grad is not None and cfg.dtype == "bf16":
        grad_bits = bf16_round_bits(grad)
        grad = bf16_to_f32_exact(grad_bits)

    return Inputs(
        config=cfg,
        value=np.ascontiguousarray(value32),
        value_bf16_bits=bits,
        spatial_shapes=ss,
        level_start_index=start,
        sampling_locations=np.ascontiguousarray(loc.astype(np.float32)),
        attention_weights=np.ascontiguousarray(attn.astype(np.float32)),
        grad_output=grad,
        grad_output_bf16_bits=grad_bits,
    )


@dataclasses.dataclass
class FusedInputs:
    """Host arrays for one call of the fused op (raw reference points, offsets and
    logits instead of locations and weights)."""

    config: Config
    value: np.ndarray                  # [B,S,M,D] float32 (bf16-representable for bf16)
    value_bf16_bits: Optional[np.ndarray]
    spatial_shapes: np.ndarray         # [L,2] int64 (H, W)
    level_start_index: np.ndarray      # [L] int64
    reference_points: np.ndarray       # [B,Lq,L,R] float32, R = 2 or 4 (boxes)
    sampling_offsets: np.ndarray       # [B,Lq,M,L,K,2] float32
    attention_logits: np.ndarray       # [B,Lq,M,L*K] float32
    grad_output: Optional[np.ndarray]  # [B,Lq,M*D] float32, backward workloads only


def make_fused_inputs(cfg: Config, seed: int = 0,
                      with_grad: Optional[bool] = None) -> FusedInputs:
    """The raw inputs behind :func:`make_inputs` (same draws in the same order):
    reference points, offsets (pixels of level l for 2-component references,
    box units for boxes) and the softmax logits.  For the "uniform" recipe the
    2-component reference points are drawn U[-0.1, 1.1]^2 and the offsets
    N(0, 1) pixels."""
    rng = np.random.default_rng(seed)
    B, M, D, K, L = cfg.B, cfg.M, cfg.D, cfg.K, cfg.L
    shapes = [tuple(s) for s in cfg.shapes]
    ss, start = level_metadata(shapes)
    S, Lq = cfg.S, cfg.queries
    wh = ss[:, ::-1].astype(np.float64)                               # [L, (W, H)]

    value64 = rng.standard_normal((B, S, M, D))
    value32 = value64.astype(np.float32)
    bits = None
    if cfg.dtype == "bf16":
        bits = bf16_round_bits(value32)
        value32 = bf16_to_f32_exact(bits)

    if cfg.recipe == "uniform":
        ref = rng.uniform(-0.1, 1.1, size=(B, Lq, L, 2))
        off = rng.standard_normal((B, Lq, M, L, K, 2))
    elif cfg.recipe == "decoder_box":
        ref = _box_references(rng, B, Lq, L)
        off = rng.standard_normal((B, Lq, M, L, K, 2)) * (K / 2.0)
    else:
        ref = _reference_points(cfg, rng, Lq)
        if cfg.recipe == "decoder":
            off = rng.standard_normal((B, Lq, M, L, K, 2)) * 0.02 * wh[None, None, None, :, None, :]
        else:
            off = rng.standard_normal((B, Lq, M, L, K, 2)) * 2.0

    logits = rng.standard_normal((B, Lq, M, L * K))
    want_grad = cfg.backward if with_grad is None else with_grad
    grad = rng.standard_normal((B, Lq, M * D)).astype(np.float32) if want_grad else None
    f32 = lambda a: np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return FusedInputs(config=cfg, value=np.ascontiguousarray(value32), value_bf16_bits=bits,
                       spatial_shapes=ss, level_start_index=start, reference_points=f32(ref),
                       sampling_offsets=f32(off), attention_logits=f32(logits),
                       grad_output=grad)


def select_fused_queries(inp: FusedInputs, queries: np.ndarray) -> FusedInputs:
    """The same fused call restricted to a subset of queries (value untouched)."""
    q = np.asarray(queries, dtype=np.int64)
    take = lambda a: np.ascontiguousarray(a[:, q])
    return dataclasses.replace(
        inp, reference_points=take(inp.reference_points),
        sampling_offsets=take(inp.sampling_offsets),
        attention_logits=take(inp.attention_logits),
        grad_output=None if inp.grad_output is None else take(inp.grad_output))


def bf16_to_f32_exact(bits: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(bf16_bits_to_f32(bits))


def select_queries(inp: Inputs, queries: np.ndarray) -> Inputs:
    """The same call restricted to a subset of queries (value untouched).

    Outputs, grad_sampling_locations and grad_attention_weights of a query depend
    only on that query's own rows, so the restricted call reproduces them."""
    q = np.asarray(queries, dtype=np.int64)
    return dataclasses.replace(
        inp,
        sampling_locations=np.ascontiguousarray(inp.sampling_locations[:, q]),
        attention_weights=np.ascontiguousarray(inp.attention_weights[:, q]),
        grad_output=None if inp.grad_output is None else np.ascontiguousarray(inp.grad_output[:, q]),
        grad_output_bf16_bits=None if inp.grad_output_bf16_bits is None
        else np.ascontiguousarray(inp.grad_output_bf16_bits[:, q]),
    )
