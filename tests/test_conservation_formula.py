"""The conservation identity that test_conservation_gpu.py checks the kernels
against, checked here against the float64 oracle on 3,000 queries of one image
of the training workload (where a fifth of the points have corners outside the
map, so the in-map mass matters)."""
import numpy as np

import oracle
import test_conservation_gpu as T
from scale_deformable_attention_backward_b200 import workloads as W


def test_conservation_identity_matches_the_oracle():
    inp = W.make_inputs(W.CONFIGS["encoder_train_fp32"].with_batch(1), seed=21)
    inp = W.select_queries(inp, np.arange(3000))
    gv, _, _ = oracle.backward(inp.value, inp.spatial_shapes, inp.level_start_index,
                               inp.sampling_locations, inp.attention_weights, inp.grad_output)
    B, S, M, D = inp.value.shape
    Lq = inp.sampling_locations.shape[1]
    mass = T.in_map_mass(inp.sampling_locations, [tuple(s) for s in inp.spatial_shapes])
    assert 0.1 < (mass < 1).mean() < 0.5
    per_query = (inp.attention_weights.astype(np.float64) * mass).sum(axis=(3, 4))
    want = np.einsum("bqm,bqmd->bmd", per_query,
                     inp.grad_output.astype(np.float64).reshape(B, Lq, M, D))
    np.testing.assert_allclose(gv.sum(axis=1), want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
