"""msda_backward_noalloc through the C ABI: the backward for callers that cannot
allocate device memory at call time (a framework that owns the whole memory pool,
or a latency-critical path where cudaMalloc / cudaFree would block).  Its scratch
is a fixed array inside the library, so its results must equal those of
msda_backward given a workspace by the caller -- on every call, since the array
keeps the previous call's contents.

This file is collected last, so that a run stopping at its first failure has
already run every other test; it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import gpu_support as G
from scale_deformable_attention_backward_b200 import binding
from scale_deformable_attention_backward_b200 import workloads as W

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20  # MSDA_NOALLOC_SCRATCH_BYTES in include/msda.h


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dims(d):
    B, S, M, D = d["value"].shape
    _, Lq, _, L, K, _ = d["sampling_locations"].shape
    return B, S, M, D, Lq, L, K


def _outputs(d):
    return (torch.full_like(d["value"], 3.0), torch.full_like(d["sampling_locations"], 3.0),
            torch.full_like(d["attention_weights"], 3.0))


def _noalloc(lib, d, outs):
    gv, gl, ga = outs
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.msda_backward_noalloc(*_dims(d), 0, _p(d["value"]), _p(d["spatial_shapes"]),
                                     _p(d["level_start_index"]), _p(d["sampling_locations"]),
                                     _p(d["attention_weights"]), _p(d["grad_output"]), _p(gv),
                                     _p(gl), _p(ga), stream)


def _with_workspace(lib, d, outs):
    gv, gl, ga = outs
    need = binding.workspace_size(*_dims(d))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.msda_backward(*_dims(d), 0, _p(d["value"]), _p(d["spatial_shapes"]),
                             _p(d["level_start_index"]), _p(d["sampling_locations"]),
                             _p(d["attention_weights"]), _p(d["grad_output"]), _p(gv), _p(gl),
                             _p(ga), _p(ws), need, stream)


def _inputs(name, seed):
    if name == "tiny_fp32":
        return W.make_inputs(W.CONFIGS["tiny_fp32"], seed=seed)
    enc = W.make_inputs(W.CONFIGS["encoder_train_fp32"].with_batch(1), seed=seed)
    return W.select_queries(enc, np.arange(0, enc.config.queries, 9))  # 2217 queries


NAMES = ("grad_value", "grad_sampling_locations", "grad_attention_weights")


def test_noalloc_matches_backward_with_workspace_and_oracle():
    """Calls with different layouts and inputs in a row -- the encoder subset,
    the tiny workload, the encoder subset with another seed, and the first
    input again -- each compared with msda_backward given a caller workspace
    and with the float64 oracle.  The array keeps each call's contents, so a
    leftover from the previous call would show up in the next one.  From the
    second call on, the device's free memory must not change across a call:
    the first call has loaded the kernels and reserved the array."""
    lib = binding.library()
    sequence = [("encoder_b1_subset", 5), ("tiny_fp32", 0), ("encoder_b1_subset", 6),
                ("encoder_b1_subset", 5)]
    for call, (name, seed) in enumerate(sequence):
        inp = _inputs(name, seed)
        d = G.device_inputs(inp)
        assert binding.workspace_size(*_dims(d)) <= SCRATCH_BYTES
        ref = _outputs(d)
        assert _with_workspace(lib, d, ref) == 0
        outs = _outputs(d)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        assert _noalloc(lib, d, outs) == 0
        torch.cuda.synchronize()
        if call > 0:
            assert torch.cuda.mem_get_info()[0] == free_before, \
                f"call {call + 1} changed the free device memory"
        want_oracle = G.oracle_backward(inp)
        for got, want_ws, want_or, what in zip(outs, ref, want_oracle, NAMES):
            got = got.double().cpu().numpy()
            tag = f"{name} seed {seed} {what}, no-alloc call {call + 1}"
            G.assert_backward_f32(got, want_ws.double().cpu().numpy(), tag + " vs workspace")
            G.assert_backward_f32(got, want_or, tag + " vs oracle")
    assert not binding.wait_failed()


def test_noalloc_rejects_sizes_beyond_its_scratch_and_bf16():
    lib = binding.library()
    B, S, M, D, Lq, L, K = 4, 19947, 8, 32, 19947, 4, 4
    assert binding.workspace_size(B, S, M, D, Lq, L, K) > SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the call is rejected first
    status = lib.msda_backward_noalloc(B, S, M, D, Lq, L, K, 0, *([fake] * 9), None)
    assert status == 6  # MSDA_ERR_WORKSPACE
    status = lib.msda_backward_noalloc(1, 80, 2, 8, 80, 2, 2, 1, *([fake] * 9), None)
    assert status == 3  # MSDA_ERR_UNSUPPORTED: the sorted path is float32 only
