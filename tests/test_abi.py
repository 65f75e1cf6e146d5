"""The C-ABI library on the host (no GPU): it loads, exports every symbol that
include/msda.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

from scale_deformable_attention_backward_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msda.h")

OK, NULLP, BAD, UNSUP, MISAL, CUDA, WORKSPACE = 0, 1, 2, 3, 4, 5, 6


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(msda_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return binding.library()


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"msda_forward", "msda_backward"} <= set(names)
    for name in names:
        assert hasattr(lib, name), f"libmsda.so does not export {name}"
        assert name in binding.SIGNATURES, f"binding has no signature for {name}"


def test_debug_library_exports_every_declared_symbol():
    from scale_deformable_attention_backward_b200.csrc import build
    path = build.DEBUG_LIBRARY
    assert os.path.exists(path), "libmsda_debug.so is missing: build.py --debug builds it"
    dbg = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(dbg, name), f"libmsda_debug.so does not export {name}"
    # The clip is host state only: no device is touched.
    dbg.msda_debug_bounds_clip.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
    assert dbg.msda_debug_bounds_clip(0, 0) == OK


def test_release_library_has_no_bounds_checks(lib):
    kind, address = ctypes.c_int(7), ctypes.c_uint64(7)
    assert lib.msda_debug_bounds_check(ctypes.byref(kind), ctypes.byref(address)) == UNSUP
    assert (kind.value, address.value) == (0, 0)
    assert lib.msda_debug_bounds_check(None, None) == NULLP
    assert lib.msda_debug_bounds_clip(16, 16) == UNSUP
    with pytest.raises(binding.MSDAError):
        binding.debug_bounds_check()


def test_status_strings_and_version(lib):
    for code in range(7):
        assert lib.msda_status_string(code)
    assert lib.msda_status_string(99) == b"unknown status"
    assert lib.msda_version() >= 100


def _i64(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int64))
    return a, ctypes.c_void_p(a.ctypes.data)


def test_check_metadata(lib):
    ss, pss = _i64([[100, 150], [50, 75], [25, 38], [13, 19]])
    st, pst = _i64([0, 15000, 18750, 19700])
    assert lib.msda_check_metadata(19947, 4, pss, pst) == OK
    assert lib.msda_check_metadata(19946, 4, pss, pst) == BAD
    st2, pst2 = _i64([0, 15000, 18751, 19700])
    assert lib.msda_check_metadata(19947, 4, pss, pst2) == BAD
    ss3, pss3 = _i64([[0, 150], [50, 75], [25, 38], [13, 19]])
    assert lib.msda_check_metadata(19947, 4, pss3, pst) == BAD
    assert lib.msda_check_metadata(19947, 4, None, pst) == NULLP
    assert lib.msda_check_metadata(0, 0, None, None) == OK
    assert lib.msda_check_metadata(-1, 0, None, None) == BAD


FAKE = 0x10000  # aligned, never dereferenced: every call below fails validation first


def _fwd(lib, B=1, S=80, M=2, D=8, Lq=80, L=2, K=2, dtype=0, value=FAKE, shapes=FAKE,
         starts=FAKE, loc=FAKE, attn=FAKE, out=FAKE):
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    return lib.msda_forward(B, S, M, D, Lq, L, K, dtype, v(value), v(shapes), v(starts), v(loc),
                            v(attn), v(out), None)


def _bwd(lib, B=1, S=80, M=2, D=8, Lq=80, L=2, K=2, dtype=0, ptrs=None, ws=None, ws_bytes=0):
    p = [FAKE] * 9 if ptrs is None else ptrs
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.msda_backward(B, S, M, D, Lq, L, K, dtype, *[v(x) for x in p], v(ws), ws_bytes,
                             None)


def _ws_size(lib, B=1, S=80, M=2, D=8, Lq=80, L=2, K=2):
    n = ctypes.c_size_t(0)
    st = lib.msda_backward_workspace_size(B, S, M, D, Lq, L, K, ctypes.byref(n))
    return st, n.value


def test_forward_argument_errors(lib):
    assert _fwd(lib, B=-1) == BAD
    assert _fwd(lib, K=-2) == BAD
    assert _fwd(lib, L=0) == UNSUP
    assert _fwd(lib, L=17) == UNSUP
    assert _fwd(lib, K=65) == UNSUP
    assert _fwd(lib, D=6) == UNSUP                 # float32 needs D % 4 == 0
    assert _fwd(lib, D=12, dtype=1) == UNSUP       # bfloat16 needs D % 8 == 0
    assert _fwd(lib, dtype=7) == UNSUP
    assert _fwd(lib, value=None) == NULLP
    assert _fwd(lib, out=None) == NULLP
    assert _fwd(lib, loc=None) == NULLP
    assert _fwd(lib, value=FAKE + 8) == MISAL
    assert _fwd(lib, out=FAKE + 4) == MISAL
    assert _fwd(lib, loc=FAKE + 4) == MISAL
    assert _fwd(lib, attn=FAKE + 2) == MISAL
    assert _fwd(lib, B=1 << 40, S=1 << 40) == BAD  # element count overflow


def test_forward_empty_work_is_ok_without_launch(lib):
    # Nothing to compute: OK, no launch, NULL pointers allowed.
    assert _fwd(lib, B=0, value=None, loc=None, attn=None, out=None) == OK
    assert _fwd(lib, Lq=0, loc=None, attn=None, out=None) == OK
    assert _fwd(lib, M=0, value=None, loc=None, attn=None, out=None) == OK


def test_backward_argument_errors(lib):
    # bfloat16 only on the scratch-free path; unknown dtype codes are refused.
    assert _bwd(lib, dtype=1, ws=FAKE, ws_bytes=1 << 40) == UNSUP
    assert _bwd(lib, dtype=2) == UNSUP
    p = [FAKE] * 9
    p[0] = FAKE + 4                                # bfloat16 value: 8-byte alignment
    assert _bwd(lib, dtype=1, ptrs=p) == MISAL
    p = [FAKE] * 9
    p[5] = FAKE + 2                                # bfloat16 grad_output
    assert _bwd(lib, dtype=1, ptrs=p) == MISAL
    assert _bwd(lib, D=260) == UNSUP               # at most 256 channels per head
    assert _bwd(lib, D=132, ws=FAKE, ws_bytes=1 << 40) == UNSUP  # cell-sorted: at most 128
    assert _bwd(lib, D=6) == UNSUP
    assert _bwd(lib, S=-3) == BAD
    p = [FAKE] * 9
    p[6] = None                                    # grad_value
    assert _bwd(lib, ptrs=p) == NULLP
    p = [FAKE] * 9
    p[6] = FAKE + 4
    assert _bwd(lib, ptrs=p) == MISAL
    p = [FAKE] * 9
    p[5] = FAKE + 8                                # grad_output
    assert _bwd(lib, ptrs=p) == MISAL
    p = [FAKE] * 9
    p[7] = FAKE + 4                                # grad_sampling_locations
    assert _bwd(lib, ptrs=p) == MISAL
    assert _bwd(lib, B=0, ptrs=[None] * 9) == OK  # nothing to write at all
    # A workspace that is too small, or misaligned, is rejected before any launch.
    st, need = _ws_size(lib)
    assert st == OK and need > 0
    assert _bwd(lib, ws=FAKE, ws_bytes=need - 1) == WORKSPACE
    assert _bwd(lib, ws=FAKE + 16, ws_bytes=need) == MISAL


def test_workspace_size(lib):
    st, need = _ws_size(lib, B=4, S=19947, M=8, D=32, Lq=19947, L=4, K=4)
    assert st == OK
    points = 4 * 19947 * 8 * 16
    chunks = -(-19947 * 4 // 16384)
    keys = 4 * 8 * (2 * 19947 + 2 * 4)
    counts = keys * chunks
    # slot 4 B + record 16 B + record key 4 B per point; one counter per (chunk, cell)
    # and one total per cell.
    fixed = 24 * points + 4 * counts + 4 * keys
    assert fixed <= need < fixed + 64 * 1024
    assert _ws_size(lib, B=-1)[0] == BAD
    assert _ws_size(lib, B=1 << 14, Lq=1 << 14, M=8)[0] == UNSUP  # 32-bit point ids overflow
    assert lib.msda_backward_workspace_size(1, 80, 2, 8, 80, 2, 2, None) == NULLP


def _ffwd(lib, R=2, dtype=0, B=1, S=80, M=2, D=8, Lq=80, L=2, K=2, ptrs=None):
    p = [FAKE] * 7 if ptrs is None else ptrs
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.msda_fused_forward(B, S, M, D, Lq, L, K, R, dtype, *[v(x) for x in p], None)


def _fbwd(lib, R=2, dtype=0, B=1, S=80, M=2, D=8, Lq=80, L=2, K=2, ptrs=None):
    p = [FAKE] * 11 if ptrs is None else ptrs
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.msda_fused_backward(B, S, M, D, Lq, L, K, R, dtype, *[v(x) for x in p], None)


def test_fused_argument_errors(lib):
    # Reference points must have 2 or 4 components.
    for R in (0, 1, 3, 5):
        assert _ffwd(lib, R=R) == BAD
        assert _fbwd(lib, R=R) == BAD
    # Shared size rules of the core.
    assert _ffwd(lib, B=-1) == BAD
    assert _ffwd(lib, L=17) == UNSUP and _fbwd(lib, K=65) == UNSUP
    assert _ffwd(lib, D=6) == UNSUP
    # Both passes take float32 or bfloat16 value; the backward needs D <= 128.
    assert _fbwd(lib, dtype=2) == UNSUP
    assert _fbwd(lib, D=132) == UNSUP
    for i in (0, 6):                        # bfloat16 value / grad_output: 8-byte aligned
        ptrs = [FAKE] * 11
        ptrs[i] = FAKE + 4
        assert _fbwd(lib, dtype=1, ptrs=ptrs) == MISAL, i
    # Every required pointer; grad_reference_points (the 11th) may be NULL.
    for i in range(7):
        ptrs = [FAKE] * 7
        ptrs[i] = None
        assert _ffwd(lib, ptrs=ptrs) == NULLP, i
    for i in range(10):
        ptrs = [FAKE] * 11
        ptrs[i] = None
        assert _fbwd(lib, ptrs=ptrs) == NULLP, i
    # Alignment: offsets (index 4) need 8 bytes, value 16, logits 4.
    for i, off in ((0, 8), (4, 4), (5, 2), (6, 8)):
        ptrs = [FAKE] * 7
        ptrs[i] = FAKE + off
        assert _ffwd(lib, ptrs=ptrs) == MISAL, i
    ptrs = [FAKE] * 11
    ptrs[8] = FAKE + 4                      # grad_sampling_offsets
    assert _fbwd(lib, ptrs=ptrs) == MISAL
    ptrs = [FAKE] * 11
    ptrs[10] = FAKE + 2                     # grad_reference_points
    assert _fbwd(lib, ptrs=ptrs) == MISAL
    # Empty problems launch nothing.
    assert _ffwd(lib, Lq=0) == OK
    assert _fbwd(lib, B=0) == OK


def _dbwd(lib, B=1, S=80, M=2, D=8, Lq=80, L=2, K=2, dtype=0, ptrs=None, ws=FAKE,
          ws_bytes=1 << 40):
    p = [FAKE] * 9 if ptrs is None else ptrs
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.msda_backward_deterministic(B, S, M, D, Lq, L, K, dtype, *[v(x) for x in p],
                                           v(ws), ws_bytes, None)


def test_deterministic_backward_arguments(lib):
    n = ctypes.c_size_t(0)
    assert lib.msda_backward_deterministic_workspace_size(4, 19947, 8, 32, 19947, 4, 4,
                                                          ctypes.byref(n)) == OK
    # 8 bytes per grad_value element plus an 8 KB header.
    assert n.value == 8192 + 8 * 4 * 19947 * 8 * 32
    assert lib.msda_backward_deterministic_workspace_size(-1, 1, 1, 4, 1, 1, 1,
                                                          ctypes.byref(n)) == BAD
    assert lib.msda_backward_deterministic_workspace_size(1, 1, 1, 4, 1, 1, 1, None) == NULLP
    # Every call below fails validation before any launch.
    assert _dbwd(lib, ws=None) == NULLP                 # the workspace is required
    need = 8192 + 8 * 80 * 2 * 8
    assert _dbwd(lib, ws_bytes=need - 1) == WORKSPACE
    assert _dbwd(lib, ws=FAKE + 16) == MISAL
    assert _dbwd(lib, dtype=2) == UNSUP
    assert _dbwd(lib, D=132) == UNSUP
    assert _dbwd(lib, D=6) == UNSUP
    p = [FAKE] * 9
    p[6] = None                                         # grad_value
    assert _dbwd(lib, ptrs=p) == NULLP
    p = [FAKE] * 9
    p[5] = FAKE + 4                                     # float32 grad_output: 16-byte
    assert _dbwd(lib, ptrs=p) == MISAL
    p = [FAKE] * 9
    p[0] = FAKE + 4                                     # bfloat16 value: 8-byte
    assert _dbwd(lib, dtype=1, ptrs=p) == MISAL
    assert _dbwd(lib, B=0, ptrs=[None] * 9, ws=None) == OK


@pytest.mark.parametrize("entry", ["msda_output_projection", "msda_output_projection_f32"])
def test_output_projection_arguments(lib, entry):
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    fn = getattr(lib, entry)

    def proj(rows=128, c_in=256, c_out=256, x=FAKE, w=FAKE, b=FAKE, y=FAKE):
        return fn(rows, c_in, c_out, v(x), v(w), v(b), v(y), None)

    # Every call below fails validation before any launch.
    assert proj(rows=-1) == BAD
    assert proj(c_in=12) == UNSUP and proj(c_in=0) == UNSUP and proj(c_in=4104) == UNSUP
    assert proj(c_out=8) == UNSUP and proj(c_out=24) == UNSUP and proj(c_out=272) == UNSUP
    assert proj(rows=2**31 - 128) == UNSUP  # past the TMA's 32-bit row coordinates
    assert proj(x=None) == NULLP and proj(w=None) == NULLP and proj(y=None) == NULLP
    assert proj(x=FAKE + 8) == MISAL and proj(w=FAKE + 4) == MISAL and proj(y=FAKE + 8) == MISAL
    assert proj(b=FAKE + 2) == MISAL
    assert proj(rows=0, x=None, w=None, b=None, y=None) == OK
    assert lib.msda_output_projection_check(None) == NULLP


def test_binding_rejects_cpu_tensors_and_bad_ranks():
    """The binding validates before any CUDA call: CPU tensors are refused (there
    is no CPU path) and the projection's operands must have the right ranks."""
    import torch
    x = torch.zeros(4, 8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding.output_projection(x, torch.zeros(16, 8))
    with pytest.raises(ValueError):
        binding.output_projection(torch.zeros(()), torch.zeros(16, 8))
    with pytest.raises(ValueError):
        binding.output_projection(x, torch.zeros(16))
    with pytest.raises(ValueError, match="weight must be"):
        binding.output_projection(x, torch.zeros(16, 4))
    v = torch.zeros(1, 5, 2, 4)
    loc = torch.zeros(1, 3, 2, 1, 1, 2)
    a = torch.zeros(1, 3, 2, 1, 1)
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding.forward(v, torch.tensor([[1, 5]]), torch.tensor([0]), loc, a)


def test_noalloc_argument_errors(lib):
    """msda_backward_noalloc refuses, before any device call, a bfloat16 value
    (its cell-sorted path is float32 only) and sizes whose scratch would not fit
    the library's fixed array."""
    ptrs = [ctypes.c_void_p(FAKE)] * 9
    tiny = (1, 80, 2, 8, 80, 2, 2)
    assert lib.msda_backward_noalloc(*tiny, 1, *ptrs, None) == UNSUP
    assert lib.msda_backward_noalloc(*tiny, 2, *ptrs, None) == UNSUP
    big = (4, 19947, 8, 32, 19947, 4, 4)
    st, need = ctypes.c_int(0), ctypes.c_size_t(0)
    assert lib.msda_backward_workspace_size(*big, ctypes.byref(need)) == OK
    assert need.value > 32 << 20
    assert lib.msda_backward_noalloc(*big, 0, *ptrs, None) == WORKSPACE
