"""flashmask_fwd_noalloc: the forward for callers that cannot allocate device
memory while they run (a server that reserved its whole budget at start-up,
a plugin whose host framework owns the allocator).  Its scratch is a static
device array inside the library instead of a caller-provided workspace.

These tests call the new entry point through the C ABI (ctypes, no binding
helper) and compare it with the regular entry point, flashmask_fwd, on calls
in a row -- a later call must not be affected by what an earlier one left in
the shared array:
  - two problems of different shapes;
  - two problems of the SAME shape, the first with no masked pair (every
    tile in every work list), the second a sparse document mask, so that
    stale work lists of the first would be read back if the second did not
    rewrite them.
Both paths run the same deterministic kernels on the same inputs, so the
outputs must be equal bit for bit; one case is also checked against the
oracle at the parity tolerance (|err| <= 2e-2 + 2^-8 |ref| for O, <= 1e-3 for
LSE, -inf matched exactly).  Repeated calls must leave the device's free
memory and torch's allocator untouched.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import column_sparse_masked_b200 as fm
from column_sparse_masked_b200._binding import _Dims

from _parity import check_lse, check_out, make_case

NOALLOC_SCRATCH_BYTES = 16 << 20

ERR_TOO_LARGE = -8


def _lib():
    lib = fm.load_library()
    fn = lib.flashmask_fwd_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p]
    return lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_fwd(lib, q, k, v, masks):
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    dims = _Dims(B, Hq, Hkv, masks[0].shape[1], Nq, Nk, d)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, Nq, dtype=torch.float32, device=q.device)
    rc = lib.flashmask_fwd_noalloc(_p(q), _p(k), _p(v), *[_p(m) for m in masks], ctypes.c_float(0.0),
                                   ctypes.byref(dims), _p(o), _p(lse),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, lib.flashmask_strerror(rc)
    return o, lse


def _run_pair(lib, case):
    q, k, v, do, masks = make_case(*case)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    mg = [m.cuda() for m in masks]
    o, lse = _noalloc_fwd(lib, qg, kg, vg, mg)
    ro, rl = fm.fwd(qg, kg, vg, *mg)
    torch.cuda.synchronize()
    assert fm.get_status() == 0
    assert torch.equal(o, ro) and torch.equal(lse, rl), "no-alloc forward differs from flashmask_fwd"
    return (q, k, v, masks), o, lse


@pytest.mark.gpu
def test_noalloc_forward_matches_workspace_forward_twice(oracle_mod):
    lib = _lib()
    cases = [(2, 517, 389, 4, 2, 1, 128, "random", 81),    # ragged tails, GQA, random intervals
             (1, 1000, 1000, 2, 2, 1, 64, "doc", 82)]     # different shape and mask family
    for i, case in enumerate(cases):
        (q, k, v, masks), o, lse = _run_pair(lib, case)
        if i == 0:
            ro, rl = oracle_mod.attention_forward(q, k, v, *masks)
            check_out("O(no-alloc)", o, ro, case="noalloc")
            check_lse(lse, rl, case="noalloc")


@pytest.mark.gpu
def test_noalloc_same_shape_dense_then_sparse():
    lib = _lib()
    _run_pair(lib, (1, 1024, 1024, 4, 2, 1, 128, "none", 83))   # every tile listed
    _run_pair(lib, (1, 1024, 1024, 4, 2, 1, 128, "doc", 84))    # short lists, same offsets
    _run_pair(lib, (1, 1024, 1024, 4, 2, 1, 128, "causal", 85))


@pytest.mark.gpu
def test_noalloc_calls_allocate_nothing():
    lib = _lib()
    q, k, v, do, masks = make_case(1, 700, 700, 4, 2, 1, 128, "random", 86)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    masks = [m.cuda() for m in masks]
    B, Nq, Hq, d = q.shape
    dims = _Dims(B, Hq, k.shape[2], 1, Nq, k.shape[1], d)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, Nq, dtype=torch.float32, device=q.device)
    args = [_p(q), _p(k), _p(v), *[_p(m) for m in masks], ctypes.c_float(0.0), ctypes.byref(dims), _p(o), _p(lse),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)]
    assert lib.flashmask_fwd_noalloc(*args) == 0  # first call on the device: the array's address lookup
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(5):
        assert lib.flashmask_fwd_noalloc(*args) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"
    assert fm.get_status() == 0


def _fwd_ws(lib, n):
    lib.flashmask_fwd_workspace_size.restype = ctypes.c_size_t
    lib.flashmask_fwd_workspace_size.argtypes = [ctypes.c_void_p]
    dims = _Dims(1, 32, 8, 1, n, n, 128)
    return int(lib.flashmask_fwd_workspace_size(ctypes.byref(dims)))


def test_noalloc_limit_boundary_cpu():
    """CPU only: the documented example (one 131072-token sequence, one mask head, 32 q-heads)
    fits the 16 MiB array; the largest fitting length (multiple of 128) is found and one tile
    more is rejected with FLASHMASK_ERR_TOO_LARGE before any device access."""
    from column_sparse_masked_b200 import build

    build.build()
    lib = _lib()
    assert 0 < _fwd_ws(lib, 131072) <= NOALLOC_SCRATCH_BYTES
    lo, hi = 131072, 1 << 22  # size(lo) fits, size(hi) does not
    assert _fwd_ws(lib, hi) > NOALLOC_SCRATCH_BYTES
    while hi - lo > 128:
        mid = (lo + hi) // 2 // 128 * 128
        if _fwd_ws(lib, mid) <= NOALLOC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    assert _fwd_ws(lib, lo) <= NOALLOC_SCRATCH_BYTES < _fwd_ws(lib, lo + 128)
    dims = _Dims(1, 32, 8, 1, lo + 128, lo + 128, 128)
    rc = lib.flashmask_fwd_noalloc(None, None, None, None, None, None, None, ctypes.c_float(0.0),
                                   ctypes.byref(dims), None, None, None)
    assert rc == ERR_TOO_LARGE


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_the_scratch():
    lib = _lib()
    lib.flashmask_strerror.restype = ctypes.c_char_p
    dims = _Dims(4, 8, 8, 8, 1 << 18, 1 << 18, 128)  # lists alone need far more than 16 MiB
    rc = lib.flashmask_fwd_noalloc(None, None, None, None, None, None, None, ctypes.c_float(0.0),
                                   ctypes.byref(dims), None, None, None)
    assert rc == ERR_TOO_LARGE
    assert b"FLASHMASK_NOALLOC_SCRATCH_BYTES" in lib.flashmask_strerror(rc)
