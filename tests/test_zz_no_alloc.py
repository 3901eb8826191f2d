"""flashmask_fwd_noalloc: the forward for callers that cannot allocate device
memory while they run (a server that reserved its whole budget at start-up,
a plugin whose host framework owns the allocator).  Its scratch is a static
device array inside the library instead of a caller-provided workspace.

These tests call the new entry point through the C ABI (ctypes, no binding
helper) and compare it with the regular entry point, flashmask_fwd, on two
calls in a row with different problems -- the second call must not be
affected by what the first left in the shared array.  Tolerance: the one the
other parity tests use (|err| <= 2e-2 + 2^-8 |ref| for O, <= 1e-3 for LSE,
-inf matched exactly); the two paths run the same kernels, so in practice
they agree bit for bit.

The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import column_sparse_masked_b200 as fm
from column_sparse_masked_b200._binding import _Dims

from _parity import make_case

pytestmark = pytest.mark.gpu

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


def _close(o, lse, ro, rl):
    err = (o.float() - ro.float()).abs()
    assert (err <= 2e-2 + 2.0 ** -8 * ro.float().abs()).all(), f"O max err {err.max().item()}"
    assert torch.equal(torch.isneginf(lse), torch.isneginf(rl))
    fin = torch.isfinite(rl)
    assert (lse[fin] - rl[fin]).abs().max().item() <= 1e-3 if fin.any() else True


def test_noalloc_forward_matches_workspace_forward_twice():
    lib = _lib()
    cases = [(2, 517, 389, 4, 2, 1, 128, "random", 81),    # ragged tails, GQA, random intervals
             (1, 1000, 1000, 2, 2, 1, 64, "doc", 82)]     # different shape and mask family
    for case in cases:
        q, k, v, do, masks = make_case(*case)
        q, k, v = q.cuda(), k.cuda(), v.cuda()
        masks = [m.cuda() for m in masks]
        o, lse = _noalloc_fwd(lib, q, k, v, masks)
        ro, rl = fm.fwd(q, k, v, *masks)
        torch.cuda.synchronize()
        assert fm.get_status() == 0
        _close(o, lse, ro, rl)


def test_noalloc_rejects_problems_beyond_the_scratch():
    lib = _lib()
    lib.flashmask_strerror.restype = ctypes.c_char_p
    dims = _Dims(4, 8, 8, 8, 1 << 18, 1 << 18, 128)  # lists alone need far more than 16 MiB
    rc = lib.flashmask_fwd_noalloc(None, None, None, None, None, None, None, ctypes.c_float(0.0),
                                   ctypes.byref(dims), None, None, None)
    assert rc == ERR_TOO_LARGE
    assert b"FLASHMASK_NOALLOC_SCRATCH_BYTES" in lib.flashmask_strerror(rc)
