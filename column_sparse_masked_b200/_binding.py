"""ctypes marshalling for libflashmask.so (see include/flashmask.h)."""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libflashmask.so"
_lib = None

# Entry points of include/flashmask.h: name -> (restype, argtypes)
_P = ctypes.c_void_p
_DIMS = ctypes.c_void_p  # const flashmask_dims*
_SIGS = {
    "flashmask_fwd_workspace_size": (ctypes.c_size_t, [_DIMS]),
    "flashmask_bwd_workspace_size": (ctypes.c_size_t, [_DIMS]),
    "flashmask_fwd": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_float, _DIMS, _P, _P, _P,
                                     ctypes.c_size_t, _P]),
    "flashmask_bwd": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_float, _DIMS, _P, _P, _P,
                                     _P, ctypes.c_size_t, _P]),
    "flashmask_classify": (ctypes.c_int, [_P, _P, _P, _P, _DIMS, _P, _P, ctypes.c_size_t, _P]),
    "flashmask_localize": (ctypes.c_int, [_P, _P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P]),
    "flashmask_localize_multi": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P, _P, ctypes.c_int32, _P]),
    "flashmask_count_unmasked": (ctypes.c_int, [_P, _P, _P, _P, _DIMS, _P, _P]),
    "flashmask_tile_costs": (ctypes.c_int, [_P, _P, _P, _P, _DIMS, _P, _P]),
    "flashmask_merge_partials": (ctypes.c_int, [_P, _P, ctypes.c_int32, _DIMS, _P, _P, _P]),
    "flashmask_balance_chunks": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, _P, _P]),
    "flashmask_set_max_ctas": (ctypes.c_int, [ctypes.c_int32]),
    "flashmask_set_bwd_mode": (ctypes.c_int, [ctypes.c_int32]),
    "flashmask_get_bwd_mode": (ctypes.c_int, []),
    "flashmask_set_fwd_pairing": (ctypes.c_int, [ctypes.c_int32]),
    "flashmask_get_fwd_pairing": (ctypes.c_int, []),
    "flashmask_get_timeout_info": (ctypes.c_int, [_P]),
    "flashmask_get_status": (ctypes.c_int, []),
    "flashmask_set_wait_limit_ns": (None, [ctypes.c_int64]),
    "flashmask_test_wait_timeout": (ctypes.c_int, [ctypes.c_int64, _P]),
    "flashmask_profiler_enable": (ctypes.c_int, [ctypes.c_int]),
    "flashmask_profiler_read": (ctypes.c_int, [_P, _P]),
    "flashmask_launch_count": (ctypes.c_int64, []),
    "flashmask_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "flashmask_version": (ctypes.c_int, []),
}


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Hq", "Hkv", "Hm", "Nq", "Nk", "d")]


class FlashMaskError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = load_library().flashmask_strerror(code).decode()
        super().__init__(f"{where}: {msg} (code {code})")
        self.code = code


def lib_path() -> str:
    """The library this process loads: libflashmask.so, or the checks build
    (libflashmask_checks.so) when FLASHMASK_LIBRARY=checks."""
    name = "libflashmask_checks.so" if os.environ.get("FLASHMASK_LIBRARY") == "checks" else _LIB_NAME
    return os.path.join(_HERE, name)


def load_library():
    """Loads libflashmask.so from the package directory; raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python column_sparse_masked_b200/build.py`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def version() -> int:
    return int(load_library().flashmask_version())


def _check(code: int, where: str):
    if code != 0:
        raise FlashMaskError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dims(B, Hq, Hkv, Hm, Nq, Nk, d) -> _Dims:
    return _Dims(int(B), int(Hq), int(Hkv), int(Hm), int(Nq), int(Nk), int(d))


def _need_cuda(name: str, t: torch.Tensor, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _masks(lts, lte, uts, ute):
    vecs = [lts, lte, uts, ute]
    for n, x in zip(("lts", "lte", "uts", "ute"), vecs):
        if x is not None:
            _need_cuda(n, x, torch.int32)
    ref = next((x for x in vecs if x is not None), None)
    Hm = ref.shape[1] if ref is not None else 1
    return vecs, Hm


def _shaped(name: str, t, shape, dtype):
    """Checks type, dtype and shape of an argument (any device); the kernels trust these sizes."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _qkv_shapes(q, k, v):
    for n, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dim() != 4:
            raise ValueError(f"{n} must be a 4-D tensor [B, N, H, d]")
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    _shaped("q", q, (B, Nq, Hq, d), torch.bfloat16)
    _shaped("k", k, (B, Nk, Hkv, d), torch.bfloat16)
    _shaped("v", v, (B, Nk, Hkv, d), torch.bfloat16)
    return B, Nq, Hq, d, Nk, Hkv


def _mask_shapes(lts, lte, uts, ute, B: int, Nk: int) -> int:
    vecs = [lts, lte, uts, ute]
    ref = next((x for x in vecs if x is not None), None)
    if ref is not None and (not isinstance(ref, torch.Tensor) or ref.dim() != 3):
        raise ValueError("mask vectors must be 3-D tensors [B, Hm, Nk]")
    Hm = ref.shape[1] if ref is not None else 1
    for n, x in zip(("lts", "lte", "uts", "ute"), vecs):
        if x is not None:
            _shaped(n, x, (B, Hm, Nk), torch.int32)
    return Hm


def _on_device(dev, named):
    """Every tensor on the CUDA device `dev` and contiguous."""
    for n, t in named:
        if t is None:
            continue
        if not t.is_cuda:
            raise TypeError(f"{n} must be a CUDA tensor")
        if t.device != dev:
            raise ValueError(f"{n} is on {t.device}, expected {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")


def _ws_bytes(ws: torch.Tensor) -> int:
    return ws.numel() * ws.element_size()


def workspace_size(kind: str, B, Hq, Hkv, Hm, Nq, Nk, d) -> int:
    lib = load_library()
    dm = _dims(B, Hq, Hkv, Hm, Nq, Nk, d)
    fn = lib.flashmask_fwd_workspace_size if kind == "fwd" else lib.flashmask_bwd_workspace_size
    return int(fn(ctypes.byref(dm)))


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, lts=None, lte=None, uts=None, ute=None,
        scale: Optional[float] = None, out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
        workspace: Optional[torch.Tensor] = None):
    """Masked attention forward -> (o [B,Nq,Hq,d] bf16, lse [B,Hq,Nq] fp32)."""
    lib = load_library()
    B, Nq, Hq, d, Nk, Hkv = _qkv_shapes(q, k, v)
    Hm = _mask_shapes(lts, lte, uts, ute, B, Nk)
    vecs = [lts, lte, uts, ute]
    if out is not None:
        o, lse = out
        _shaped("o", o, (B, Nq, Hq, d), torch.bfloat16)
        _shaped("lse", lse, (B, Hq, Nq), torch.float32)
    _on_device(q.device, [("q", q), ("k", k), ("v", v)] + list(zip(("lts", "lte", "uts", "ute"), vecs)))
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(B, Hq, Nq, dtype=torch.float32, device=q.device)
    dm = _dims(B, Hq, Hkv, Hm, Nq, Nk, d)
    need = int(lib.flashmask_fwd_workspace_size(ctypes.byref(dm)))
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _on_device(q.device, [("o", o), ("lse", lse), ("workspace", ws)])
    rc = lib.flashmask_fwd(_ptr(q), _ptr(k), _ptr(v), *[_ptr(x) for x in vecs], ctypes.c_float(scale or 0.0),
                           ctypes.byref(dm), _ptr(o), _ptr(lse), _ptr(ws), ctypes.c_size_t(_ws_bytes(ws)),
                           _stream(q.device))
    _check(rc, "flashmask_fwd")
    return o, lse


def bwd(q, k, v, o, lse, dout, lts=None, lte=None, uts=None, ute=None, scale: Optional[float] = None,
        out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
        workspace: Optional[torch.Tensor] = None):
    """Masked attention backward of sum(O * dO) -> (dq, dk, dv), bf16."""
    lib = load_library()
    B, Nq, Hq, d, Nk, Hkv = _qkv_shapes(q, k, v)
    _shaped("o", o, (B, Nq, Hq, d), torch.bfloat16)
    _shaped("dout", dout, (B, Nq, Hq, d), torch.bfloat16)
    _shaped("lse", lse, (B, Hq, Nq), torch.float32)
    Hm = _mask_shapes(lts, lte, uts, ute, B, Nk)
    vecs = [lts, lte, uts, ute]
    if out is not None:
        dq, dk, dv = out
        _shaped("dq", dq, (B, Nq, Hq, d), torch.bfloat16)
        _shaped("dk", dk, (B, Nk, Hkv, d), torch.bfloat16)
        _shaped("dv", dv, (B, Nk, Hkv, d), torch.bfloat16)
    _on_device(q.device, [("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse), ("dout", dout)]
               + list(zip(("lts", "lte", "uts", "ute"), vecs)))
    if out is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dm = _dims(B, Hq, Hkv, Hm, Nq, Nk, d)
    need = int(lib.flashmask_bwd_workspace_size(ctypes.byref(dm)))
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _on_device(q.device, [("dq", dq), ("dk", dk), ("dv", dv), ("workspace", ws)])
    rc = lib.flashmask_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), *[_ptr(x) for x in vecs],
                           ctypes.c_float(scale or 0.0), ctypes.byref(dm), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                           ctypes.c_size_t(_ws_bytes(ws)), _stream(q.device))
    _check(rc, "flashmask_bwd")
    return dq, dk, dv


def classify(lts, lte, uts, ute, Nq: int, Nk: Optional[int] = None, Hq: int = 1) -> torch.Tensor:
    """Tile classes uint8 [B, Hm, ceil(Nq/128), ceil(Nk/128)]: 0 skip, 1 partial, 2 full."""
    lib = load_library()
    vecs, Hm = _masks(lts, lte, uts, ute)
    ref = next(x for x in vecs if x is not None)
    B, Nk = ref.shape[0], (ref.shape[2] if Nk is None else Nk)
    Hq = max(Hq, Hm)
    dm = _dims(B, Hq, 1, Hm, Nq, Nk, 128)
    nqt, nkt = -(-Nq // 128), -(-Nk // 128)
    cls = torch.empty(B, Hm, nqt, nkt, dtype=torch.uint8, device=ref.device)
    ws = _workspace(lib.flashmask_fwd_workspace_size(ctypes.byref(dm)), ref.device)
    rc = lib.flashmask_classify(*[_ptr(x) for x in vecs], ctypes.byref(dm), _ptr(cls), _ptr(ws),
                                ctypes.c_size_t(ws.numel()), _stream(ref.device))
    _check(rc, "flashmask_classify")
    return cls


def localize(x: torch.Tensor, a: int, b: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Clip-shift-max of boundary values onto the query chunk [a, b)."""
    lib = load_library()
    _need_cuda("x", x, torch.int32)
    out = torch.empty_like(x) if out is None else out
    rc = lib.flashmask_localize(_ptr(x), _ptr(out), ctypes.c_int64(x.numel()), int(a), int(b), _stream(x.device))
    _check(rc, "flashmask_localize")
    return out


def localize_multi(x: torch.Tensor, chunks: Sequence[Tuple[int, int]], out: Optional[torch.Tensor] = None):
    """Localisation onto increasing disjoint chunks concatenated in order."""
    lib = load_library()
    _need_cuda("x", x, torch.int32)
    out = torch.empty_like(x) if out is None else out
    a = (ctypes.c_int32 * max(1, len(chunks)))(*[int(c[0]) for c in chunks])
    b = (ctypes.c_int32 * max(1, len(chunks)))(*[int(c[1]) for c in chunks])
    rc = lib.flashmask_localize_multi(_ptr(x), _ptr(out), ctypes.c_int64(x.numel()), a, b, len(chunks),
                                      _stream(x.device))
    _check(rc, "flashmask_localize_multi")
    return out


def count_unmasked(lts, lte, uts, ute, Nq: int, Hq: int) -> int:
    """Unmasked (i, j) pairs over all batches and Hq query heads (closed form on the GPU)."""
    lib = load_library()
    vecs, Hm = _masks(lts, lte, uts, ute)
    ref = next(x for x in vecs if x is not None)
    B, Nk = ref.shape[0], ref.shape[2]
    dm = _dims(B, Hq, 1, Hm, Nq, Nk, 128)
    out = torch.zeros(1, dtype=torch.int64, device=ref.device)
    rc = lib.flashmask_count_unmasked(*[_ptr(x) for x in vecs], ctypes.byref(dm), _ptr(out), _stream(ref.device))
    _check(rc, "flashmask_count_unmasked")
    return int(out.item())


def tile_costs(lts, lte, uts, ute, Nq: int, Hq: int) -> torch.Tensor:
    """Unmasked pairs of each 128-row q-tile over batches and Hq query heads (int64 CUDA tensor)."""
    lib = load_library()
    vecs, Hm = _masks(lts, lte, uts, ute)
    ref = next(x for x in vecs if x is not None)
    B, Nk = ref.shape[0], ref.shape[2]
    dm = _dims(B, Hq, 1, Hm, Nq, Nk, 128)
    out = torch.zeros(max(1, -(-int(Nq) // 128)), dtype=torch.int64, device=ref.device)
    rc = lib.flashmask_tile_costs(*[_ptr(x) for x in vecs], ctypes.byref(dm), _ptr(out), _stream(ref.device))
    _check(rc, "flashmask_tile_costs")
    return out[: -(-int(Nq) // 128)]


def merge_partials(o_parts: Sequence[torch.Tensor], lse_parts: Sequence[torch.Tensor]):
    """Attention over the union of disjoint key sets from per-set results (o_c, lse_c):
    lse = ln sum exp(lse_c), o = sum exp(lse_c - lse) o_c, per row.  Returns (o, lse)."""
    lib = load_library()
    n = len(o_parts)
    if n < 1 or n != len(lse_parts):
        raise ValueError("need as many lse parts as o parts (at least one)")
    B, Nq, Hq, d = o_parts[0].shape
    for i, (oc, lc) in enumerate(zip(o_parts, lse_parts)):
        _shaped(f"o_parts[{i}]", oc, (B, Nq, Hq, d), torch.bfloat16)
        _shaped(f"lse_parts[{i}]", lc, (B, Hq, Nq), torch.float32)
    _on_device(o_parts[0].device, [(f"o{i}", t) for i, t in enumerate(o_parts)] +
               [(f"l{i}", t) for i, t in enumerate(lse_parts)])
    o = torch.empty_like(o_parts[0])
    lse = torch.empty_like(lse_parts[0])
    op = (ctypes.c_void_p * n)(*[t.data_ptr() for t in o_parts])
    lp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in lse_parts])
    dm = _dims(B, Hq, 1, 1, Nq, 0, d)
    rc = lib.flashmask_merge_partials(op, lp, n, ctypes.byref(dm), _ptr(o), _ptr(lse), _stream(o.device))
    _check(rc, "flashmask_merge_partials")
    return o, lse


def set_max_ctas(n: int) -> None:
    """Caps the attention kernels' persistent grid at n CTAs (0 = one per SM); for tests."""
    _check(load_library().flashmask_set_max_ctas(int(n)), "flashmask_set_max_ctas")


BWD_FUSED, BWD_SPLIT = 0, 1
_BWD_MODES = {"fused": BWD_FUSED, "split": BWD_SPLIT}


def set_bwd_mode(mode) -> None:
    """Backward mode of later ``bwd`` calls: "fused" (default; one key-stationary pass, dQ by fp32
    reductions) or "split" (separate dK/dV and dQ kernels, bit-reproducible)."""
    m = _BWD_MODES.get(mode, mode)
    _check(load_library().flashmask_set_bwd_mode(int(m)), "flashmask_set_bwd_mode")


def get_bwd_mode() -> str:
    m = int(load_library().flashmask_get_bwd_mode())
    return {v: k for k, v in _BWD_MODES.items()}[m]


def set_fwd_pairing(on: bool) -> None:
    """Forward items of later ``fwd`` calls: one q-tile of two q-heads that share a KV head (True,
    the default; used when the shape has one mask head and an even GQA group) or two q-tiles of one
    q-head (False).  Outputs are bit-identical either way."""
    _check(load_library().flashmask_set_fwd_pairing(1 if on else 0), "flashmask_set_fwd_pairing")


def get_fwd_pairing() -> bool:
    return bool(load_library().flashmask_get_fwd_pairing())


def balance_chunks(costs: Sequence[int], parts: int) -> Tuple[List[int], int]:
    """Splits q-tiles into ``parts`` contiguous chunks with the smallest possible largest cost.

    ``costs`` holds the work of each q-tile (its unmasked pairs); returns ``(bounds, max_cost)``
    with chunk p = tiles ``[bounds[p], bounds[p + 1])``.  Host computation in the library
    (``flashmask_balance_chunks``).
    """
    lib = load_library()
    c = (ctypes.c_int64 * max(1, len(costs)))(*[int(x) for x in costs])
    bounds = (ctypes.c_int32 * (max(0, int(parts)) + 1))()
    best = ctypes.c_int64(0)
    rc = lib.flashmask_balance_chunks(c, len(costs), int(parts), bounds, ctypes.byref(best))
    _check(rc, "flashmask_balance_chunks")
    return [int(x) for x in bounds], int(best.value)


def get_status() -> int:
    """Synchronises the device; returns and clears the kernels' status word."""
    return int(load_library().flashmask_get_status())


ERR_BOUNDS = -9

_TIMEOUT_KERNELS = ("forward", "backward key side", "backward query side", "wait self-test", "fused backward")


def get_timeout_info() -> dict:
    """The bounded wait behind the first timeout since the status word was last cleared."""
    info = (ctypes.c_int32 * 5)()
    _check(load_library().flashmask_get_timeout_info(info), "flashmask_get_timeout_info")
    k = int(info[0])
    return {"kernel": _TIMEOUT_KERNELS[k] if 0 <= k < len(_TIMEOUT_KERNELS) else k,
            "barrier_offset": int(info[1]), "parity": int(info[2]), "block": int(info[3]), "thread": int(info[4])}


def set_wait_limit_ns(ns: int) -> None:
    load_library().flashmask_set_wait_limit_ns(ctypes.c_int64(int(ns)))


def test_wait_timeout(limit_ns: int, device=None) -> None:
    """Launches the bounded-wait self test (one CTA waits on a barrier nothing arrives on)."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check(load_library().flashmask_test_wait_timeout(ctypes.c_int64(int(limit_ns)), _stream(dev)),
           "flashmask_test_wait_timeout")


def profiler_enable(on: bool = True) -> None:
    """Brackets every attention-kernel launch with CUDA events (for benchmarks)."""
    _check(load_library().flashmask_profiler_enable(1 if on else 0), "flashmask_profiler_enable")


PROFILER_KINDS = ("fwd", "bwd_kv", "bwd_q", "bwd", "bwd_fused", "dq_finalize")


def profiler_read():
    """{'<kind>_ms', '<kind>_launches'} since the last read.  Kinds: fwd; bwd_kv and bwd_q (split
    backward's two kernels, concurrent); bwd (the backward's attention unit: split, the two kernels
    from fork to join; fused, the fused kernel and the dQ finalize); bwd_fused; dq_finalize."""
    n = len(PROFILER_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(load_library().flashmask_profiler_read(ms, cnt), "flashmask_profiler_read")
    out = {}
    for i, k in enumerate(PROFILER_KINDS):
        out[f"{k}_ms"] = ms[i]
        out[f"{k}_launches"] = cnt[i]
    return out


def launch_count() -> int:
    """Kernels launched by the library since process start."""
    return int(load_library().flashmask_launch_count())


class _FlashMaskFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, lts, lte, uts, ute, scale):
        o, lse = fwd(q, k, v, lts, lte, uts, ute, scale)
        ctx.save_for_backward(q, k, v, o, lse, *(x if x is not None else torch.empty(0) for x in (lts, lte, uts, ute)))
        ctx.none = tuple(x is None for x in (lts, lte, uts, ute))
        ctx.scale = scale
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, *m = ctx.saved_tensors
        m = [None if n else x for x, n in zip(m, ctx.none)]
        dq, dk, dv = bwd(q, k, v, o, lse, do.contiguous(), *m, scale=ctx.scale)
        return dq, dk, dv, None, None, None, None, None


def flashmask_attention(q, k, v, lts=None, lte=None, uts=None, ute=None, scale: Optional[float] = None):
    """Autograd-aware masked attention returning O (bf16)."""
    return _FlashMaskFn.apply(q, k, v, lts, lte, uts, ute, scale)
