"""Plain CPU oracle for column-sparse masked attention (FlashMask encoding).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``column_sparse_masked_b200``) never imports it and shares no code with it.

The arithmetic lives in ``flashmask_oracle.c`` (double precision, plain loops,
OpenMP over rows); this module only marshals arrays.  Every function follows
"FlashMask-3 targets masked distributed attention on Hopper GPUs", section
"In-depth insight" (column-wise mask of four query-axis boundary vectors per
key column; clip-shift-max localisation), with the predicate
``masked(i, j) = LTS[j] <= i < LTE[j] or UTS[j] <= i < UTE[j]``.

Inputs given as torch bf16 tensors are widened to float64 exactly.
Layouts: q/o/dO/dq ``[B, Nq, Hq, d]``; k/v/dk/dv ``[B, Nk, Hkv, d]``; the four
mask vectors ``[B, Hm, Nk]`` int32 with Hm in {1, Hq}; q-head h uses KV head
``h // (Hq // Hkv)`` and mask head ``0 if Hm == 1 else h``.

Parity pins: see ``tests/test_oracle_pins.py`` (library special cases, closed
forms, finite differences, brute force) and, for the per-tile costs and the
exhaustive chunk split, ``tests/test_balance.py``; nothing here is unpinned.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
from typing import List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flashmask_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)
_U8 = ctypes.POINTER(ctypes.c_uint8)


def _compile(src: str, out: str) -> None:
    cmd = ["gcc", "-O2", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)


def build_oracle(force: bool = False) -> str:
    """Compiles the C oracle with gcc (OpenMP, portable x86-64-v3 code)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    _compile(_SRC, tmp)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def source() -> str:
    """The C source of the oracle."""
    with open(_SRC) as f:
        return f.read()


def build_variant(c_source: str, out_dir: str) -> str:
    """Compiles another version of the oracle's C source (the tests plant mistakes in a copy to
    show that the pins catch them); returns the path of the shared library."""
    src = os.path.join(out_dir, "oracle_variant.c")
    with open(src, "w") as f:
        f.write(c_source)
    out = os.path.join(out_dir, "liboracle_variant.so")
    _compile(src, out)
    return out


@contextlib.contextmanager
def use_library(path: str):
    """Routes every oracle function through the library at `path` inside the block."""
    global _lib
    saved = _lib
    _lib = _bind(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = saved


def _load():
    global _lib
    if _lib is not None:
        return _lib
    _lib = _bind(ctypes.CDLL(build_oracle()))
    return _lib


def _bind(lib):
    lib.oracle_fwd_head.argtypes = [_D, _I64, ctypes.c_int64, _D, _D, ctypes.c_int64, ctypes.c_int64,
                                    _I32, _I32, _I32, _I32, ctypes.c_double, _D, _D]
    lib.oracle_dq_head.argtypes = [_D, _D, _I64, ctypes.c_int64, _D, _D, ctypes.c_int64, ctypes.c_int64,
                                   _I32, _I32, _I32, _I32, ctypes.c_double, _D]
    lib.oracle_dkdv_head.argtypes = [_D, _D, ctypes.c_int64, _D, _D, ctypes.c_int64, ctypes.c_int64,
                                     _I32, _I32, _I32, _I32, ctypes.c_double, _I64, ctypes.c_int64, _D, _D]
    lib.oracle_classify.argtypes = [_I32, _I32, _I32, _I32, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                    ctypes.c_int64, _U8]
    lib.oracle_localize.argtypes = [_I32, _I32, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]
    lib.oracle_localize_multi.argtypes = [_I32, _I32, ctypes.c_int64, _I32, _I32, ctypes.c_int64]
    lib.oracle_count_unmasked.argtypes = [_I32, _I32, _I32, _I32, ctypes.c_int64, ctypes.c_int64]
    lib.oracle_count_unmasked.restype = ctypes.c_int64
    lib.oracle_mask_row.argtypes = [_I32, _I32, _I32, _I32, ctypes.c_int64, ctypes.c_int64, _U8]
    lib.oracle_tile_costs.argtypes = [_I32, _I32, _I32, _I32, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.POINTER(ctypes.c_int64)]
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------
def _f64(x) -> np.ndarray:
    """Widens a torch tensor (bf16/fp32/fp64) or array to a C-contiguous float64 array."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _mask_arrays(lts, lte, uts, ute, B: int, Nk: int):
    """Returns four int32 arrays [B, Hm, Nk]; a None pair means an empty interval."""
    if lts is None and lte is None:
        ref = uts if uts is not None else ute
        hm = _i32(ref).shape[1] if ref is not None else 1
        lts = np.zeros((B, hm, Nk), np.int32)
        lte = np.zeros((B, hm, Nk), np.int32)
    if uts is None and ute is None:
        hm = _i32(lts).shape[1]
        uts = np.zeros((B, hm, Nk), np.int32)
        ute = np.zeros((B, hm, Nk), np.int32)
    out = [_i32(x) for x in (lts, lte, uts, ute)]
    for x in out:
        if x.ndim != 3 or x.shape[0] != B or x.shape[2] != Nk:
            raise ValueError(f"mask vector shape {x.shape} does not match [B={B}, Hm, Nk={Nk}]")
    return out


def _head_maps(Hq: int, Hkv: int, Hm: int):
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if Hm not in (1, Hq):
        raise ValueError("Hm must be 1 or Hq")
    G = Hq // Hkv
    return (lambda h: h // G), (lambda h: 0 if Hm == 1 else h)


# ----------------------------------------------------------------------------
# public oracle API
# ----------------------------------------------------------------------------
def attention_forward(q, k, v, lts, lte, uts, ute, scale: Optional[float] = None,
                      samples: Optional[Sequence[Tuple[int, int, int]]] = None):
    """Masked softmax attention forward.

    Returns ``(o, lse)``: full ``[B, Nq, Hq, d]`` / ``[B, Hq, Nq]`` float64
    arrays, or, when ``samples`` (a list of ``(b, h, i)``) is given, arrays
    ``[n, d]`` / ``[n]`` for those rows only.
    """
    lib = _load()
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    m4 = _mask_arrays(lts, lte, uts, ute, B, Nk)
    kv_of, m_of = _head_maps(Hq, Hkv, m4[0].shape[1])
    sc = float(scale) if scale else 1.0 / np.sqrt(d)
    if samples is None:
        o = np.zeros((B, Nq, Hq, d))
        lse = np.zeros((B, Hq, Nq))
        groups = {(b, h): None for b in range(B) for h in range(Hq)}
    else:
        samples = [tuple(int(t) for t in s) for s in samples]
        o = np.zeros((len(samples), d))
        lse = np.zeros(len(samples))
        groups = {}
        for n, (b, h, i) in enumerate(samples):
            groups.setdefault((b, h), []).append((n, i))
    kv_cache = {}
    for (b, h), sel in groups.items():
        hk, hm = kv_of(h), m_of(h)
        if (b, hk) not in kv_cache:
            kv_cache = {(b, hk): (_f64(k[b, :, hk, :]), _f64(v[b, :, hk, :]))}
        kb, vb = kv_cache[(b, hk)]
        vecs = [np.ascontiguousarray(x[b, hm]) for x in m4]
        if sel is None:
            qb = _f64(q[b, :, h, :])
            rows = None
            n = Nq
        else:
            idx = np.array([i for _, i in sel], np.int64)
            qb = np.ascontiguousarray(_f64(q[b, :, h, :])[idx]) if len(sel) > 64 else np.ascontiguousarray(
                np.stack([_f64(q[b, i, h, :]) for _, i in sel]))
            rows = idx
            n = len(sel)
        ob = np.zeros((n, d))
        lb = np.zeros(n)
        lib.oracle_fwd_head(_p(qb, _D), _p(rows, _I64) if rows is not None else None, n, _p(kb, _D), _p(vb, _D),
                            Nk, d, *[_p(x, _I32) for x in vecs], sc, _p(ob, _D), _p(lb, _D))
        if sel is None:
            o[b, :, h, :] = ob
            lse[b, h, :] = lb
        else:
            for r, (nidx, _) in enumerate(sel):
                o[nidx] = ob[r]
                lse[nidx] = lb[r]
    return o, lse


def attention_backward_dq(q, k, v, dout, lts, lte, uts, ute, scale: Optional[float] = None,
                          samples: Optional[Sequence[Tuple[int, int, int]]] = None):
    """dQ of the loss sum(O * dO); full ``[B, Nq, Hq, d]`` or ``[n, d]`` for ``samples``."""
    lib = _load()
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    m4 = _mask_arrays(lts, lte, uts, ute, B, Nk)
    kv_of, m_of = _head_maps(Hq, Hkv, m4[0].shape[1])
    sc = float(scale) if scale else 1.0 / np.sqrt(d)
    if samples is None:
        out = np.zeros((B, Nq, Hq, d))
        groups = {(b, h): None for b in range(B) for h in range(Hq)}
    else:
        samples = [tuple(int(t) for t in s) for s in samples]
        out = np.zeros((len(samples), d))
        groups = {}
        for n, (b, h, i) in enumerate(samples):
            groups.setdefault((b, h), []).append((n, i))
    kv_cache = {}
    for (b, h), sel in groups.items():
        hk, hm = kv_of(h), m_of(h)
        if (b, hk) not in kv_cache:
            kv_cache = {(b, hk): (_f64(k[b, :, hk, :]), _f64(v[b, :, hk, :]))}
        kb, vb = kv_cache[(b, hk)]
        vecs = [np.ascontiguousarray(x[b, hm]) for x in m4]
        if sel is None:
            qb, gb, rows, n = _f64(q[b, :, h, :]), _f64(dout[b, :, h, :]), None, Nq
        else:
            idx = np.array([i for _, i in sel], np.int64)
            qb = np.ascontiguousarray(np.stack([_f64(q[b, i, h, :]) for _, i in sel]))
            gb = np.ascontiguousarray(np.stack([_f64(dout[b, i, h, :]) for _, i in sel]))
            rows, n = idx, len(sel)
        res = np.zeros((n, d))
        lib.oracle_dq_head(_p(qb, _D), _p(gb, _D), _p(rows, _I64) if rows is not None else None, n,
                           _p(kb, _D), _p(vb, _D), Nk, d, *[_p(x, _I32) for x in vecs], sc, _p(res, _D))
        if sel is None:
            out[b, :, h, :] = res
        else:
            for r, (nidx, _) in enumerate(sel):
                out[nidx] = res[r]
    return out


def attention_backward_dkdv(q, k, v, dout, lts, lte, uts, ute, scale: Optional[float] = None,
                            samples: Optional[Sequence[Tuple[int, int, int]]] = None):
    """dK, dV of the loss sum(O * dO), summed over the q-heads sharing each KV head.

    ``samples`` is a list of ``(b, hkv, j)`` key columns; returns ``[n, d]``
    arrays.  Without samples, full ``[B, Nk, Hkv, d]`` arrays.
    """
    lib = _load()
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    m4 = _mask_arrays(lts, lte, uts, ute, B, Nk)
    kv_of, m_of = _head_maps(Hq, Hkv, m4[0].shape[1])
    G = Hq // Hkv
    sc = float(scale) if scale else 1.0 / np.sqrt(d)
    if samples is None:
        dk = np.zeros((B, Nk, Hkv, d))
        dv = np.zeros((B, Nk, Hkv, d))
        groups = {(b, hk): None for b in range(B) for hk in range(Hkv)}
    else:
        samples = [tuple(int(t) for t in s) for s in samples]
        dk = np.zeros((len(samples), d))
        dv = np.zeros((len(samples), d))
        groups = {}
        for n, (b, hk, j) in enumerate(samples):
            groups.setdefault((b, hk), []).append((n, j))
    for (b, hk), sel in groups.items():
        kb, vb = _f64(k[b, :, hk, :]), _f64(v[b, :, hk, :])
        cols = np.arange(Nk, dtype=np.int64) if sel is None else np.array([j for _, j in sel], np.int64)
        acc_k = np.zeros((len(cols), d))
        acc_v = np.zeros((len(cols), d))
        for h in range(hk * G, (hk + 1) * G):
            hm = m_of(h)
            vecs = [np.ascontiguousarray(x[b, hm]) for x in m4]
            qb, gb = _f64(q[b, :, h, :]), _f64(dout[b, :, h, :])
            rk = np.zeros((len(cols), d))
            rv = np.zeros((len(cols), d))
            lib.oracle_dkdv_head(_p(qb, _D), _p(gb, _D), Nq, _p(kb, _D), _p(vb, _D), Nk, d,
                                 *[_p(x, _I32) for x in vecs], sc, _p(cols, _I64), len(cols), _p(rk, _D), _p(rv, _D))
            acc_k += rk
            acc_v += rv
        if sel is None:
            dk[b, :, hk, :] = acc_k
            dv[b, :, hk, :] = acc_v
        else:
            for r, (nidx, _) in enumerate(sel):
                dk[nidx] = acc_k[r]
                dv[nidx] = acc_v[r]
    return dk, dv


def attention_backward(q, k, v, dout, lts, lte, uts, ute, scale: Optional[float] = None):
    """Full backward: ``(dq, dk, dv)`` as float64 arrays."""
    dq = attention_backward_dq(q, k, v, dout, lts, lte, uts, ute, scale)
    dk, dv = attention_backward_dkdv(q, k, v, dout, lts, lte, uts, ute, scale)
    return dq, dk, dv


def classify(lts, lte, uts, ute, Nq: int, Nk: int, bm: int = 128, bn: int = 128) -> np.ndarray:
    """Tile classes ``uint8 [B, Hm, ceil(Nq/bm), ceil(Nk/bn)]``: 0 skip, 1 partial, 2 full."""
    lib = _load()
    B = _i32(lts if lts is not None else uts).shape[0]
    m4 = _mask_arrays(lts, lte, uts, ute, B, Nk)
    Hm = m4[0].shape[1]
    nqt, nkt = -(-Nq // bm), -(-Nk // bn)
    out = np.zeros((B, Hm, nqt, nkt), np.uint8)
    for b in range(B):
        for hm in range(Hm):
            vecs = [np.ascontiguousarray(x[b, hm]) for x in m4]
            res = np.zeros((nqt, nkt), np.uint8)
            lib.oracle_classify(*[_p(x, _I32) for x in vecs], Nq, Nk, bm, bn, _p(res, _U8))
            out[b, hm] = res
    return out


def localize(x, a: int, b: int) -> np.ndarray:
    """Clip-shift-max of boundary values onto the query chunk [a, b)."""
    lib = _load()
    xi = _i32(x)
    flat = np.ascontiguousarray(xi.reshape(-1))
    out = np.zeros_like(flat)
    lib.oracle_localize(_p(flat, _I32), _p(out, _I32), flat.size, int(a), int(b))
    return out.reshape(xi.shape)


def localize_multi(x, chunks: Sequence[Tuple[int, int]]) -> np.ndarray:
    """Localisation onto increasing disjoint chunks concatenated in order."""
    lib = _load()
    xi = _i32(x)
    flat = np.ascontiguousarray(xi.reshape(-1))
    out = np.zeros_like(flat)
    a = np.array([c[0] for c in chunks], np.int32)
    b = np.array([c[1] for c in chunks], np.int32)
    lib.oracle_localize_multi(_p(flat, _I32), _p(out, _I32), flat.size, _p(a, _I32), _p(b, _I32), len(chunks))
    return out.reshape(xi.shape)


def count_unmasked(lts, lte, uts, ute, Nq: int, Nk: int, Hq: int) -> int:
    """Unmasked (i, j) pairs summed over batches and all Hq query heads (brute force)."""
    lib = _load()
    B = _i32(lts if lts is not None else uts).shape[0]
    m4 = _mask_arrays(lts, lte, uts, ute, B, Nk)
    Hm = m4[0].shape[1]
    total = 0
    for b in range(B):
        per_head = []
        for hm in range(Hm):
            vecs = [np.ascontiguousarray(x[b, hm]) for x in m4]
            per_head.append(int(lib.oracle_count_unmasked(*[_p(x, _I32) for x in vecs], Nq, Nk)))
        total += per_head[0] * Hq if Hm == 1 else sum(per_head)
    return total


def tile_costs(lts, lte, uts, ute, Nq: int, Nk: int, Hq: int, bm: int = 128) -> np.ndarray:
    """Unmasked (row, key) pairs of each ``bm``-row query tile, summed over batches and all Hq
    query heads (brute force over the mask predicate): ``int64 [ceil(Nq / bm)]``.

    This is the per-tile work that the load balancer of "FlashMask-3 targets masked distributed
    attention on Hopper GPUs", section "In-depth insight" (named there, HCC-IPO) evens out
    across ranks.
    """
    lib = _load()
    B = _i32(lts if lts is not None else uts).shape[0]
    m4 = _mask_arrays(lts, lte, uts, ute, B, Nk)
    Hm = m4[0].shape[1]
    nt = -(-Nq // bm)
    total = np.zeros(nt, np.int64)
    one = np.zeros(nt, np.int64)
    for b in range(B):
        for hm in range(Hm):
            vecs = [np.ascontiguousarray(x[b, hm]) for x in m4]
            lib.oracle_tile_costs(*[_p(x, _I32) for x in vecs], Nq, Nk, bm, one.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
            total += one * (Hq if Hm == 1 else 1)
    return total


def balance_minimax(costs: Sequence[int], parts: int) -> Tuple[int, List[int]]:
    """Splits tiles 0..n-1 into ``parts`` contiguous (possibly empty) chunks so that the largest
    chunk cost is as small as possible, by trying every split (small inputs only).

    Returns ``(best, bounds)``: the optimal largest cost and the first optimal split found in
    lexicographic order of the boundaries (``bounds[0] = 0``, ``bounds[parts] = n``).
    """
    import itertools

    c = [int(x) for x in costs]
    n = len(c)
    prefix = [0]
    for x in c:
        prefix.append(prefix[-1] + x)
    best, arg = None, None
    for cuts in itertools.combinations_with_replacement(range(n + 1), parts - 1):
        bounds = [0, *cuts, n]
        worst = max(prefix[bounds[p + 1]] - prefix[bounds[p]] for p in range(parts))
        if best is None or worst < best:
            best, arg = worst, bounds
    return best, arg


def mask_dense(lts, lte, uts, ute, Nq: int) -> np.ndarray:
    """Dense boolean mask ``[Nq, Nk]`` (True = masked) of ONE (batch, head): 1-D vectors in."""
    lib = _load()
    vecs = [np.ascontiguousarray(_i32(x).reshape(-1)) for x in (lts, lte, uts, ute)]
    Nk = vecs[0].size
    out = np.zeros((Nq, Nk), np.uint8)
    row = np.zeros(Nk, np.uint8)
    for i in range(Nq):
        lib.oracle_mask_row(*[_p(x, _I32) for x in vecs], Nk, i, _p(row, _U8))
        out[i] = row
    return out.astype(bool)
