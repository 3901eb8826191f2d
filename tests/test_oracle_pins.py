"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties one oracle function to an independent fact: a library routine
that computes the same thing in a special case (torch's CPU scaled dot-product
attention in float64), a closed form, central finite differences, or brute
force over a dense mask built here with numpy.  The mask predicate is the one
of "FlashMask-3 targets masked distributed attention on Hopper GPUs",
section "In-depth insight" (four query-axis boundary vectors per key column).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from column_sparse_masked_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def dense_mask_np(lts, lte, uts, ute, nq):
    """Dense mask [nq, nk] (True = masked) built with numpy broadcasting."""
    i = np.arange(nq)[:, None]
    return ((lts[None, :] <= i) & (i < lte[None, :])) | ((uts[None, :] <= i) & (i < ute[None, :]))


def rand64(rng, *shape):
    return rng.standard_normal(shape)


def sdpa64(q, k, v, allowed=None, causal=False, scale=None):
    """torch CPU SDPA in float64; q [Nq, H, d] etc. -> O [Nq, H, d]."""
    qt = torch.as_tensor(q).permute(1, 0, 2)[None]
    kt = torch.as_tensor(k).permute(1, 0, 2)[None]
    vt = torch.as_tensor(v).permute(1, 0, 2)[None]
    m = None if allowed is None else torch.as_tensor(allowed)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, is_causal=causal, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


# ----------------------------------------------------------------------------
# forward
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("nq,nk,d", [(7, 7, 4), (33, 50, 16), (64, 64, 64)])
def test_unmasked_equals_sdpa(oracle_mod, nq, nk, d):
    rng = np.random.default_rng(1)
    q, k, v = rand64(rng, 1, nq, 2, d), rand64(rng, 1, nk, 2, d), rand64(rng, 1, nk, 2, d)
    z = np.zeros((1, 1, nk), np.int32)
    o, lse = oracle_mod.attention_forward(q, k, v, z, z, z, z)
    ref = sdpa64(q[0], k[0], v[0])
    assert np.abs(o[0] - ref).max() < 1e-12
    # LSE of the unmasked row: log-sum-exp of the scaled logits (scipy-free closed form)
    s = np.einsum("ihd,jhd->hij", q[0], k[0]) / math.sqrt(d)
    m = s.max(-1, keepdims=True)
    lse_ref = (m + np.log(np.exp(s - m).sum(-1, keepdims=True)))[..., 0]
    assert np.abs(lse[0] - lse_ref).max() < 1e-12


@pytest.mark.parametrize("n,d", [(9, 4), (40, 32)])
def test_causal_encoding_equals_sdpa_causal(oracle_mod, n, d):
    rng = np.random.default_rng(2)
    q, k, v = rand64(rng, 1, n, 3, d), rand64(rng, 1, n, 3, d), rand64(rng, 1, n, 3, d)
    vecs = [x[None, None] for x in wl.causal_vectors(n)]
    o, _ = oracle_mod.attention_forward(q, k, v, *vecs)
    ref = sdpa64(q[0], k[0], v[0], causal=True)
    assert np.abs(o[0] - ref).max() < 1e-12


def test_random_mask_equals_sdpa_boolean_mask(oracle_mod):
    """Arbitrary masks agree with SDPA given the dense boolean mask (rows with >= 1 visible key)."""
    rng = np.random.default_rng(3)
    nq, nk, d, H = 37, 45, 8, 2
    vecs = wl.random_interval_vectors(rng, nq, nk)
    dense = dense_mask_np(*vecs, nq)
    q, k, v = rand64(rng, 1, nq, H, d), rand64(rng, 1, nk, H, d), rand64(rng, 1, nk, H, d)
    o, lse = oracle_mod.attention_forward(q, k, v, *[x[None, None] for x in vecs], scale=0.3)
    ok_rows = ~dense.all(1)
    ref = sdpa64(q[0], k[0], v[0], allowed=~dense, scale=0.3)
    assert np.abs(o[0][ok_rows] - ref[ok_rows]).max() < 1e-12
    assert np.all(o[0][~ok_rows] == 0.0)
    assert np.all(np.isneginf(lse[0][:, ~ok_rows]))


@pytest.mark.parametrize("name", ["tiny_doc"])
def test_zero_query_closed_form(oracle_mod, name):
    """With Q = 0 every visible logit is 0: O_i = mean of visible v_j, LSE_i = ln |V_i|."""
    w = wl.CONFIGS[name]
    inp = wl.make_inputs(w, with_grad=False)
    q = torch.zeros_like(inp["q"])
    o, lse = oracle_mod.attention_forward(q, inp["k"], inp["v"], inp["lts"], inp["lte"], inp["uts"], inp["ute"])
    vecs = [inp[n][0, 0].numpy() for n in ("lts", "lte", "uts", "ute")]
    vis = ~dense_mask_np(*vecs, w.N)
    cnt = vis.sum(1)
    v = inp["v"].double().numpy()
    for h in range(w.Hq):
        mean = (vis.astype(np.float64) @ v[0, :, h, :]) / np.maximum(cnt, 1)[:, None]
        assert np.abs(o[0, :, h, :] - mean).max() < 1e-12
        assert np.abs(lse[0, h] - np.log(cnt)).max() < 1e-12


def _count_visible_by_intervals(vecs, nq):
    """|V_i| from interval arithmetic: per key, the rows it hides are [a,b) U [c,d)."""
    lts, lte, uts, ute = [x.astype(np.int64) for x in vecs]
    nk = lts.size
    hidden = np.zeros(nq + 1, np.int64)

    def add(lo, hi, sgn):
        lo = np.clip(lo, 0, nq)
        hi = np.clip(hi, 0, nq)
        ok = hi > lo
        np.add.at(hidden, lo[ok], sgn)
        np.add.at(hidden, hi[ok], -sgn)

    add(lts, lte, 1)
    add(uts, ute, 1)
    add(np.maximum(lts, uts), np.minimum(lte, ute), -1)  # intersection counted twice
    return nk - np.cumsum(hidden)[:nq]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_zero_query_closed_form_random_masks(oracle_mod, seed):
    rng = np.random.default_rng(100 + seed)
    nq, nk, d = 150, 170, 8
    vecs = wl.random_interval_vectors(rng, nq, nk)
    k, v = rand64(rng, 1, nk, 1, d), rand64(rng, 1, nk, 1, d)
    q = np.zeros((1, nq, 1, d))
    o, lse = oracle_mod.attention_forward(q, k, v, *[x[None, None] for x in vecs])
    cnt = _count_visible_by_intervals(vecs, nq)
    with np.errstate(divide="ignore"):
        assert np.array_equal(np.isneginf(lse[0, 0]), cnt == 0)
        assert np.abs(lse[0, 0][cnt > 0] - np.log(cnt[cnt > 0])).max() < 1e-12


def test_fully_masked_rows(oracle_mod):
    """Every key hidden from rows 5 and 6: those rows give O = 0, LSE = -inf, dQ = 0."""
    rng = np.random.default_rng(4)
    n, d = 12, 4
    lts = np.full(n, 5, np.int32)
    lte = np.full(n, 7, np.int32)
    z = np.zeros(n, np.int32)
    vecs = [x[None, None] for x in (lts, lte, z, z)]
    q, k, v, g = rand64(rng, 1, n, 1, d), rand64(rng, 1, n, 1, d), rand64(rng, 1, n, 1, d), rand64(rng, 1, n, 1, d)
    o, lse = oracle_mod.attention_forward(q, k, v, *vecs)
    assert np.all(o[0, 5:7] == 0.0) and np.all(np.isneginf(lse[0, 0, 5:7]))
    assert np.all(np.isfinite(lse[0, 0, :5])) and np.all(np.isfinite(lse[0, 0, 7:]))
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, g, *vecs)
    assert np.all(dq[0, 5:7] == 0.0)


def test_golden_hand_example(oracle_mod):
    """Hand-derived 4-token example (tests/golden/hand_doc4.json)."""
    with open(os.path.join(GOLDEN, "hand_doc4.json")) as f:
        g = json.load(f)
    vecs = [np.array(g[n], np.int32)[None, None] for n in ("lts", "lte", "uts", "ute")]
    v = np.array(g["v"], np.float64)[None, :, None, :]
    n, d = v.shape[1], v.shape[3]
    q = np.zeros((1, n, 1, d))
    k = np.ones((1, n, 1, d))
    o, lse = oracle_mod.attention_forward(q, k, v, *vecs)
    assert np.abs(o[0, :, 0, :] - np.array(g["o"])).max() < 1e-12
    assert np.abs(lse[0, 0] - np.log(np.array(g["visible_count"], np.float64))).max() < 1e-12


def test_gqa_and_batches_equal_sdpa_with_repeated_kv(oracle_mod):
    """Grouped KV heads and batches: torch SDPA per batch on K, V repeated over each group.

    q-head h reads KV head h // (Hq / Hkv) (consecutive q-heads share a KV
    head); batch b uses its own mask vectors.  The reference expands K and V
    with np.repeat along the head axis and builds each batch's dense mask here.
    """
    rng = np.random.default_rng(9)
    B, nq, nk, hq, hkv, d = 2, 29, 23, 6, 2, 8
    per_batch = [wl.random_interval_vectors(rng, nq, nk) for _ in range(B)]
    vecs = [np.stack([pb[t] for pb in per_batch])[:, None, :] for t in range(4)]
    q, k, v = rand64(rng, B, nq, hq, d), rand64(rng, B, nk, hkv, d), rand64(rng, B, nk, hkv, d)
    o, lse = oracle_mod.attention_forward(q, k, v, *vecs, scale=0.4)
    G = hq // hkv
    for b in range(B):
        dense = dense_mask_np(*per_batch[b], nq)
        ok_rows = ~dense.all(1)
        assert ok_rows.sum() > nq // 2
        ref = sdpa64(q[b], np.repeat(k[b], G, axis=1), np.repeat(v[b], G, axis=1), allowed=~dense, scale=0.4)
        assert np.abs(o[b][ok_rows] - ref[ok_rows]).max() < 1e-12
        assert np.all(o[b][~ok_rows] == 0.0)
        assert np.all(np.isneginf(lse[b][:, ~ok_rows]))


def test_per_head_masks_equal_sdpa_per_head(oracle_mod):
    """One mask per q-head (Hm = Hq): head h follows its own vectors, checked head by head."""
    rng = np.random.default_rng(10)
    nq, nk, h, d = 31, 27, 3, 8
    per_head = [wl.random_interval_vectors(rng, nq, nk, p_empty=0.1) for _ in range(h)]
    vecs = [np.stack([ph[t] for ph in per_head])[None] for t in range(4)]
    q, k, v = rand64(rng, 1, nq, h, d), rand64(rng, 1, nk, h, d), rand64(rng, 1, nk, h, d)
    o, lse = oracle_mod.attention_forward(q, k, v, *vecs)
    distinct = 0
    for hh in range(h):
        dense = dense_mask_np(*per_head[hh], nq)
        distinct += int(not np.array_equal(dense, dense_mask_np(*per_head[0], nq)))
        ok_rows = ~dense.all(1)
        ref = sdpa64(q[0][:, hh:hh + 1], k[0][:, hh:hh + 1], v[0][:, hh:hh + 1], allowed=~dense)
        assert np.abs(o[0][ok_rows, hh] - ref[ok_rows, 0]).max() < 1e-12
        assert np.all(o[0][~ok_rows, hh] == 0.0) and np.all(np.isneginf(lse[0, hh][~ok_rows]))
    assert distinct == h - 1  # the heads' masks really differ


# ----------------------------------------------------------------------------
# backward
# ----------------------------------------------------------------------------
def _loss(oracle_mod, q, k, v, g, vecs, scale):
    o, _ = oracle_mod.attention_forward(q, k, v, *vecs, scale=scale)
    return float((o * g).sum())


@pytest.mark.parametrize("seed,hq,hkv", [(0, 1, 1), (1, 2, 1), (2, 4, 2)])
def test_backward_finite_differences(oracle_mod, seed, hq, hkv):
    rng = np.random.default_rng(200 + seed)
    nq, nk, d = 11, 13, 4
    vecs = wl.random_interval_vectors(rng, nq, nk)
    vecs[0][3], vecs[1][3] = 0, nq  # one key no row sees
    vecs = [x[None, None] for x in vecs]
    q, k, v, g = rand64(rng, 1, nq, hq, d), rand64(rng, 1, nk, hkv, d), rand64(rng, 1, nk, hkv, d), \
        rand64(rng, 1, nq, hq, d)
    scale = 0.7
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, g, *vecs, scale=scale)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + eps
            lp = _loss(oracle_mod, q, k, v, g, vecs, scale)
            x[idx] = old - eps
            lm = _loss(oracle_mod, q, k, v, g, vecs, scale)
            x[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        err = np.abs(num - grad).max() / max(1.0, np.abs(num).max())
        assert err < 1e-6, (name, err)
    assert np.all(dk[0, 3] == 0.0) and np.all(dv[0, 3] == 0.0)


def test_backward_equals_torch_autograd_sdpa(oracle_mod):
    """Library special case: autograd of float64 SDPA with the dense boolean mask."""
    rng = np.random.default_rng(5)
    nq, nk, d = 30, 30, 16
    vecs = wl.causal_vectors(nq)
    q, k, v, g = (torch.tensor(rand64(rng, 1, n, 2, d), requires_grad=True) for n in (nq, nk, nk, nq))
    g = g.detach()
    o = sdpa_t = torch.nn.functional.scaled_dot_product_attention(
        q.permute(0, 2, 1, 3), k.permute(0, 2, 1, 3), v.permute(0, 2, 1, 3), is_causal=True).permute(0, 2, 1, 3)
    (o * g).sum().backward()
    dq, dk, dv = oracle_mod.attention_backward(q.detach(), k.detach(), v.detach(), g, *[x[None, None] for x in vecs])
    for a, b in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
        assert np.abs(a - b.numpy()).max() < 1e-12
    del sdpa_t


def test_gqa_backward_equals_torch_autograd_repeated_kv(oracle_mod):
    """Grouped KV heads and batches in the backward: autograd of float64 SDPA on K, V repeated
    over each group (repeat_interleave sums the group's gradients into each KV head), with each
    batch's own causal-document mask as a dense boolean mask."""
    rng = np.random.default_rng(11)
    B, n, hq, hkv, d = 2, 26, 4, 2, 8
    G = hq // hkv
    docs = [[9, 17], [5, 12, 9]]
    per_batch = [wl.causal_document_vectors(L) for L in docs]
    vecs = [np.stack([pb[t] for pb in per_batch])[:, None, :] for t in range(4)]
    allowed = torch.as_tensor(np.stack([~dense_mask_np(*pb, n) for pb in per_batch]))[:, None]
    q, k, v = (torch.tensor(rand64(rng, B, n, h, d), requires_grad=True) for h in (hq, hkv, hkv))
    g = torch.tensor(rand64(rng, B, n, hq, d))
    kr, vr = (x.repeat_interleave(G, dim=2) for x in (k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        q.permute(0, 2, 1, 3), kr.permute(0, 2, 1, 3), vr.permute(0, 2, 1, 3), attn_mask=allowed,
        scale=0.5).permute(0, 2, 1, 3)
    (o * g).sum().backward()
    dq, dk, dv = oracle_mod.attention_backward(q.detach(), k.detach(), v.detach(), g, *vecs, scale=0.5)
    for a, b in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
        assert np.abs(a - b.numpy()).max() < 1e-12


def test_backward_half_squared_norm(oracle_mod):
    """With dO = O (held fixed) the backward is the gradient of sum|O|^2 / 2.

    Checked against central finite differences of that loss through the
    forward; this exercises the D_i = sum_j P_ij dP_ij term with dO correlated
    with the output.
    """
    rng = np.random.default_rng(6)
    nq, d = 9, 3
    vecs = [x[None, None] for x in wl.random_interval_vectors(rng, nq, nq)]
    q, k, v = rand64(rng, 1, nq, 1, d), rand64(rng, 1, nq, 1, d), rand64(rng, 1, nq, 1, d)
    o, _ = oracle_mod.attention_forward(q, k, v, *vecs)
    dq = oracle_mod.attention_backward_dq(q, k, v, o, *vecs)
    eps = 1e-6
    num = np.zeros_like(q)
    for i in range(nq):
        for c in range(d):
            old = q[0, i, 0, c]
            q[0, i, 0, c] = old + eps
            lp = float((oracle_mod.attention_forward(q, k, v, *vecs)[0] ** 2).sum()) / 2
            q[0, i, 0, c] = old - eps
            lm = float((oracle_mod.attention_forward(q, k, v, *vecs)[0] ** 2).sum()) / 2
            q[0, i, 0, c] = old
            num[0, i, 0, c] = (lp - lm) / (2 * eps)
    # d/dq of sum|O|^2 / 2 with O held as dO (first-order identical)
    assert np.abs(num - dq).max() < 1e-6


def test_sampled_rows_and_cols_match_full(oracle_mod):
    rng = np.random.default_rng(7)
    B, nq, hq, hkv, d = 2, 20, 4, 2, 8
    vecs = [np.stack([x for x in wl.random_interval_vectors(rng, nq, nq)])[None].repeat(B, 0)[:, :, :]
            for _ in range(1)][0]
    vecs = [vecs[:, t:t + 1, :].copy() for t in range(4)]
    q, k, v, g = rand64(rng, B, nq, hq, d), rand64(rng, B, nq, hkv, d), rand64(rng, B, nq, hkv, d), \
        rand64(rng, B, nq, hq, d)
    o, lse = oracle_mod.attention_forward(q, k, v, *vecs)
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, g, *vecs)
    rows = [(1, 3, 7), (0, 0, 0), (1, 2, 19)]
    so, sl = oracle_mod.attention_forward(q, k, v, *vecs, samples=rows)
    sdq = oracle_mod.attention_backward_dq(q, k, v, g, *vecs, samples=rows)
    for n, (b, h, i) in enumerate(rows):
        assert np.array_equal(so[n], o[b, i, h]) and (sl[n] == lse[b, h, i])
        assert np.array_equal(sdq[n], dq[b, i, h])
    cols = [(0, 1, 5), (1, 0, 19)]
    sdk, sdv = oracle_mod.attention_backward_dkdv(q, k, v, g, *vecs, samples=cols)
    for n, (b, hk, j) in enumerate(cols):
        assert np.abs(sdk[n] - dk[b, j, hk]).max() < 1e-13 and np.abs(sdv[n] - dv[b, j, hk]).max() < 1e-13


# ----------------------------------------------------------------------------
# classification, localisation, pair count
# ----------------------------------------------------------------------------
def _check_sound(cls, dense, bm, bn):
    nq, nk = dense.shape
    for r in range(cls.shape[0]):
        for c in range(cls.shape[1]):
            t = dense[r * bm:(r + 1) * bm, c * bn:(c + 1) * bn]
            if cls[r, c] == 0:
                assert t.all(), (r, c)
            elif cls[r, c] == 2:
                assert not t.any(), (r, c)


@pytest.mark.parametrize("seed", range(6))
def test_classify_sound_random(oracle_mod, seed):
    rng = np.random.default_rng(300 + seed)
    nq, nk, bm, bn = int(rng.integers(1, 90)), int(rng.integers(1, 90)), 8, 8
    vecs = wl.random_interval_vectors(rng, nq, nk, p_empty=0.5)
    cls = oracle_mod.classify(*[x[None, None] for x in vecs], nq, nk, bm, bn)[0, 0]
    _check_sound(cls, dense_mask_np(*vecs, nq), bm, bn)
    assert cls.shape == (-(-nq // bm), -(-nk // bn))


@pytest.mark.parametrize("name", ["tiny_doc", "doc8k"])
def test_classify_sound_configs(oracle_mod, name):
    w = wl.CONFIGS[name]
    vecs = [x[0, 0] for x in wl.mask_vectors(w)]
    cls = oracle_mod.classify(*[x[None, None] for x in vecs], w.N, w.N)[0, 0]
    n = min(w.N, 2048)
    _check_sound(cls[: n // 128, : n // 128], dense_mask_np(*[x[:n] for x in vecs], n), 128, 128)


def test_classify_causal_closed_form(oracle_mod):
    n = 1000
    cls = oracle_mod.classify(*[x[None, None] for x in wl.causal_vectors(n)], n, n)[0, 0]
    nt = -(-n // 128)
    r, c = np.meshgrid(np.arange(nt), np.arange(nt), indexing="ij")
    expect = np.where(c < r, 2, np.where(c == r, 1, 0))
    assert np.array_equal(cls, expect)


def classify_golden():
    """Vectors, Nq and expected classes of tests/golden/classify_clauses.json (hand-derived)."""
    with open(os.path.join(GOLDEN, "classify_clauses.json")) as f:
        d = json.load(f)
    vec = {n: [] for n in ("lts", "lte", "uts", "ute")}
    for t in d["ktiles"]:
        for n in vec:
            x = t[n]
            vec[n] += list(x) if isinstance(x, list) else [x] * t["n"]
            assert len(vec[n]) == len(vec["lts"]) or n == "lts"
    vecs = [np.array(vec[n], np.int32) for n in ("lts", "lte", "uts", "ute")]
    return vecs, int(d["Nq"]), np.array(d["expected"], np.uint8)


def test_classify_golden_clauses(oracle_mod):
    """Every clause of the tile rule, at its boundary, is the only one deciding some tile of the
    hand-derived golden: a dropped clause or a strict/non-strict slip changes a class."""
    vecs, nq, expect = classify_golden()
    nk = vecs[0].size
    cls = oracle_mod.classify(*[x[None, None] for x in vecs], nq, nk)[0, 0]
    assert cls.shape == expect.shape
    assert np.array_equal(cls, expect), np.argwhere(cls != expect)
    _check_sound(expect, dense_mask_np(*vecs, nq), 128, 128)  # the golden itself is sound


def test_classify_tile_aligned_documents(oracle_mod):
    lengths = [256, 128, 384, 256]
    vecs = wl.causal_document_vectors(lengths)
    n = sum(lengths)
    cls = oracle_mod.classify(*[x[None, None] for x in vecs], n, n)[0, 0]
    doc = np.repeat(np.arange(len(lengths)), np.array(lengths) // 128)
    nt = n // 128
    for r in range(nt):
        for c in range(nt):
            e = 0 if (doc[r] != doc[c] or c > r) else (1 if c == r else 2)
            assert cls[r, c] == e, (r, c)


@pytest.mark.parametrize("seed", range(5))
def test_localize_reproduces_dense_rows(oracle_mod, seed):
    """Zero-communication localisation: the local vectors encode exactly rows [a, b) of the full mask."""
    rng = np.random.default_rng(400 + seed)
    nq, nk = 97, 61
    vecs = wl.random_interval_vectors(rng, nq, nk)
    full = dense_mask_np(*vecs, nq)
    for _ in range(5):
        a, b = sorted(int(x) for x in rng.integers(0, nq + 1, size=2))
        loc = [oracle_mod.localize(x, a, b) for x in vecs]
        assert all(((x >= 0) & (x <= b - a)).all() for x in loc)
        assert np.array_equal(dense_mask_np(*loc, b - a), full[a:b])


@pytest.mark.parametrize("seed", range(5))
def test_localize_multi_reproduces_dense_rows(oracle_mod, seed):
    rng = np.random.default_rng(500 + seed)
    nq, nk = 120, 40
    vecs = wl.random_interval_vectors(rng, nq, nk)
    full = dense_mask_np(*vecs, nq)
    cuts = sorted(set(int(x) for x in rng.integers(0, nq + 1, size=6)))
    chunks = [(cuts[t], cuts[t + 1]) for t in range(0, len(cuts) - 1, 2)]
    loc = [oracle_mod.localize_multi(x, chunks) for x in vecs]
    rows = np.concatenate([np.arange(a, b) for a, b in chunks]) if chunks else np.zeros(0, int)
    assert np.array_equal(dense_mask_np(*loc, rows.size), full[rows])
    # a single chunk reduces to clip-shift-max
    a, b = 17, 90
    assert all(np.array_equal(oracle_mod.localize_multi(x, [(a, b)]), oracle_mod.localize(x, a, b)) for x in vecs)


def test_count_unmasked(oracle_mod):
    rng = np.random.default_rng(8)
    nq, nk = 70, 55
    vecs = wl.random_interval_vectors(rng, nq, nk)
    dense = dense_mask_np(*vecs, nq)
    assert oracle_mod.count_unmasked(*[x[None, None] for x in vecs], nq, nk, 3) == 3 * int((~dense).sum())
    n = 777
    assert oracle_mod.count_unmasked(*[x[None, None] for x in wl.causal_vectors(n)], n, n, 1) == n * (n + 1) // 2
    lengths = [100, 300, 377]
    got = oracle_mod.count_unmasked(*[x[None, None] for x in wl.causal_document_vectors(lengths)], n, n, 2)
    assert got == 2 * sum(L * (L + 1) // 2 for L in lengths)


def test_count_unmasked_batches_and_per_head_masks(oracle_mod):
    """B = 2 batches with one mask per q-head (Hm = Hq): the count is the sum of every
    (batch, head) dense count; with Hm = 1 each batch's count is taken Hq times."""
    rng = np.random.default_rng(12)
    B, nq, nk, hq = 2, 41, 37, 3
    per = [[wl.random_interval_vectors(rng, nq, nk) for _ in range(hq)] for _ in range(B)]
    vecs = [np.stack([np.stack([per[b][h][t] for h in range(hq)]) for b in range(B)]) for t in range(4)]
    want = sum(int((~dense_mask_np(*per[b][h], nq)).sum()) for b in range(B) for h in range(hq))
    assert oracle_mod.count_unmasked(*vecs, nq, nk, hq) == want
    first = [x[:, :1].copy() for x in vecs]
    want1 = hq * sum(int((~dense_mask_np(*per[b][0], nq)).sum()) for b in range(B))
    assert oracle_mod.count_unmasked(*first, nq, nk, hq) == want1
