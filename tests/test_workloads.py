"""The seeded workload generators encode the mask families they name (CPU only).

Each family's boundary vectors are checked against a dense mask built here
from the family's own definition (document ids, question/answer parts, prefix
and window distances), not from the vectors; the five workloads are checked
against the recipe they state (length ranges, totals, dropped-tile share).
"""
import numpy as np
import pytest
import torch

from column_sparse_masked_b200 import workloads as wl


def dense_from_vectors(lts, lte, uts, ute, nq):
    i = np.arange(nq)[:, None]
    return ((lts[None, :] <= i) & (i < lte[None, :])) | ((uts[None, :] <= i) & (i < ute[None, :]))


def test_causal_documents_match_document_ids():
    lengths = [5, 1, 9, 3, 12]
    n = sum(lengths)
    doc = np.repeat(np.arange(len(lengths)), lengths)
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    visible = (doc[i] == doc[j]) & (j <= i)
    assert np.array_equal(dense_from_vectors(*wl.causal_document_vectors(lengths), n), ~visible)


def test_causal_vectors_match_lower_triangle():
    n = 17
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    assert np.array_equal(dense_from_vectors(*wl.causal_vectors(n), n), j > i)
    assert not dense_from_vectors(*wl.empty_vectors(n), n).any()


def test_share_question_matches_parts():
    """An answer sees its own question and itself causally, never a sibling answer or another segment."""
    segs = [[4, 2, 3, 1], [3, 5], [2, 1, 1, 2, 3]]
    n = sum(sum(s) for s in segs)
    seg_id = np.concatenate([np.full(sum(s), t) for t, s in enumerate(segs)])
    part = np.concatenate([np.repeat(np.arange(len(s)), s) for s in segs])  # 0 = question, k = answer k
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    visible = (seg_id[i] == seg_id[j]) & (j <= i) & ((part[j] == 0) | (part[j] == part[i]))
    assert np.array_equal(dense_from_vectors(*wl.share_question_vectors(segs), n), ~visible)


@pytest.mark.parametrize("n,prefix,window", [(60, 7, 11), (40, 0, 40), (33, 33, 5)])
def test_prefix_window_matches_distances(n, prefix, window):
    """Prefix keys are seen by every row (also earlier ones), others causally; rows at distance
    >= window no longer see a key, prefix keys included."""
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    visible = ((j < prefix) | (j <= i)) & (i - j < window)
    assert np.array_equal(dense_from_vectors(*wl.prefix_window_vectors(n, prefix, window), n), ~visible)


def test_dropped_key_tiles_are_hidden_from_every_row():
    rng = np.random.default_rng(3)
    lengths = [20, 30, 14]
    n = sum(lengths)
    base = wl.causal_document_vectors(lengths)
    out = wl.drop_key_tiles(base, rng, 0.5, tile=8)
    dense_base = dense_from_vectors(*base, n)
    dense = dense_from_vectors(*out, n)
    dropped = [t for t in range(-(-n // 8)) if dense[:, t * 8:(t + 1) * 8].all()]
    assert 0 < len(dropped) < -(-n // 8)
    for t in range(-(-n // 8)):
        cols = slice(t * 8, (t + 1) * 8)
        if t in dropped:
            assert dense[:, cols].all()
        else:
            assert np.array_equal(dense[:, cols], dense_base[:, cols])


def _runs(x):
    """Lengths of the runs of equal values in a 1-D array."""
    cut = np.flatnonzero(np.diff(x)) + 1
    return np.diff(np.concatenate([[0], cut, [x.size]]))


def test_doc8k_recipe():
    w = wl.CONFIGS["doc8k"]
    lts, lte, uts, ute = [x[0, 0] for x in wl.mask_vectors(w)]
    lengths = _runs(lts)  # LTS is the end of each key's document
    assert lengths.sum() == w.N and np.all(lts == np.cumsum(lengths).repeat(lengths))
    assert np.all((lengths[:-1] >= 256) & (lengths[:-1] <= 4096)) and 1 <= lengths[-1] <= 4096
    assert np.all(lte == w.N) and np.all(uts == 0) and np.array_equal(ute, np.arange(w.N))


def test_sharequestion32k_recipe():
    w = wl.CONFIGS["sharequestion32k"]
    segs = wl.share_question_lengths(np.random.default_rng(w.seed + 4), w.N)
    assert len(segs) == 8 and all(len(s) == 5 for s in segs)
    assert sum(sum(s) for s in segs) == w.N and min(min(s) for s in segs) >= 1
    # the proportional rescale keeps questions longer than the shortest-possible answers' scale
    raw_ratio = 32768 / (8 * (4096 + 4 * 1024))
    assert all(s[0] >= int(1024 * raw_ratio) for s in segs)
    lts = wl.mask_vectors(w)[0][0, 0]
    assert np.array_equal(lts, wl.share_question_vectors(segs)[0])


def test_prefixwindow64k_recipe():
    w = wl.CONFIGS["prefixwindow64k"]
    v = wl.mask_vectors(w)
    assert v[0].shape == (2, 1, 65536) and np.array_equal(v[0][0], v[0][1])
    lts, lte, uts, ute = [x[0, 0] for x in v]
    # spot rows of the dense definition, away from the ends
    for jj in (0, 2047, 2048, 30000, 65535):
        col = dense_from_vectors(lts[jj:jj + 1], lte[jj:jj + 1], uts[jj:jj + 1], ute[jj:jj + 1], w.N)[:, 0]
        rows = np.arange(w.N)
        visible = ((jj < 2048) | (jj <= rows)) & (rows - jj < 4096)
        assert np.array_equal(col, ~visible), jj


def test_docblocksparse128k_recipe():
    w = wl.CONFIGS["docblocksparse128k"]
    lts, lte, uts, ute = [x[0, 0] for x in wl.mask_vectors(w)]
    ntiles = w.N // 128
    dropped = np.array([np.all(lts[t * 128:(t + 1) * 128] == 0) and np.all(lte[t * 128:(t + 1) * 128] == w.N)
                        for t in range(ntiles)])
    # Binomial(1024, 0.3): mean 307.2, sd 14.7; four sd either way
    assert abs(int(dropped.sum()) - 0.3 * ntiles) < 4 * np.sqrt(ntiles * 0.3 * 0.7)
    kept = ~np.repeat(dropped, 128)
    lengths = _runs(lts[kept])  # documents of the kept columns (a document may lose whole tiles)
    assert np.all(lengths <= 32768)
    assert np.all(uts == 0) and np.array_equal(ute, np.arange(w.N))


def test_tensors_are_seeded_bf16_and_distinct():
    w = wl.CONFIGS["tiny_doc"]
    a, b = wl.make_inputs(w), wl.make_inputs(w)
    for name in ("q", "k", "v"):
        assert a[name].dtype == torch.bfloat16 and torch.equal(a[name], b[name])
    assert a["q"].shape == (w.B, w.N, w.Hq, w.d) and a["k"].shape == (w.B, w.N, w.Hkv, w.d)
    assert not torch.equal(a["q"][..., : w.Hkv, :], a["k"])
    assert abs(float(a["q"].float().std()) - 1.0) < 0.05
