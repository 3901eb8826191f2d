"""GPU parity on the five workloads at full size, in the launch configuration
the benchmark times (flashmask_fwd + flashmask_bwd through the C ABI).

 - tiny causal-document case: every output against the oracle;
 - 8K..128K cases: sampled query rows (O, LSE, dQ) and sampled key columns
   (dK, dV) against the oracle computed one by one, plus identities that
   hold at any size over ALL key columns: sum_j dV_j = sum over the group's
   q-heads of sum_{i with a visible key} dO_i, and sum_j dK_j = 0;
 - the 128K case also runs the 4-chunk clip-shift-max localisation check:
   the forward of each query chunk against all keys, with the boundary
   vectors localised onto the chunk, equals rows [a, b) of the full-sequence
   run bit for bit (O and LSE); per-chunk dQ and the chunk sums of dK/dV
   match the full run within tolerance.
"""
import numpy as np
import pytest
import torch

import column_sparse_masked_b200 as fm
from column_sparse_masked_b200 import workloads as wl

from _parity import BF16_HALF_ULP_REL, check_lse, check_out

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oracle_mod():
    import oracle

    oracle.build_oracle()
    return oracle


def visible_counts(vecs, nq):
    """Per key column: number of query rows in [0, nq) that see it (interval arithmetic)."""
    lts, lte, uts, ute = [x.astype(np.int64) for x in vecs]

    def ov(a, b):
        return np.clip(np.minimum(b, nq) - np.maximum(a, 0), 0, None)

    return nq - (ov(lts, lte) + ov(uts, ute) - ov(np.maximum(lts, uts), np.minimum(lte, ute)))


def rows_with_visible_key(vecs, nq):
    """Boolean per query row: at least one key visible (difference array over hidden intervals)."""
    lts, lte, uts, ute = [x.astype(np.int64) for x in vecs]
    nk = lts.size
    hidden = np.zeros(nq + 1, np.int64)

    def add(lo, hi, sgn):
        lo, hi = np.clip(lo, 0, nq), np.clip(hi, 0, nq)
        ok = hi > lo
        np.add.at(hidden, lo[ok], sgn)
        np.add.at(hidden, hi[ok], -sgn)

    add(lts, lte, 1)
    add(uts, ute, 1)
    add(np.maximum(lts, uts), np.minimum(lte, ute), -1)
    return (nk - np.cumsum(hidden)[:nq]) > 0


def pick_columns(vecs, nq, hkv_count, seed, n_cheap=3, n_rand=3, max_rows=2048, extra=()):
    """Key columns for the sampled dK/dV check, spread over the whole range of visible-row counts:
    the column the most rows see (the first key of the longest document, the last prefix key),
    columns at 3/4, 1/2 and 1/4 of that count which the same rows see (the heaviest column's
    neighbours to its right), the cheapest columns, random columns seen by <= max_rows rows,
    `extra` columns, and a column no row sees (dK = dV = 0)."""
    cnt = visible_counts(vecs, nq)
    rng = np.random.default_rng(seed)
    heavy = int(np.argmax(cnt))
    cols = {heavy}
    for frac in (0.75, 0.5, 0.25):  # long-range accumulation over many q-tiles, same rows as `heavy`
        right = np.nonzero((np.arange(cnt.size) > heavy) & (cnt > 0) & (cnt <= frac * cnt[heavy]))[0]
        if right.size:
            cols.add(int(right[0]))
    ok = np.nonzero((cnt > 0) & (cnt <= max_rows))[0]
    cols |= set(int(x) for x in ok[np.argsort(cnt[ok], kind="stable")[:n_cheap]])
    if ok.size:
        cols |= set(int(x) for x in rng.choice(ok, size=min(n_rand, ok.size), replace=False))
    cols |= set(int(j) for j in extra)
    cols = sorted(cols)
    none = np.nonzero(cnt == 0)[0]
    if none.size:
        cols.append(int(none[0]))  # a column no row sees: dK = dV = 0
    return [(0, int(rng.integers(0, hkv_count)), j) for j in cols], cnt


def run_full(w, inp):
    dev = {n: inp[n].cuda() for n in ("q", "k", "v", "do", "lts", "lte", "uts", "ute")}
    m = [dev[n] for n in ("lts", "lte", "uts", "ute")]
    o, lse = fm.fwd(dev["q"], dev["k"], dev["v"], *m)
    dq, dk, dv = fm.bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], *m)
    torch.cuda.synchronize()
    assert fm.get_status() == 0
    return dev, m, o, lse, dq, dk, dv


def test_tiny_doc_all_outputs(oracle_mod):
    w = wl.CONFIGS["tiny_doc"]
    inp = wl.make_inputs(w)
    dev, m, o, lse, dq, dk, dv = run_full(w, inp)
    masks = [inp[n] for n in ("lts", "lte", "uts", "ute")]
    ro, rl = oracle_mod.attention_forward(inp["q"], inp["k"], inp["v"], *masks)
    check_out("O", o, ro, case="tiny_doc")
    check_lse(lse, rl, case="tiny_doc")
    rdq, rdk, rdv = oracle_mod.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], *masks)
    check_out("dQ", dq, rdq, case="tiny_doc")
    check_out("dK", dk, rdk, case="tiny_doc")
    check_out("dV", dv, rdv, case="tiny_doc")


def _identity_checks(w, inp, dk, dv):
    vecs = [inp[n][0, 0].numpy() for n in ("lts", "lte", "uts", "ute")]
    vis_rows = torch.from_numpy(rows_with_visible_key(vecs, w.N))
    G = w.Hq // w.Hkv
    for b in range(w.B):
        do_b = inp["do"][b][vis_rows]  # [rows with a visible key, Hq, d] bf16
        for hk in range(w.Hkv):
            gv = dv[b, :, hk].double().cpu().numpy()
            gk = dk[b, :, hk].double().cpu().numpy()
            expect_v = do_b[:, hk * G:(hk + 1) * G].double().sum((0, 1)).numpy()
            for name, g, e in (("sum dV", gv, expect_v), ("sum dK", gk, np.zeros(w.d))):
                sigma = np.sqrt(((BF16_HALF_ULP_REL * np.abs(g)) ** 2 + 1e-3 ** 2).sum(0))
                err = np.abs(g.sum(0) - e)
                assert (err <= 8 * sigma + 1e-3).all(), f"{name} b{b} hkv{hk}: err {err.max()} sigma {sigma.max()}"


@pytest.mark.parametrize("name", ["doc8k", "sharequestion32k", "prefixwindow64k", "docblocksparse128k"])
def test_config_sampled_parity(oracle_mod, name):
    """Fused backward (the default mode); the split mode's agreement with it on the 8K and 32K
    workloads is checked in test_gpu_kernels.py."""
    w = wl.CONFIGS[name]
    inp = wl.make_inputs(w)
    dev, m, o, lse, dq, dk, dv = run_full(w, inp)
    masks = [inp[n] for n in ("lts", "lte", "uts", "ute")]
    rows = wl.sample_rows(w, 24, seed=w.seed + 10)
    ro, rl = oracle_mod.attention_forward(inp["q"], inp["k"], inp["v"], *masks, samples=rows)
    rdq = oracle_mod.attention_backward_dq(inp["q"], inp["k"], inp["v"], inp["do"], *masks, samples=rows)
    go = torch.stack([o[b, i, h] for b, h, i in rows])
    gl = torch.stack([lse[b, h, i] for b, h, i in rows])
    gdq = torch.stack([dq[b, i, h] for b, h, i in rows])
    check_out("O(sampled)", go, ro, case=name)
    check_lse(gl, rl, case=name)
    check_out("dQ(sampled)", gdq, rdq, case=name)
    vecs0 = [x[0, 0].numpy() for x in masks]
    extra = (0,) if name == "prefixwindow64k" else ()  # first prefix key: seen by the first 4096 rows
    cols, cnt = pick_columns(vecs0, w.N, w.Hkv, seed=w.seed + 20, extra=extra)
    assert max(cnt[j] for _, _, j in cols) == cnt.max()
    rdk, rdv = oracle_mod.attention_backward_dkdv(inp["q"], inp["k"], inp["v"], inp["do"], *masks, samples=cols)
    gdk = torch.stack([dk[b, j, hk] for b, hk, j in cols])
    gdv = torch.stack([dv[b, j, hk] for b, hk, j in cols])
    check_out("dK(sampled)", gdk, rdk, case=name)
    check_out("dV(sampled)", gdv, rdv, case=name)
    _identity_checks(w, inp, dk, dv)

    if w.chunks:
        n = w.N // w.chunks
        dk_sum = torch.zeros_like(dk, dtype=torch.float32)
        dv_sum = torch.zeros_like(dv, dtype=torch.float32)
        for c in range(w.chunks):
            a, b = c * n, (c + 1) * n
            loc = [fm.localize(x, a, b) for x in m]
            qc = dev["q"][:, a:b].contiguous()
            oc, lc = fm.fwd(qc, dev["k"], dev["v"], *loc)
            assert torch.equal(oc, o[:, a:b]), f"chunk {c}: O differs from rows [{a},{b}) of the full run"
            assert torch.equal(lc, lse[:, :, a:b].contiguous()), f"chunk {c}: LSE differs"
            dqc, dkc, dvc = fm.bwd(qc, dev["k"], dev["v"], oc, lc, dev["do"][:, a:b].contiguous(), *loc)
            err = (dqc.float() - dq[:, a:b].float()).abs()
            assert (err <= 2e-2 + BF16_HALF_ULP_REL * dq[:, a:b].float().abs()).all(), f"chunk {c}: dQ"
            dk_sum += dkc.float()
            dv_sum += dvc.float()
        torch.cuda.synchronize()
        assert fm.get_status() == 0
        for nm, s, full in (("dK", dk_sum, dk), ("dV", dv_sum, dv)):
            err = (s - full.float()).abs()
            bound = 2e-2 + 4 * BF16_HALF_ULP_REL * full.float().abs()
            assert (err <= bound).all(), f"sum over chunks of {nm} vs full run: max err {err.max().item()}"


@pytest.mark.parametrize("name", ["doc8k", "docblocksparse128k"])
def test_zigzag_multichunk_equals_full_run(name):
    """Multi-chunk localisation ("FlashMask-3 targets masked distributed attention on Hopper GPUs",
    In-depth insight: exchange-free localisation under any multi-chunk context-parallel assignment).
    A 4-rank zigzag assignment: rank r holds query chunks [r N/8, (r+1) N/8) and
    [(7-r) N/8, (8-r) N/8), concatenated in order, with the boundary vectors localised onto the
    pair.  Against all keys, each rank's O and LSE equal the full run's rows bit for bit (chunk
    ends are multiples of 256 rows); its dQ rows match within tolerance; the ranks' dK, dV sum to
    the full run's within tolerance."""
    w = wl.CONFIGS[name]
    inp = wl.make_inputs(w)
    dev, m, o, lse, dq, dk, dv = run_full(w, inp)
    n8 = w.N // 8
    assert n8 % 256 == 0
    dk_sum = torch.zeros_like(dk, dtype=torch.float32)
    dv_sum = torch.zeros_like(dv, dtype=torch.float32)
    for r in range(4):
        chunks = [(r * n8, (r + 1) * n8), ((7 - r) * n8, (8 - r) * n8)]
        loc = [fm.localize_multi(x, chunks) for x in m]
        rows = torch.cat([torch.arange(a, b, device="cuda") for a, b in chunks])
        qc = dev["q"][:, rows].contiguous()
        doc = dev["do"][:, rows].contiguous()
        oc, lc = fm.fwd(qc, dev["k"], dev["v"], *loc)
        assert torch.equal(oc, o[:, rows]), f"rank {r}: O differs from the full run's rows"
        assert torch.equal(lc, lse[:, :, rows].contiguous()), f"rank {r}: LSE differs"
        dqc, dkc, dvc = fm.bwd(qc, dev["k"], dev["v"], oc, lc, doc, *loc)
        ref = dq[:, rows].float()
        err = (dqc.float() - ref).abs()
        assert (err <= 2e-2 + BF16_HALF_ULP_REL * ref.abs()).all(), f"rank {r}: dQ max err {err.max().item()}"
        dk_sum += dkc.float()
        dv_sum += dvc.float()
    torch.cuda.synchronize()
    assert fm.get_status() == 0
    for nm, s_, full in (("dK", dk_sum, dk), ("dV", dv_sum, dv)):
        err = (s_ - full.float()).abs()
        bound = 2e-2 + 4 * BF16_HALF_ULP_REL * full.float().abs()
        assert (err <= bound).all(), f"sum over zigzag ranks of {nm} vs full run: max err {err.max().item()}"
