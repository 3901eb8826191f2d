"""GPU parity: CUDA path (through the C ABI) vs the CPU oracle, element by
element, on seeded inputs that span several 128-tiles with ragged tails,
GQA, per-head masks, unmasked/causal/document/random/block-sparse masks and
fully masked rows.  Classification, localisation and pair counts bit-exact."""
import numpy as np
import pytest
import torch

import column_sparse_masked_b200 as fm
from column_sparse_masked_b200 import workloads as wl

from _parity import TOL_LSE, TOL_OUT, check_lse, check_out, cuda, make_case

pytestmark = pytest.mark.gpu

# (B, Nq, Nk, Hq, Hkv, Hm, d, mask kind, seed)
CASES = [
    (1, 256, 256, 2, 2, 1, 128, "causal", 11),
    (1, 384, 384, 2, 1, 1, 64, "none", 12),
    (1, 300, 300, 2, 1, 1, 64, "random", 13),
    (2, 517, 389, 4, 2, 1, 128, "random", 14),
    (1, 640, 640, 4, 4, 4, 128, "random", 15),
    (1, 1000, 1000, 4, 2, 1, 128, "doc", 16),
    (1, 200, 200, 2, 2, 1, 64, "fullrows", 17),
    (1, 1100, 1100, 2, 1, 1, 128, "blocksparse", 18),
    (1, 129, 1, 2, 2, 1, 128, "random", 19),
    (1, 1, 300, 2, 2, 1, 128, "random", 20),
]


def _ids(c):
    return f"B{c[0]}_q{c[1]}_k{c[2]}_h{c[3]}-{c[4]}-m{c[5]}_d{c[6]}_{c[7]}"


@pytest.fixture(scope="module")
def oracle_mod():
    import oracle

    oracle.build_oracle()
    return oracle


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_forward_backward_parity(oracle_mod, case, bwd_mode):
    B, Nq, Nk, Hq, Hkv, Hm, d, kind, seed = case
    q, k, v, do, masks = make_case(*case)
    qg, kg, vg, dog = cuda(q, k, v, do)
    mg = cuda(*masks)
    o, lse = fm.fwd(qg, kg, vg, *mg)
    dq, dk, dv = fm.bwd(qg, kg, vg, o, lse, dog, *mg)
    torch.cuda.synchronize()
    assert fm.get_status() == 0
    ro, rl = oracle_mod.attention_forward(q, k, v, *masks)
    cid = f"{_ids(case)}_{bwd_mode}"
    check_out("O", o, ro, case=cid)
    check_lse(lse, rl, case=cid)
    rdq, rdk, rdv = oracle_mod.attention_backward(q, k, v, do, *masks)
    check_out("dQ", dq, rdq, case=cid)
    check_out("dK", dk, rdk, case=cid)
    check_out("dV", dv, rdv, case=cid)


# Cases whose work items outnumber a capped persistent grid many times over:
# with 1-3 CTAs each CTA walks 5-32 items, so every item-to-item path of the
# three persistent kernels runs and is compared element by element: the
# 4-deep item ring wrapping round, the Q/O (Q/dO, K/V) buffer hand-over
# between items, the accumulator phase flips, zero-work items between real
# ones and the next item's L2 prefetch.
CAP_CASES = [
    (1, 1000, 1000, 4, 2, 1, 128, "doc", 16),      # 16 fwd / 16 key-side / 32 query-side items
    (1, 2048, 2048, 2, 1, 1, 64, "random", 91),    # d = 64: 16 / 16 / 32 items
    (2, 517, 389, 4, 2, 1, 128, "random", 14),     # ragged tails, two batches
    (1, 1100, 1100, 2, 1, 1, 128, "blocksparse", 18),  # zero-work key tiles between real ones
]


@pytest.mark.parametrize("cap", [1, 2, 3])
@pytest.mark.parametrize("case", CAP_CASES, ids=_ids)
def test_persistent_walk_parity(oracle_mod, case, cap, bwd_mode):
    q, k, v, do, masks = make_case(*case)
    qg, kg, vg, dog = cuda(q, k, v, do)
    mg = cuda(*masks)
    fm.set_max_ctas(cap)
    try:
        o, lse = fm.fwd(qg, kg, vg, *mg)
        dq, dk, dv = fm.bwd(qg, kg, vg, o, lse, dog, *mg)
        torch.cuda.synchronize()
    finally:
        fm.set_max_ctas(0)
    assert fm.get_status() == 0
    cid = f"{_ids(case)}_cap{cap}_{bwd_mode}"
    ro, rl = oracle_mod.attention_forward(q, k, v, *masks)
    check_out("O", o, ro, case=cid)
    check_lse(lse, rl, case=cid)
    rdq, rdk, rdv = oracle_mod.attention_backward(q, k, v, do, *masks)
    check_out("dQ", dq, rdq, case=cid)
    check_out("dK", dk, rdk, case=cid)
    check_out("dV", dv, rdv, case=cid)
    # the full grid computes the same bits (results do not depend on the grid;
    # in fused mode dQ's fp32 sums depend on the order reductions land in)
    o2, lse2 = fm.fwd(qg, kg, vg, *mg)
    dq2, dk2, dv2 = fm.bwd(qg, kg, vg, o2, lse2, dog, *mg)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    if bwd_mode == "split":
        assert torch.equal(dq, dq2)


@pytest.mark.parametrize("name", wl.CONFIG_ORDER)
def test_tile_costs_bit_exact_configs(oracle_mod, name):
    w = wl.CONFIGS[name]
    vecs = [torch.from_numpy(x) for x in wl.mask_vectors(w)]
    got = fm.tile_costs(*cuda(*vecs), Nq=w.N, Hq=w.Hq).cpu().numpy()
    ref = oracle_mod.tile_costs(*vecs, w.N, w.N, w.Hq)
    assert got.dtype == np.int64 and np.array_equal(got, ref)
    assert int(got.sum()) == fm.count_unmasked(*cuda(*vecs), Nq=w.N, Hq=w.Hq)


@pytest.mark.parametrize("seed", range(3))
def test_tile_costs_bit_exact_random(oracle_mod, seed):
    rng = np.random.default_rng(800 + seed)
    B, Hq = 2, 3
    nq, nk = int(rng.integers(1, 1200)), int(rng.integers(1, 900))
    per = [[wl.random_interval_vectors(rng, nq, nk, p_empty=0.3) for _ in range(Hq)] for _ in range(B)]
    vecs = [torch.from_numpy(np.ascontiguousarray(np.array([[per[b][h][t] for h in range(Hq)] for b in range(B)],
                                                           np.int32))) for t in range(4)]
    got = fm.tile_costs(*cuda(*vecs), Nq=nq, Hq=Hq).cpu().numpy()
    assert np.array_equal(got, oracle_mod.tile_costs(*vecs, nq, nk, Hq))
    # the chunk split fed from the library itself
    bounds, worst = fm.balance_chunks(got.tolist(), 4)
    best, _ = oracle_mod.balance_minimax(got.tolist(), 4) if got.size <= 12 else (worst, None)
    assert worst == best


def test_forward_is_deterministic():
    q, k, v, do, masks = make_case(1, 700, 700, 4, 2, 1, 128, "random", 31)
    qg, kg, vg = cuda(q, k, v)
    mg = cuda(*masks)
    o1, l1 = fm.fwd(qg, kg, vg, *mg)
    o2, l2 = fm.fwd(qg, kg, vg, *mg)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_none_pairs_mean_empty(oracle_mod):
    q, k, v, do, masks = make_case(1, 333, 333, 2, 2, 1, 128, "causal", 41)
    qg, kg, vg = cuda(q, k, v)
    mg = cuda(*masks)
    o_a, l_a = fm.fwd(qg, kg, vg, None, None, mg[2], mg[3])
    z = torch.zeros_like(mg[0])
    o_b, l_b = fm.fwd(qg, kg, vg, z, z, mg[2], mg[3])
    assert torch.equal(o_a, o_b) and torch.equal(l_a, l_b)


def test_empty_inputs():
    q, k, v, do, masks = make_case(1, 256, 256, 2, 2, 1, 128, "causal", 51)
    # Nk = 0: every row sees nothing -> O = 0, LSE = -inf, dQ = 0
    qg = q.cuda()
    k0 = torch.empty(1, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    m0 = [torch.empty(1, 1, 0, dtype=torch.int32, device="cuda") for _ in range(4)]
    o, lse = fm.fwd(qg, k0, k0, *m0)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    dq, dk, dv = fm.bwd(qg, k0, k0, o, lse, do.cuda(), *m0)
    assert torch.all(dq == 0) and dk.numel() == 0
    # Nq = 0: dK = dV = 0
    q0 = torch.empty(1, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    o0, l0 = fm.fwd(q0, k.cuda(), v.cuda(), *cuda(*masks))
    dq, dk, dv = fm.bwd(q0, k.cuda(), v.cuda(), o0, l0, q0, *cuda(*masks))
    assert torch.all(dk == 0) and torch.all(dv == 0)
    torch.cuda.synchronize()
    assert fm.get_status() == 0


@pytest.mark.parametrize("seed", range(4))
def test_classify_bit_exact(oracle_mod, seed):
    rng = np.random.default_rng(600 + seed)
    nq, nk = int(rng.integers(1, 1500)), int(rng.integers(1, 1500))
    vecs = [np.stack([x for x in wl.random_interval_vectors(rng, nq, nk, p_empty=0.4)])]
    vecs = [torch.from_numpy(np.ascontiguousarray(vecs[0][t][None, None])) for t in range(4)]
    got = fm.classify(*cuda(*vecs), Nq=nq).cpu().numpy()
    ref = oracle_mod.classify(*vecs, nq, nk)
    assert np.array_equal(got, ref)


def test_classify_golden_clauses_on_gpu():
    """The hand-derived golden of the tile rule (tests/golden/classify_clauses.json), on the GPU."""
    from test_oracle_pins import classify_golden

    vecs, nq, expect = classify_golden()
    got = fm.classify(*cuda(*[torch.from_numpy(x[None, None].copy()) for x in vecs]), Nq=nq).cpu().numpy()
    assert np.array_equal(got[0, 0], expect), np.argwhere(got[0, 0] != expect)


@pytest.mark.parametrize("name", wl.CONFIG_ORDER)
def test_classify_configs_bit_exact(oracle_mod, name):
    w = wl.CONFIGS[name]
    vecs = [torch.from_numpy(x) for x in wl.mask_vectors(w)]
    got = fm.classify(*cuda(*vecs), Nq=w.N).cpu().numpy()
    ref = oracle_mod.classify(*vecs, w.N, w.N)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("seed", range(3))
def test_localize_bit_exact(oracle_mod, seed):
    rng = np.random.default_rng(700 + seed)
    x = torch.from_numpy(rng.integers(-5, 5000, size=(3, 1, 1000)).astype(np.int32))
    for a, b in ((0, 1000), (128, 1024), (300, 301), (4000, 4000), (17, 3999)):
        got = fm.localize(x.cuda(), a, b).cpu().numpy()
        assert np.array_equal(got, oracle_mod.localize(x, a, b))
    chunks = [(0, 100), (250, 900), (1000, 1200), (3000, 4096)]
    got = fm.localize_multi(x.cuda(), chunks).cpu().numpy()
    assert np.array_equal(got, oracle_mod.localize_multi(x, chunks))


@pytest.mark.parametrize("name", ["tiny_doc", "doc8k", "sharequestion32k"])
def test_count_unmasked_matches_oracle(oracle_mod, name):
    w = wl.CONFIGS[name]
    vecs = [torch.from_numpy(x) for x in wl.mask_vectors(w)]
    got = fm.count_unmasked(*cuda(*vecs), Nq=w.N, Hq=w.Hq)
    assert got == oracle_mod.count_unmasked(*vecs, w.N, w.N, w.Hq)


def test_count_unmasked_random(oracle_mod):
    rng = np.random.default_rng(9)
    vv = wl.random_interval_vectors(rng, 500, 700)
    vecs = [torch.from_numpy(np.ascontiguousarray(np.stack([x, x[::-1]])[:, None])) for x in vv]
    got = fm.count_unmasked(*cuda(*vecs), Nq=500, Hq=3)
    assert got == oracle_mod.count_unmasked(*vecs, 500, 700, 3)


def test_bounded_wait_timeout_reports_status():
    """A wait on a barrier that nothing arrives on gives up and records the timeout."""
    assert fm.get_status() == 0
    fm.test_wait_timeout(2_000_000)  # 2 ms
    assert fm.get_status() == -6
    info = fm.get_timeout_info()
    assert info["kernel"] == "wait self-test" and info["barrier_offset"] == 0 and info["parity"] == 0
    assert info["block"] == 0 and info["thread"] == 0
    assert fm.get_status() == 0  # cleared
    q, k, v, do, masks = make_case(1, 256, 256, 2, 2, 1, 128, "causal", 61)
    o, lse = fm.fwd(*cuda(q, k, v), *cuda(*masks))
    torch.cuda.synchronize()
    assert fm.get_status() == 0 and torch.isfinite(lse).all()


def test_autograd_wrapper(oracle_mod):
    q, k, v, do, masks = make_case(1, 300, 300, 2, 2, 1, 128, "doc", 71)
    qg, kg, vg = [t.cuda().requires_grad_(True) for t in (q, k, v)]
    o = fm.flashmask_attention(qg, kg, vg, *cuda(*masks))
    o.backward(do.cuda())
    rdq, rdk, rdv = oracle_mod.attention_backward(q, k, v, do, *masks)
    check_out("dQ", qg.grad, rdq)
    check_out("dK", kg.grad, rdk)
    check_out("dV", vg.grad, rdv)


@pytest.mark.parametrize("name", ["doc8k", "sharequestion32k"])
def test_repeated_calls_never_time_out(name, bwd_mode):
    """Hundreds of back-to-back calls with a short wait limit: every barrier
    protocol keeps its waiters within one phase (a lost phase would hang a
    role until its bounded wait gives up and sets the status word)."""
    w = wl.CONFIGS[name]
    d = {k: v.cuda() for k, v in wl.make_inputs(w, with_grad=True).items()}
    m = [d[n] for n in ("lts", "lte", "uts", "ute")]
    fm.set_wait_limit_ns(100_000_000)
    try:
        o, lse = fm.fwd(d["q"], d["k"], d["v"], *m)
        dq, dk, dv = fm.bwd(d["q"], d["k"], d["v"], o, lse, d["do"], *m)
        for i in range(300):
            if i % 3 == 0:
                fm.fwd(d["q"], d["k"], d["v"], *m, out=(o, lse))
            fm.bwd(d["q"], d["k"], d["v"], o, lse, d["do"], *m, out=(dq, dk, dv))
        st = fm.get_status()
        assert st == 0, (st, fm.get_timeout_info())
        # the last results equal a fresh call's (deterministic, no stale state;
        # fused dQ: the same within the order of its fp32 additions)
        dq2, dk2, dv2 = fm.bwd(d["q"], d["k"], d["v"], o, lse, d["do"], *m)
        assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
        if bwd_mode == "split":
            assert torch.equal(dq, dq2)
        else:
            assert ((dq.float() - dq2.float()).abs() <= 1e-2 + 2.0 ** -7 * dq2.float().abs()).all()
    finally:
        fm.set_wait_limit_ns(0)


@pytest.mark.parametrize("name", ["doc8k", "sharequestion32k"])
def test_fused_and_split_backward_agree(name):
    """Both backward modes form the same bf16 P and dS values and accumulate dK and dV over the
    same q-tiles in the same order, so dK and dV agree bit for bit; dQ (fp32 reductions vs one
    on-chip sum per row) agrees to within fp32 rounding before the bf16 conversion."""
    w = wl.CONFIGS[name]
    d = {k: v.cuda() for k, v in wl.make_inputs(w, with_grad=True).items()}
    m = [d[n] for n in ("lts", "lte", "uts", "ute")]
    o, lse = fm.fwd(d["q"], d["k"], d["v"], *m)
    try:
        fm.set_bwd_mode("split")
        sq, sk, sv = fm.bwd(d["q"], d["k"], d["v"], o, lse, d["do"], *m)
        fm.set_bwd_mode("fused")
        fq, fk, fv = fm.bwd(d["q"], d["k"], d["v"], o, lse, d["do"], *m)
        torch.cuda.synchronize()
    finally:
        fm.set_bwd_mode("fused")
    assert fm.get_status() == 0
    assert torch.equal(fk, sk) and torch.equal(fv, sv)
    err = (fq.float() - sq.float()).abs()
    assert (err <= 1e-2 + 2.0 ** -7 * sq.float().abs()).all(), err.max().item()


PAIR_CASES = [c for c in CASES if c[5] == 1 and (c[3] // c[4]) % 2 == 0] + [
    (1, 1000, 1000, 8, 2, 1, 128, "doc", 21),   # two pairs per KV head
    (1, 129, 129, 4, 1, 4, 128, "random", 22),  # one mask per head: pairing not possible
]


@pytest.mark.parametrize("case", PAIR_CASES, ids=_ids)
def test_paired_forward_items_bit_identical(case):
    """Forward items of one q-tile of two q-heads (the default where the shape allows) compute
    exactly what items of two q-tiles of one q-head do: the tiles the latter add for a q-tile that
    skips them contribute exact zeros, so O and LSE agree bit for bit, with 1 CTA and all SMs."""
    q, k, v, do, masks = make_case(*case)
    qg, kg, vg = cuda(q, k, v)
    mg = cuda(*masks)
    try:
        for cap in (0, 1):
            fm.set_max_ctas(cap)
            fm.set_fwd_pairing(True)
            o1, l1 = fm.fwd(qg, kg, vg, *mg)
            fm.set_fwd_pairing(False)
            o2, l2 = fm.fwd(qg, kg, vg, *mg)
            torch.cuda.synchronize()
            assert fm.get_status() == 0
            assert torch.equal(o1, o2) and torch.equal(l1, l2), (case, cap)
    finally:
        fm.set_fwd_pairing(True)
        fm.set_max_ctas(0)


@pytest.mark.parametrize("name", ["doc8k", "docblocksparse128k"])
def test_paired_forward_items_workloads(name):
    """The same on the GQA workloads with one mask head."""
    w = wl.CONFIGS[name]
    d = {k: v.cuda() for k, v in wl.make_inputs(w, with_grad=False).items()}
    m = [d[n] for n in ("lts", "lte", "uts", "ute")]
    try:
        fm.set_fwd_pairing(True)
        o1, l1 = fm.fwd(d["q"], d["k"], d["v"], *m)
        fm.set_fwd_pairing(False)
        o2, l2 = fm.fwd(d["q"], d["k"], d["v"], *m)
        torch.cuda.synchronize()
    finally:
        fm.set_fwd_pairing(True)
    assert fm.get_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_pairing_setting():
    assert fm.get_fwd_pairing() is True
    fm.set_fwd_pairing(False)
    assert fm.get_fwd_pairing() is False
    fm.set_fwd_pairing(True)


def test_bwd_mode_setting():
    assert fm.get_bwd_mode() == "fused"
    fm.set_bwd_mode("split")
    assert fm.get_bwd_mode() == "split"
    fm.set_bwd_mode("fused")
    with pytest.raises(fm.FlashMaskError):
        fm.set_bwd_mode(7)
