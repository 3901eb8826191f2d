"""Context-parallel attention (column_sparse_masked_b200.cp): the pruned
point-to-point exchange and the per-rank computation.

CPU, gloo, world size 2 and 4: the product's exchange code with the local
attention, classification and localisation supplied by the oracle (test
infrastructure).  Every rank's O, LSE and dQ must equal the oracle's
full-sequence run on its rows, and every rank's dK, dV (its own contributions
plus those returned by the ranks that received its chunk) the full run's on
its keys.  The pruning plan must be sound (every chunk a rank's rows can see is
exchanged) and, on masks whose structure is tile-aligned, exact.

The GPU test emulates four ranks in one process with the library's kernels:
chunks a rank does not receive are filled with NaN in its K/V buffers, so a
kernel that read one would produce NaN.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from column_sparse_masked_b200 import cp
from column_sparse_masked_b200 import workloads as wl


class OracleOps:
    """Oracle-backed local steps for the host-logic tests (CPU tensors, fp64 results)."""

    def __init__(self):
        import oracle

        oracle.build_oracle()
        self.o = oracle

    def localize(self, x, a, b):
        return torch.from_numpy(self.o.localize(x, a, b))

    def classify(self, lts, lte, uts, ute, Nq, Nk):
        return self.o.classify(lts, lte, uts, ute, Nq, Nk)

    def fwd(self, q, k, v, masks, scale):
        o, lse = self.o.attention_forward(q, k, v, *masks, scale=scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def bwd(self, q, k, v, o, lse, do, masks, scale):
        dq, dk, dv = self.o.attention_backward(q, k, v, do, *masks, scale=scale)
        return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)

    def merge(self, o_parts, lse_parts):
        """The merge identity in fp64: lse = ln sum exp(lse_c), o = sum exp(lse_c - lse) o_c."""
        L = np.stack([x.numpy() for x in lse_parts])            # [n, B, Hq, Nq]
        m = L.max(0)
        fin = np.isfinite(m)
        w = np.where(fin[None], np.exp(L - np.where(fin, m, 0)[None]), 0.0)
        s_ = w.sum(0)
        lse = np.where(fin, np.where(fin, m, 0) + np.log(np.where(fin, s_, 1)), -np.inf)
        wn = w / np.where(fin, s_, 1)[None]                       # [n, B, Hq, Nq]
        o = sum(wn[c].transpose(0, 2, 1)[..., None] * o_parts[c].numpy() for c in range(len(o_parts)))
        return torch.from_numpy(o), torch.from_numpy(lse)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _case(seed, N=1024, B=1, Hq=2, Hkv=1, d=16, kind="doc"):
    rng = np.random.default_rng(seed)
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, N, Hq, d, generator=g)
    k = torch.randn(B, N, Hkv, d, generator=g)
    v = torch.randn(B, N, Hkv, d, generator=g)
    do = torch.randn(B, N, Hq, d, generator=g)
    if kind == "doc":
        vecs = wl.causal_document_vectors(wl.doc_lengths_uniform(rng, N, 60, 500))
    elif kind == "causal":
        vecs = wl.causal_vectors(N)
    elif kind == "docs_aligned":  # documents of whole 256-row chunks: nothing crosses chunks
        vecs = wl.causal_document_vectors([256] * (N // 256))
    else:
        vecs = wl.drop_key_tiles(wl.causal_document_vectors(wl.doc_lengths_uniform(rng, N, 100, 700)), rng, 0.3)
    masks = [torch.from_numpy(np.ascontiguousarray(np.repeat(x[None, None], B, 0))) for x in vecs]
    return q, k, v, do, masks


def _worker(rank, world, port, seed, kind, out, overlap=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        ops = OracleOps()
        q, k, v, do, masks = _case(seed, kind=kind)
        N = q.shape[1]
        plan = cp.make_plan(masks, N, cp.equal_bounds(N, world), ops=ops)
        a, b = plan.bounds[rank]
        att = cp.ContextParallelAttention(plan, rank, ops=ops, overlap=overlap)
        o, lse, ctx = att.forward(q[:, a:b].contiguous(), k[:, a:b].contiguous(), v[:, a:b].contiguous(), masks)
        dq, dk, dv = att.backward(ctx, do[:, a:b].contiguous())
        out[rank] = {"o": o.numpy(), "lse": lse.numpy(), "dq": dq.numpy(), "dk": dk.numpy(), "dv": dv.numpy(),
                     "need": plan.need, "transfers": plan.transfers()}
    finally:
        dist.destroy_process_group()


def _dense_visible(masks, N):
    """vis[i, j]: row i sees key j (batch 0, mask head 0)."""
    lts, lte, uts, ute = [m[0, 0].numpy()[None, :].astype(np.int64) for m in masks]
    i = np.arange(N)[:, None]
    return ~(((lts <= i) & (i < lte)) | ((uts <= i) & (i < ute)))


@pytest.mark.timeout(600)
@pytest.mark.parametrize("world,kind,seed,overlap", [(2, "doc", 1, False), (4, "doc", 2, False),
                                                     (4, "blocksparse", 3, False), (4, "causal", 4, False),
                                                     (4, "docs_aligned", 5, False), (2, "doc", 6, True),
                                                     (4, "blocksparse", 7, True)])
def test_context_parallel_equals_full_run(world, kind, seed, overlap):
    """overlap=True: each rank attends its own chunk while the exchange runs, then each received
    chunk, and merges the per-chunk results (the compute/communication overlap)."""
    import oracle

    oracle.build_oracle()
    q, k, v, do, masks = _case(seed, kind=kind)
    N = q.shape[1]
    ro, rl = oracle.attention_forward(q, k, v, *masks)
    rdq, rdk, rdv = oracle.attention_backward(q, k, v, do, *masks)
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, port, seed, kind, out, overlap), nprocs=world, join=True,
                       start_method="spawn")
    bounds = cp.equal_bounds(N, world)
    for r, (a, b) in enumerate(bounds):
        res = out[r]
        np.testing.assert_allclose(res["o"], ro[:, a:b], rtol=0, atol=1e-9)
        fin = np.isfinite(rl[:, :, a:b])
        assert np.array_equal(np.isneginf(res["lse"]), np.isneginf(rl[:, :, a:b]))
        np.testing.assert_allclose(res["lse"][fin], rl[:, :, a:b][fin], rtol=0, atol=1e-9)
        np.testing.assert_allclose(res["dq"], rdq[:, a:b], rtol=0, atol=1e-9)
        np.testing.assert_allclose(res["dk"], rdk[:, a:b], rtol=0, atol=1e-9)
        np.testing.assert_allclose(res["dv"], rdv[:, a:b], rtol=0, atol=1e-9)
    # the plan: identical on every rank, sound against the dense mask
    need = out[0]["need"]
    assert all(out[r]["need"] == need for r in range(world))
    vis = _dense_visible(masks, N)
    for r, (a, b) in enumerate(bounds):
        for c, (ac, bc) in enumerate(bounds):
            if vis[a:b, ac:bc].any():
                assert need[r][c], (r, c)
    if kind == "causal":  # rank r sees exactly chunks 0..r: half of an all-gather's transfers
        assert need == [[c <= r for c in range(world)] for r in range(world)]
        assert out[0]["transfers"] == world * (world - 1) // 2
    if kind == "docs_aligned":  # every document inside one chunk: no exchange at all
        assert out[0]["transfers"] == 0


def test_bounds_helpers():
    assert cp.equal_bounds(1000, 4) == [(0, 256), (256, 512), (512, 768), (768, 1000)]
    assert cp.equal_bounds(256, 4) == [(0, 0), (0, 128), (128, 128), (128, 256)]
    plan = cp.CPPlan(N=512, bounds=cp.equal_bounds(512, 2), need=[[True, False], [True, True]])
    assert plan.sources(1) == [0] and plan.sinks(0) == [1] and plan.sources(0) == [] and plan.transfers() == 1


@pytest.mark.gpu
@pytest.mark.parametrize("name,balanced", [("doc8k", False), ("docblocksparse128k", True)])
def test_context_parallel_emulated_ranks_on_gpu(name, balanced):
    """Four ranks emulated in one process with the library's kernels and the product's plan: each
    rank's K/V buffer holds its own chunk and the chunks the plan sends it, NaN everywhere else."""
    import column_sparse_masked_b200 as fm

    w = wl.CONFIGS[name]
    d = {n: t.cuda() for n, t in wl.make_inputs(w, with_grad=True).items()}
    m = [d[n] for n in ("lts", "lte", "uts", "ute")]
    o, lse = fm.fwd(d["q"], d["k"], d["v"], *m)
    dq, dk, dv = fm.bwd(d["q"], d["k"], d["v"], o, lse, d["do"], *m)
    world = 4
    bounds = cp.balanced_bounds(m, w.N, w.Hq, world) if balanced else cp.equal_bounds(w.N, world)
    plan = cp.make_plan(m, w.N, bounds)
    assert plan.transfers() < world * (world - 1)  # the mask prunes part of an all-gather
    dk_sum = torch.zeros_like(dk, dtype=torch.float32)
    dv_sum = torch.zeros_like(dv, dtype=torch.float32)
    for r, (a, b) in enumerate(bounds):
        kf = torch.full_like(d["k"], float("nan"))
        vf = torch.full_like(d["v"], float("nan"))
        for c in [r] + plan.sources(r):
            ac, bc = bounds[c]
            kf[:, ac:bc] = d["k"][:, ac:bc]
            vf[:, ac:bc] = d["v"][:, ac:bc]
        loc = [fm.localize(x, a, b) for x in m]
        qr, dor = d["q"][:, a:b].contiguous(), d["do"][:, a:b].contiguous()
        orr, lr = fm.fwd(qr, kf, vf, *loc)
        assert torch.equal(orr, o[:, a:b]) and torch.equal(lr, lse[:, :, a:b].contiguous()), f"rank {r}"
        dqr, dkr, dvr = fm.bwd(qr, kf, vf, orr, lr, dor, *loc)
        ref = dq[:, a:b].float()
        assert ((dqr.float() - ref).abs() <= 2e-2 + 2.0 ** -8 * ref.abs()).all(), f"rank {r}: dQ"
        # contributions only to the chunks the rank holds; exact zeros elsewhere
        for c, (ac, bc) in enumerate(bounds):
            if c != r and c not in plan.sources(r):
                assert torch.all(dkr[:, ac:bc] == 0) and torch.all(dvr[:, ac:bc] == 0), (r, c)
        dk_sum += dkr.float()
        dv_sum += dvr.float()
    torch.cuda.synchronize()
    assert fm.get_status() == 0
    for nm, s_, full in (("dK", dk_sum, dk), ("dV", dv_sum, dv)):
        err = (s_ - full.float()).abs()
        assert (err <= 2e-2 + 4 * 2.0 ** -8 * full.float().abs()).all(), f"{nm}: {err.max().item()}"


@pytest.mark.gpu
def test_merge_partials_equals_attention_over_the_union(oracle_mod):
    """Per-chunk forwards over disjoint key chunks (mask sliced on the key axis), merged by the
    library, equal the forward over all keys (and the oracle) within the parity tolerance; rows
    that see no key at all get O = 0, LSE = -inf."""
    import column_sparse_masked_b200 as fm

    from _parity import check_lse, check_out, make_case

    q, k, v, do, masks = make_case(2, 700, 900, 4, 2, 1, 128, "random", 901)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    mg = [m.cuda() for m in masks]
    o_full, l_full = fm.fwd(qg, kg, vg, *mg)
    cuts = [(0, 256), (256, 300), (300, 900)]
    parts = [fm.fwd(qg, kg[:, a:b].contiguous(), vg[:, a:b].contiguous(), *[m[:, :, a:b].contiguous() for m in mg])
             for a, b in cuts]
    o, lse = fm.merge_partials([x[0] for x in parts], [x[1] for x in parts])
    torch.cuda.synchronize()
    assert fm.get_status() == 0
    ro, rl = oracle_mod.attention_forward(q, k, v, *masks)
    check_out("O(merged)", o, ro, case="merge")
    check_lse(lse, rl, case="merge")
    err = (o.float() - o_full.float()).abs()
    assert (err <= 1e-2 + 2.0 ** -7 * o_full.float().abs()).all(), err.max().item()
    assert torch.equal(torch.isneginf(lse), torch.isneginf(l_full))
