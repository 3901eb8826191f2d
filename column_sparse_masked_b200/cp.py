"""Context-parallel masked attention: the sequence is split into one contiguous
chunk of query rows (and the same key columns) per rank, and each rank computes
attention of its rows against every key it can see.

"FlashMask-3 targets masked distributed attention on Hopper GPUs", section
"In-depth insight": each rank derives its mask from the global column-wise
vectors without communication (clip-shift-max localisation, ``localize``), and
the K/V exchange is pruned by the mask.  Here the pruning decision comes from
the same tile classification the kernels use: rank r needs key chunk c only if
some (q-tile of r, k-tile of c) pair is not skipped.  Every rank computes every
rank's needs from the O(n) vectors (no exchange), so all ranks agree on one
point-to-point schedule:

  forward   rank c sends its K/V chunk to each rank r != c that needs it;
            each rank runs the forward of its rows against the gathered K/V
            (chunks it did not receive are never read: all their tiles are
            skipped for its rows);
  backward  each rank runs the backward of its rows, keeps its dQ, and sends
            the dK/dV contributions of every received chunk back to the
            chunk's owner, which sums them (fp32) with its own.

With ``overlap=True`` the forward attends the rank's own key chunk while the
exchange is in flight (its rows against its own keys need nothing from other
ranks), then each received chunk, and merges the per-chunk results per row
(``flashmask_merge_partials``: lse = ln sum exp(lse_c), o = sum exp(lse_c -
lse) o_c, exact up to the rounding of the bf16 partials).  The backward then
runs once on the gathered K/V with the merged O and LSE.

The exchange uses torch.distributed point-to-point operations (NCCL between
GPUs, one process per GPU; gloo on CPU for the host-logic tests) into this
rank's own buffers; no kernel reads another GPU's memory.  A plain
all-gather / reduce-scatter is the special case where every rank needs every
chunk.  The chunk split can be balanced by unmasked-pair work
(``balanced_bounds``: per-q-tile costs from the library, exact minimax split).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import torch

TILE = 128


@dataclass
class CPPlan:
    """Chunk of each rank and the pruned exchange pattern (identical on every rank)."""

    N: int
    bounds: List[Tuple[int, int]]                       # rank r owns rows/keys [a_r, b_r)
    need: List[List[bool]] = field(default_factory=list)  # need[r][c]: rank r's rows see chunk c

    @property
    def world(self) -> int:
        return len(self.bounds)

    def sources(self, r: int) -> List[int]:
        """Chunks rank r receives (needed, not its own)."""
        return [c for c in range(self.world) if c != r and self.need[r][c]]

    def sinks(self, c: int) -> List[int]:
        """Ranks that receive rank c's chunk."""
        return [r for r in range(self.world) if r != c and self.need[r][c]]

    def transfers(self) -> int:
        """KV chunk transfers of one forward (an all-gather has world * (world - 1))."""
        return sum(len(self.sources(r)) for r in range(self.world))


class LibraryOps:
    """The library's device entry points (the product path)."""

    def __init__(self):
        from . import _binding as b

        self.b = b

    def localize(self, x, a, b):
        return self.b.localize(x, a, b)

    def classify(self, lts, lte, uts, ute, Nq, Nk):
        return self.b.classify(lts, lte, uts, ute, Nq=Nq, Nk=Nk)

    def fwd(self, q, k, v, masks, scale):
        return self.b.fwd(q, k, v, *masks, scale=scale)

    def bwd(self, q, k, v, o, lse, do, masks, scale):
        return self.b.bwd(q, k, v, o, lse, do, *masks, scale=scale)

    def merge(self, o_parts, lse_parts):
        return self.b.merge_partials(o_parts, lse_parts)


def equal_bounds(N: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous chunks of whole 128-row tiles, as equal in length as possible."""
    nt = -(-N // TILE)
    cuts = [min(N, (nt * r // world) * TILE) for r in range(world + 1)]
    cuts[-1] = N
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def balanced_bounds(masks: Sequence[torch.Tensor], N: int, Hq: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous chunks of whole tiles with the most even unmasked-pair work (exact minimax),
    from the library's per-q-tile costs (the page's sparsity-aware balancer, read as equalising
    the ranks' unmasked pairs)."""
    from . import _binding as b

    costs = b.tile_costs(*masks, Nq=N, Hq=Hq).cpu().tolist()
    tb, _ = b.balance_chunks(costs, world)
    return [(min(N, tb[r] * TILE), min(N, tb[r + 1] * TILE)) for r in range(world)]


def make_plan(masks: Sequence[Optional[torch.Tensor]], N: int, bounds: List[Tuple[int, int]],
              ops=None) -> CPPlan:
    """need[r][c] for every pair of ranks, from the tile classes of each rank's localised mask
    against all N keys (the same rule and the same vectors the kernels use)."""
    ops = ops or LibraryOps()
    world = len(bounds)
    nkt = -(-N // TILE)
    need = []
    for r, (a, b) in enumerate(bounds):
        if b <= a:
            need.append([False] * world)
            continue
        loc = [None if m is None else ops.localize(m, a, b) for m in masks]
        if loc[0] is None and loc[2] is None:  # no intervals at all: every tile is full
            need.append([bounds[c][1] > bounds[c][0] for c in range(world)])
            continue
        cls = torch.as_tensor(ops.classify(*loc, Nq=b - a, Nk=N))
        kt_any = (cls != 0).reshape(-1, nkt).any(dim=0).cpu()  # over batch, mask head, q-tile
        row = []
        for c, (ac, bc) in enumerate(bounds):
            row.append(bool(bc > ac and kt_any[ac // TILE:-(-bc // TILE)].any()))
        need.append(row)
    return CPPlan(N=N, bounds=list(bounds), need=need)


def _p2p(ops_list):
    """Issues the point-to-point operations together and waits for all of them."""
    import torch.distributed as dist

    if not ops_list:
        return
    for req in dist.batch_isend_irecv(ops_list):
        req.wait()


class ContextParallelAttention:
    """One rank's side of context-parallel masked attention (see the module docstring).

    ``q``, ``k``, ``v`` (and ``do``) are this rank's chunk, [B, b - a, H, d]; ``masks`` are the
    GLOBAL boundary vectors [B, Hm, N] (replicated: O(n) per rank).  ``ops`` defaults to the
    library's kernels; ``poison_unreceived`` fills the K/V rows of chunks this rank does not
    receive with NaN (a check that pruned chunks are never read).
    """

    def __init__(self, plan: CPPlan, rank: int, ops=None, group=None, poison_unreceived: bool = False,
                 overlap: bool = False):
        self.plan, self.rank, self.group = plan, rank, group
        self.ops = ops or LibraryOps()
        self.poison = poison_unreceived
        self.overlap = overlap
        self.peer = (lambda r: r) if group is None else (lambda r: _group_rank(group, r))

    def forward(self, q, k, v, masks, scale: Optional[float] = None):
        import torch.distributed as dist

        plan, r = self.plan, self.rank
        a, b = plan.bounds[r]
        B, _, H, d = k.shape
        N = plan.N
        k_full = torch.empty(B, N, H, d, dtype=k.dtype, device=k.device)
        v_full = torch.empty_like(k_full)
        if self.poison:
            k_full.fill_(float("nan"))
            v_full.fill_(float("nan"))
        k_full[:, a:b] = k
        v_full[:, a:b] = v
        ops, recv = [], []
        kc, vc = k.contiguous(), v.contiguous()
        for dst in plan.sinks(r):  # my chunk to every rank that needs it
            ops += [dist.P2POp(dist.isend, kc, self.peer(dst), self.group),
                    dist.P2POp(dist.isend, vc, self.peer(dst), self.group)]
        for src in plan.sources(r):  # the chunks my rows see
            ac, bc = plan.bounds[src]
            kb = torch.empty(B, bc - ac, H, d, dtype=k.dtype, device=k.device)
            vb = torch.empty_like(kb)
            ops += [dist.P2POp(dist.irecv, kb, self.peer(src), self.group),
                    dist.P2POp(dist.irecv, vb, self.peer(src), self.group)]
            recv.append((ac, bc, kb, vb))
        loc = [None if m is None else self.ops.localize(m, a, b) for m in masks]
        if not self.overlap:
            _p2p(ops)
            for ac, bc, kb, vb in recv:
                k_full[:, ac:bc] = kb
                v_full[:, ac:bc] = vb
            o, lse = self.ops.fwd(q, k_full, v_full, loc, scale)
        else:
            works = dist.batch_isend_irecv(ops) if ops else []
            # own rows against own keys while the exchange is in flight
            own = [None if m is None else self.ops.localize(m[:, :, a:b].contiguous(), a, b) for m in masks]
            parts = [self.ops.fwd(q, k, v, own, scale)]
            for wk in works:
                wk.wait()
            for ac, bc, kb, vb in recv:  # then each received chunk, merged per row
                k_full[:, ac:bc] = kb
                v_full[:, ac:bc] = vb
                loc_c = [None if m is None else self.ops.localize(m[:, :, ac:bc].contiguous(), a, b) for m in masks]
                parts.append(self.ops.fwd(q, kb, vb, loc_c, scale))
            if len(parts) == 1:
                o, lse = parts[0]
            else:
                o, lse = self.ops.merge([x[0] for x in parts], [x[1] for x in parts])
        ctx = {"q": q, "k_full": k_full, "v_full": v_full, "loc": loc, "o": o, "lse": lse, "scale": scale}
        return o, lse, ctx

    def backward(self, ctx, do):
        import torch.distributed as dist

        plan, r = self.plan, self.rank
        a, b = plan.bounds[r]
        dq, dk_full, dv_full = self.ops.bwd(ctx["q"], ctx["k_full"], ctx["v_full"], ctx["o"], ctx["lse"], do,
                                            ctx["loc"], ctx["scale"])
        acc_dtype = torch.float64 if dk_full.dtype == torch.float64 else torch.float32
        dk = dk_full[:, a:b].to(acc_dtype)
        dv = dv_full[:, a:b].to(acc_dtype)
        ops, recv = [], []
        for src in plan.sources(r):  # contributions to the chunks I received go back to their owners
            ac, bc = plan.bounds[src]
            ops += [dist.P2POp(dist.isend, dk_full[:, ac:bc].contiguous(), self.peer(src), self.group),
                    dist.P2POp(dist.isend, dv_full[:, ac:bc].contiguous(), self.peer(src), self.group)]
        for dst in plan.sinks(r):  # ranks that received my chunk return their contributions
            kb = torch.empty(dk_full.shape[0], b - a, *dk_full.shape[2:], dtype=dk_full.dtype, device=dk_full.device)
            vb = torch.empty_like(kb)
            ops += [dist.P2POp(dist.irecv, kb, self.peer(dst), self.group),
                    dist.P2POp(dist.irecv, vb, self.peer(dst), self.group)]
            recv.append((kb, vb))
        _p2p(ops)
        for kb, vb in recv:
            dk += kb.to(acc_dtype)
            dv += vb.to(acc_dtype)
        return dq, dk.to(dk_full.dtype), dv.to(dv_full.dtype)


def _group_rank(group, r: int) -> int:
    import torch.distributed as dist

    return dist.get_global_rank(group, r)
