"""The attention kernels' barrier protocols, checked on a randomised model (CPU only).

``protocol_model.py`` restates each kernel's wait / arrive / issue sequence.
Every real protocol must finish without deadlock, phase skew or buffer hazard
on many random schedules; each planted protocol mistake (applied to a copy of
the model's source) must be caught, which shows that the checks can fail.
One of them is the query-side kernel's earlier bug: a single "dS written"
barrier that the compute warps could advance two phases past the MMA warp's
wait.

Not among them: dropping the MMA warp's wait for the accumulator's release
(O, dQ, dK/dV) at an item's first step.  In these kernels the same warps that
read the accumulator out also produce the next item's first P or dS, so the
MMA warp's wait for that operand already orders the accumulator's reuse; the
model finds those waits redundant here.  They are kept so that the release
stays explicit.  The fused backward's dQ is the exception: a separate warpgroup
reads it out, so there the wait for its release is necessary, and dropping it is
one of the planted mistakes below.
"""
import os
import random
import types

import pytest

import protocol_model as pm

SRC = os.path.join(os.path.dirname(__file__), "protocol_model.py")


@pytest.mark.parametrize("name", sorted(pm.MODELS))
def test_protocol_is_safe(name):
    rng = random.Random(100)
    for seed in range(1500):
        pm.MODELS[name](pm.random_items(rng), seed)


MUTATIONS = [
    ("fwd", "S(t+1) issued before P(t) was consumed",
     [('                yield wait(f"slot_full{sv}", (pos + 1) // SLOTS)\n                yield wait("p_full0", tile)\n',
       '                yield wait(f"slot_full{sv}", (pos + 1) // SLOTS)\n                if t + 1 < n:\n'
       '                    yield wait(f"slot_full{sk2}", (pos + 2) // SLOTS)\n'
       '                    sim.pipe.append(("mma", op_s(0, j, t + 1, sk2)))\n                yield wait("p_full0", tile)\n')]),
    ("fwd", "O committed before the item's last P V",
     [('                sim.pipe.append(("mma", op_pv(0, j, t, sv)))\n                if t == n - 1:\n'
       '                    sim.pipe.append(("commit", "o_full0"))\n',
       '                if t == n - 1:\n                    sim.pipe.append(("commit", "o_full0"))\n'
       '                sim.pipe.append(("mma", op_pv(0, j, t, sv)))\n')]),
    ("fwd", "V slot released before its last P V",
     [('                sim.pipe.append(("mma", op_pv(1, j, t, sv)))\n                if t == n - 1:\n'
       '                    sim.pipe.append(("commit", "o_full1"))\n                sim.pipe.append(("commit", f"slot_empty{sv}"))\n',
       '                sim.pipe.append(("commit", f"slot_empty{sv}"))\n                sim.pipe.append(("mma", op_pv(1, j, t, sv)))\n'
       '                if t == n - 1:\n                    sim.pipe.append(("commit", "o_full1"))\n')]),
    ("fwd", "item ring released by too few readers",
     [('        sim.bar(f"ring_empty{i}", 1 + 2)  # MMA + the two softmax groups', '        sim.bar(f"ring_empty{i}", 1 + 1)')]),
    ("dq", "single dS barrier waited by tile index (the earlier bug)",
     [('                yield wait(f"ds_full{tj & 1}", tj >> 1)\n', '                yield wait("ds_full0", tj)\n'),
      ('                sim.arrive(f"ds_full{b}")\n', '                sim.arrive("ds_full0")\n')]),
    ("dq", "dQ handed to the epilogue before the item's last dQ step",
     [('                sim.pipe += [("mma", op_dq(j, t, tj, ks)), ("commit", f"k_empty{ks}")]',
       '                if t == n - 1:\n                    sim.pipe.append(("commit", "dq_full"))\n'
       '                sim.pipe += [("mma", op_dq(j, t, tj, ks)), ("commit", f"k_empty{ks}")]'),
      ('            act += 1\n            sim.pipe.append(("commit", "dq_full"))\n', '            act += 1\n')]),
    ("dq", "dP(t+1) issued before the compute warps hold dP(t)",
     [('                    yield wait("dp_read", tj)\n', '')]),
    ("dq", "K stage released before its dQ step",
     [('                sim.pipe += [("mma", op_dq(j, t, tj, ks)), ("commit", f"k_empty{ks}")]',
       '                sim.pipe += [("commit", f"k_empty{ks}"), ("mma", op_dq(j, t, tj, ks))]')]),
    ("dkdv", "S^T(t+1) issued before dV(t) read P^T(t)",
     [('                yield wait("p_full", tj)\n                sim.pipe += [("mma", op_dv(j, t, tj, ds)), ("commit", f"do_empty{ds}")]\n'
       '                if t + 1 < n:\n                    yield wait(f"q_full{qs2}", (sj + 1) // QST)\n'
       '                    sim.pipe += [("mma", op_s(j, t + 1, tj + 1, qs2)), ("commit", "s_full")]\n'
       '                    if t + 2 == n:\n                        sim.pipe.append(("commit", "k_empty"))\n',
       '                if t + 1 < n:\n                    yield wait(f"q_full{qs2}", (sj + 1) // QST)\n'
       '                    sim.pipe += [("mma", op_s(j, t + 1, tj + 1, qs2)), ("commit", "s_full")]\n'
       '                    if t + 2 == n:\n                        sim.pipe.append(("commit", "k_empty"))\n'
       '                yield wait("p_full", tj)\n                sim.pipe += [("mma", op_dv(j, t, tj, ds)), ("commit", f"do_empty{ds}")]\n')]),
    ("dkdv", "dV/dK handed to the epilogue before the item's last dK step",
     [('                sim.pipe += [("mma", op_dk(j, t, tj, qs)), ("commit", f"q_empty{qs}")]\n'
       '                if t + 1 < n:\n                    yield wait(f"do_full{ds2}"',
       '                if t == n - 1:\n                    sim.pipe.append(("commit", "dkdv_full"))\n'
       '                sim.pipe += [("mma", op_dk(j, t, tj, qs)), ("commit", f"q_empty{qs}")]\n'
       '                if t + 1 < n:\n                    yield wait(f"do_full{ds2}"'),
      ('            act += 1\n            sim.pipe.append(("commit", "dkdv_full"))\n', '            act += 1\n')]),
    ("dkdv", "Q stage released before its dK step",
     [('                sim.pipe += [("mma", op_dk(j, t, tj, qs)), ("commit", f"q_empty{qs}")]\n'
       '                if t + 1 < n:\n                    yield wait(f"do_full{ds2}"',
       '                sim.pipe += [("commit", f"q_empty{qs}"), ("mma", op_dk(j, t, tj, qs))]\n'
       '                if t + 1 < n:\n                    yield wait(f"do_full{ds2}"')]),
    ("fused", "dP^T(t+1) issued before dQ(t) was read out of its region",
     [('                    yield wait("dq_free", tj)\n', '')]),
    ("fused", "an item's first dP^T issued before the previous item's last dQ was read out",
     [('            if tc > 0:\n                yield wait("dq_free", tc - 1)\n', '')]),
    ("fused", "dQ(t) issued before dK(t) read dS^T(t) from the same TMEM columns",
     [('                sim.pipe += [("mma", op_dk(j, t, tj, qs)), ("commit", f"q_empty{qs}")]\n'
       '                sim.pipe += [("mma", op_dq(j, t, tj)), ("commit", "dq_full")]\n',
       '                sim.pipe += [("mma", op_dq(j, t, tj)), ("commit", "dq_full")]\n'
       '                sim.pipe += [("mma", op_dk(j, t, tj, qs)), ("commit", f"q_empty{qs}")]\n')]),
    ("fused", "K released before the item's last dQ",
     [('                sim.pipe += [("mma", op_dq(j, t, tj)), ("commit", "dq_full")]\n'
       '                if t + 1 == n:\n                    sim.pipe.append(("commit", "k_empty"))\n',
       '                if t + 1 == n:\n                    sim.pipe.append(("commit", "k_empty"))\n'
       '                sim.pipe += [("mma", op_dq(j, t, tj)), ("commit", "dq_full")]\n')]),
    ("fused", "dS(t+1) written over dQ(t) staged in the dS buffer before its reduction read it",
     [('                if tc > 0:\n                    yield wait("dsbuf_free", tc - 1)  # the reduction has read dQ(tc-1) staged there\n', '')]),
    ("fused", "dQ(t+1) staged before the previous reductions read the buffers",
     [('                if tc > 0:\n                    yield wait("buf_free", tc - 1)\n', '')]),
    ("fused", "dQ region freed before the drain read it",
     [('                yield STEP\n                st["dP"] = [("used", tc), ("used", tc)]\n                sim.arrive("dq_free")\n',
       '                sim.arrive("dq_free")\n                yield STEP\n                st["dP"] = [("used", tc), ("used", tc)]\n')]),
    ("dkdv", "P^T counted complete after one warpgroup",
     [('    for nm in ("p_full", "ds_full", "dkdv_free"):\n        sim.bar(nm, 2)\n',
       '    for nm in ("ds_full", "dkdv_free"):\n        sim.bar(nm, 2)\n    sim.bar("p_full", 1)\n')]),
]


@pytest.mark.parametrize("model,name,edits", MUTATIONS, ids=[f"{m[0]}-{m[1]}" for m in MUTATIONS])
def test_planted_protocol_mistake_is_caught(model, name, edits):
    with open(SRC) as f:
        text = f.read()
    for old, new in edits:
        assert text.count(old) == 1, f"{name}: the text to change must occur exactly once"
        text = text.replace(old, new)
    mod = types.ModuleType("protocol_model_variant")
    exec(compile(text, SRC, "exec"), mod.__dict__)
    rng = random.Random(200)
    for seed in range(3000):
        try:
            mod.MODELS[model](mod.random_items(rng), seed)
        except mod.Hazard:
            return
    pytest.fail(f"{name}: no schedule exposed the planted mistake")
