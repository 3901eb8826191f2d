"""The checks build (libflashmask_checks.so, compiled with FLASHMASK_CHECKS):
mask values outside [0, Nq] are reported as FLASHMASK_ERR_BOUNDS in the status
word, in-range problems run clean and match the oracle.  Out-of-range values
are host-side inputs only (the release build applies them literally, and the
kernels never index with them).  Runs in a child process that loads the checks
library through FLASHMASK_LIBRARY=checks."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import numpy as np, torch
import column_sparse_masked_b200 as fm
import oracle
from _parity import make_case, check_out, check_lse, cuda
assert fm.lib_path().endswith("libflashmask_checks.so")
out = {}
# in range: a document mask, fwd + both backward modes, against the oracle
q, k, v, do, masks = make_case(1, 640, 640, 4, 2, 1, 128, "doc", 501)
o, lse = fm.fwd(*cuda(q, k, v), *cuda(*masks))
dq, dk, dv = fm.bwd(*cuda(q, k, v), o, lse, do.cuda(), *cuda(*masks))
torch.cuda.synchronize()
out["in_range_status"] = fm.get_status()
ro, rl = oracle.attention_forward(q, k, v, *masks)
check_out("O", o, ro); check_lse(lse, rl)
rdq, rdk, rdv = oracle.attention_backward(q, k, v, do, *masks)
check_out("dQ", dq, rdq); check_out("dK", dk, rdk); check_out("dV", dv, rdv)
# out of range (values in [-2, Nq + 3]): forward, backward and classify each report it
q, k, v, do, masks = make_case(1, 300, 300, 2, 1, 1, 64, "random", 502)
mg = cuda(*masks)
o, lse = fm.fwd(*cuda(q, k, v), *mg)
out["fwd_status"] = fm.get_status()
fm.bwd(*cuda(q, k, v), o, lse, do.cuda(), *mg)
out["bwd_status"] = fm.get_status()
fm.classify(*mg, Nq=300)
out["classify_status"] = fm.get_status()
# one bad value among in-range ones, then a clean call again
qq, kk, vv, _, good = make_case(1, 256, 256, 2, 2, 1, 128, "causal", 503)
assert all(int(g.min()) >= 0 and int(g.max()) <= 256 for g in good)
bad = [g.clone() for g in good]
bad[3][0, 0, 77] = 257  # UTE above Nq = 256
fm.fwd(*cuda(qq, kk, vv), *cuda(*bad))
out["one_bad_status"] = fm.get_status()
fm.fwd(*cuda(qq, kk, vv), *cuda(*good))
out["clean_again_status"] = fm.get_status()
print("RESULT " + json.dumps(out))
'''


def test_checks_build_reports_out_of_range_mask_values():
    from column_sparse_masked_b200 import build

    build.build(checks=True)
    env = dict(os.environ, FLASHMASK_LIBRARY="checks")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], capture_output=True, text=True, timeout=600, env=env,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    out = json.loads(line[len("RESULT "):])
    assert out["in_range_status"] == 0
    for key in ("fwd_status", "bwd_status", "classify_status", "one_bad_status"):
        assert out[key] == -9, (key, out)
    assert out["clean_again_status"] == 0
