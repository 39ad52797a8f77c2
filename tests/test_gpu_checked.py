"""The checked build (CSWATTN_CHECK=1: device-side bounds checks that record
an error flag instead of faulting) on the GPU: a forward+backward layer, a
decode step and a Newton-Schulz call run in a fresh process that loads
libcswattn_check.so; no check fires and the results match the float64
oracle at the usual tolerance."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
import numpy as np, torch
from causal_sliding_window_rope_b200.build import build
build(check=True)
import causal_sliding_window_rope_b200 as cs
assert cs.CHECKED and cs.LIB_PATH.endswith("libcswattn_check.so")
import oracle
from _helpers import make_inputs, oracle_layer, rel_frob, run_gpu
spec = cs.LayerSpec(2, 300, 6, 2, 128, 130, has_ve=True)
inp = make_inputs(2, 300, 6, 2, 128, True, "bf16", config=97)
got, _ = run_gpu(spec, inp)
_, ref = oracle_layer(spec, inp)
for k in ("O", "lse", "dq", "dk", "dv", "dve", "dgate"):
    assert rel_frob(got[k], ref[k]) <= 2e-2, k
X = (torch.randn(512, 256, dtype=torch.float64) / 30).to(torch.bfloat16)
Y = torch.empty_like(X).cuda()
ws = torch.empty(cs.muon_ns_workspace_bytes(512, 256), dtype=torch.uint8, device="cuda")
cs.muon_newton_schulz(X.cuda(), Y, oracle.POLAR_EXPRESS_PRINTED, ws)
cs.cswattn_sync_status()   # raises CswattnError(ERR_BOUNDS) if a check fired
r = oracle.newton_schulz(X.double().numpy(), oracle.POLAR_EXPRESS_PRINTED)
assert rel_frob(Y.double().cpu().numpy(), r) <= 2e-2
print("checked ok")
"""


def test_checked_build_runs_clean():
    env = dict(os.environ, CSWATTN_CHECK="1")
    r = subprocess.run([sys.executable, "-c", SCRIPT.replace("ROOT", repr(ROOT))], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "checked ok" in r.stdout
