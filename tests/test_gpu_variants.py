"""GPU parity for the layer variants the pages mention besides the five
workloads: another RoPE base (the autoresearch runs raised it from 10,000 to
50,000), a non-default softmax scale and other per-layer window patterns.

Page "weappnet.com" (section "Результаты": RoPE base 10,000 -> 50,000);
page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "1. GPT 모델"
(a per-layer window pattern string such as "SSSL").

Same bar as the other parity tests: relative Frobenius error <= 2e-2 per
output tensor against the float64 oracle on the bf16-rounded inputs.
"""
import numpy as np
import pytest

import causal_sliding_window_rope_b200 as cs
import oracle
from _helpers import OUT_KEYS, f64, make_inputs, rel_frob, run_gpu

pytestmark = pytest.mark.gpu
TOL = 2e-2


def check(spec, inp, scale=None):
    got, _ = run_gpu(spec, inp)
    L = oracle.Layer(spec.B, spec.T, spec.n_head, spec.n_kv_head, spec.head_dim, spec.window,
                     spec.has_ve, rope_base=spec.rope_base, eps=spec.eps, scale=scale)
    ref = oracle.layer(L, *(f64(inp[k]) for k in ("q", "k", "v", "ve", "gate", "dO")))
    errs = {k: rel_frob(got[k], ref[k]) for k in OUT_KEYS if ref[k] is not None}
    for k in ("qt", "kt"):
        errs[k] = rel_frob(got[k], ref[k])
    bad = {k: v for k, v in errs.items() if not np.isfinite(v) or v > TOL}
    assert not bad, (spec, errs)
    return errs


@pytest.mark.parametrize("base", [50000.0, 500000.0])
@pytest.mark.parametrize("D", [128, 64])
def test_rope_base(base, D):
    spec = cs.LayerSpec(2, 384, 6, 2, D, 200, has_ve=True, dtype="bf16", rope_base=base)
    inp = make_inputs(2, 384, 6, 2, D, True, "bf16", config=80, layer=D % 9)
    check(spec, inp)


def test_rope_base_changes_the_result():
    """The base reaches the kernels: base 50000 and base 10000 give
    different rotated keys on the same inputs."""
    inp = make_inputs(1, 256, 2, 1, 128, False, "bf16", config=81)
    a, _ = run_gpu(cs.LayerSpec(1, 256, 2, 1, 128, 256, has_ve=False, rope_base=10000.0), inp)
    b, _ = run_gpu(cs.LayerSpec(1, 256, 2, 1, 128, 256, has_ve=False, rope_base=50000.0), inp)
    assert rel_frob(a["kt"], b["kt"]) > 1e-2


def test_softmax_scale():
    spec = cs.LayerSpec(1, 300, 4, 2, 128, 150, has_ve=True, dtype="bf16", softmax_scale=0.05)
    inp = make_inputs(1, 300, 4, 2, 128, True, "bf16", config=82)
    check(spec, inp, scale=0.05)


@pytest.mark.parametrize("pattern,short,long", [("SSL", 96, 512), ("SL", 129, 300), ("L", 64, 640)])
def test_window_patterns(pattern, short, long):
    """A small stack per pattern: every layer with its own window and inputs."""
    windows = cs.window_pattern(pattern, short, long, 3)
    for i, W in enumerate(windows):
        spec = cs.LayerSpec(1, 640, 4, 2, 128, W, has_ve=i % 2 == 1, dtype="bf16")
        inp = make_inputs(1, 640, 4, 2, 128, i % 2 == 1, "bf16", config=83, layer=i)
        check(spec, inp)
