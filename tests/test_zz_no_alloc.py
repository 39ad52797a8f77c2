"""attn_bwd_noalloc, the backward entry point for callers that cannot allocate
device memory (their memory belongs to another allocator, or cudaMalloc's
device synchronization is not allowed in their step loop). Its scratch is a
fixed array inside the library instead of a caller workspace.

The test calls it through the C ABI twice in a row on the same inputs and
compares both results with attn_bwd given an ordinary caller workspace, at
the tolerance of the parity tests (relative Frobenius 2e-2 for bf16, max-abs
1e-4 for fp32). Between the two calls another layer of a different shape
(longer sequence, other window, other number of backward parts) runs
through the same array, so the second call starts from scratch contents
that a different layout left behind, as it would when several layers share
the array in a training step. It allocates its own tensors, so it passes
alone in a fresh process and after the other tests. This file is collected
last on purpose.
"""
import numpy as np
import pytest
import torch

import causal_sliding_window_rope_b200 as cs
from _helpers import make_inputs, max_abs, rel_frob

pytestmark = pytest.mark.gpu

GRAD_NAMES = ("dQ", "dK", "dV", "dve", "dgate")


def _forward(spec, dtype, config):
    B, T, H, Hk, D = spec.B, spec.T, spec.n_head, spec.n_kv_head, spec.head_dim
    inp = make_inputs(B, T, H, Hk, D, spec.has_ve, dtype, config=config)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    buf = cs.LayerBuffers(spec)
    cs.layer_forward(spec, buf, dev["q"], dev["k"], dev["v"], dev["ve"], dev["gate"])
    return dev, buf


def _noalloc(spec, dev, buf, out):
    cs.attn_bwd_noalloc(spec, dev["q"], dev["k"], dev["ve"], dev["gate"], buf.q_out,
                        buf.k_out, buf.v_out, buf.rstd_q, buf.rstd_k, buf.O, buf.lse,
                        dev["dO"], out["dQ"], out["dK"], out["dV"], out.get("dve"),
                        out.get("dgate"))


def _run_both(spec, dtype, config, other=None):
    dev, buf = _forward(spec, dtype, config)
    cs.layer_backward(spec, buf, dev["q"], dev["k"], dev["ve"], dev["gate"], dev["dO"])
    cs.cswattn_sync_status()
    ref = {n: getattr(buf, n).clone() for n in GRAD_NAMES if getattr(buf, n) is not None}
    results = []
    for call in range(2):
        out = {n: torch.full_like(t, float("nan")) for n, t in ref.items()}
        _noalloc(spec, dev, buf, out)
        cs.cswattn_sync_status()
        torch.cuda.synchronize()
        results.append(out)
        if call == 0 and other is not None:
            # Another layer through the same array, different layout.
            odev, obuf = _forward(other, dtype, config + 1)
            oout = {n: torch.empty_like(getattr(obuf, n)) for n in GRAD_NAMES
                    if getattr(obuf, n) is not None}
            _noalloc(other, odev, obuf, oout)
            cs.cswattn_sync_status()
            torch.cuda.synchronize()
            assert all(torch.isfinite(t.float()).all() for t in oout.values())
    return ref, results


def test_noalloc_bf16_matches_workspace_entry_point_twice():
    spec = cs.LayerSpec(2, 300, 6, 2, 128, 130, has_ve=True, dtype="bf16")
    other = cs.LayerSpec(1, 1000, 4, 1, 128, 1000, has_ve=False, dtype="bf16")
    for s in (spec, other):
        assert cs.attn_bwd_workspace_bytes(s) <= cs.NOALLOC_SCRATCH_BYTES
    ref, results = _run_both(spec, "bf16", config=95, other=other)
    for out in results:
        for n, r in ref.items():
            got = out[n].double().cpu().numpy()
            assert np.isfinite(got).all(), n
            assert rel_frob(got, r.double().cpu().numpy()) <= 2e-2, n


def test_noalloc_f32_matches_workspace_entry_point_twice():
    spec = cs.LayerSpec(32, 16, 4, 4, 4, 16, has_ve=False, dtype="f32")
    other = cs.LayerSpec(4, 64, 2, 1, 4, 7, has_ve=True, dtype="f32")
    ref, results = _run_both(spec, "f32", config=96, other=other)
    for out in results:
        for n, r in ref.items():
            assert max_abs(out[n].cpu().numpy(), r.cpu().numpy()) <= 1e-4, n


def test_noalloc_rejects_layers_beyond_the_fixed_scratch():
    spec = cs.LayerSpec(4, 2048, 12, 4, 128, 1024, has_ve=True, dtype="bf16")
    assert cs.attn_bwd_workspace_bytes(spec) > cs.NOALLOC_SCRATCH_BYTES
    with pytest.raises(cs.CswattnError) as err:
        cs.attn_bwd_noalloc(spec, *([256] * 17))
    assert err.value.status == cs.ERR_UNSUPPORTED
    assert "scratch" in str(err.value)
