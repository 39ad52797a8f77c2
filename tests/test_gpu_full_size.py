"""Full-size parity for the d12 / d24 / long-context workloads (configs 2-5),
every layer of each stack, in the launch configuration the benchmark times.

The oracle cannot redo a whole T=2048..8192 layer in seconds, so it computes
sampled rows one by one from the definition: query rows (O, lse, dQ) at tile
edges, the start and the end; key rows (dK, dV, dve, dgate) near the end of
the sequence and, for windowed layers, in the middle. The chain rule back
through RMSNorm/RoPE is evaluated per row by the oracle on a single token at
the row's position. Errors are relative Frobenius norms over the stacked
samples of each tensor (bar: 2e-2). The whole output is also checked finite.
"""
import numpy as np
import pytest
import torch

import causal_sliding_window_rope_b200 as cs
import oracle
from _helpers import f64, make_inputs, rel_frob, run_gpu

pytestmark = pytest.mark.gpu
TOL = 2e-2


def query_rows(B, H, T, rng):
    pts = sorted({0, 1, 63, 64, 127, 128, 129, T // 2, T - 129, T - 128, T - 2, T - 1})
    rows = []
    for b in sorted({0, B - 1}):
        for h in sorted({0, H - 1, int(rng.integers(0, H))}):
            rows += [(b, h, i) for i in pts if 0 <= i < T]
    return rows


def key_rows(B, Hk, T, W, rng):
    """Key rows at the sequence end, in the middle of windowed layers, and in
    the first key tiles: keys 0..129 are seen by every query of a full-causal
    layer (the heaviest tiles, whose steps the backward splits into parts)."""
    pts = {0, 1, 63, 64, 127, 128, 129, T - 1, T - 2, T - 128, T - 129}
    if W < T:
        pts.add(T // 2 + 3)
    rows = []
    for b in sorted({0, B - 1}):
        for hk in sorted({0, Hk - 1}):
            rows += [(b, hk, j) for j in sorted(pts) if 0 <= j < T]
    return rows


def chain_rule_row(L, t, q_row, k_row, ve_row, gate, dqt_row, dkt_row, dveff_row):
    """Per-row backward through the prologue at position t (oracle, one token)."""
    D = L.D
    has_ve = L.has_ve and ve_row is not None
    L1 = oracle.Layer(1, 1, 1, 1, D, 1, has_ve, rope_base=L.rope_base, eps=L.eps, pos_offset=t)
    shp = (1, 1, 1, D)
    r = oracle.prologue_bwd(L1, q_row.reshape(shp), k_row.reshape(shp),
                            ve_row.reshape(shp) if has_ve else None,
                            np.array(gate).reshape(1, 1, 1) if has_ve else None,
                            dqt_row.reshape(shp), dkt_row.reshape(shp), dveff_row.reshape(shp))
    dq, dk, dv, dve, dgate = r
    return (dq.reshape(D), dk.reshape(D), dv.reshape(D),
            None if dve is None else dve.reshape(D), None if dgate is None else float(dgate.reshape(())))


@pytest.mark.parametrize("config", [2, 3, 4, 5])
def test_full_size_layer_stack(config):
    w = cs.WORKLOADS[config]
    rng = np.random.default_rng(config)
    for layer, (W, ve) in enumerate(zip(w.windows, w.ve)):
        spec = cs.LayerSpec(w.B, w.T, w.H, w.Hk, w.D, W, has_ve=ve, dtype=w.dtype,
                            rope_base=w.rope_base, eps=w.eps)
        inp = make_inputs(w.B, w.T, w.H, w.Hk, w.D, ve, w.dtype, config=config, layer=layer,
                          dO_std=w.dO_std)
        got, _ = run_gpu(spec, inp)
        torch.cuda.empty_cache()
        for k, v in got.items():
            if v is not None:
                assert np.isfinite(v).all(), (config, layer, k)

        L = oracle.Layer(w.B, w.T, w.H, w.Hk, w.D, W, ve, rope_base=w.rope_base, eps=w.eps)
        x = {k: f64(v) for k, v in inp.items()}
        qt, kt, veff, rq, rk = oracle.prologue(L, x["q"], x["k"], x["v"], x["ve"], x["gate"])
        assert rel_frob(got["qt"], qt) < TOL and rel_frob(got["kt"], kt) < TOL
        assert rel_frob(got["veff"], veff) < TOL and rel_frob(got["rstd_q"], rq) < TOL
        assert rel_frob(got["rstd_k"], rk) < TOL

        qr = query_rows(w.B, w.H, w.T, rng)
        O, lse = oracle.fwd_rows(L, qt, kt, veff, qr)
        dqt = oracle.dq_rows(L, qt, kt, veff, x["dO"], qr)
        gO = np.stack([got["O"][b, i, h] for b, h, i in qr])
        glse = np.array([got["lse"][b, h, i] for b, h, i in qr])
        ref_dq, gdq = [], []
        for n, (b, h, i) in enumerate(qr):
            dq, *_ = chain_rule_row(L, i, x["q"][b, i, h], x["k"][b, i, 0], None, None,
                                    dqt[n], np.zeros(w.D), np.zeros(w.D))
            ref_dq.append(dq)
            gdq.append(got["dq"][b, i, h])
        errs = {"O": rel_frob(gO, O), "lse": rel_frob(glse, lse), "dq": rel_frob(gdq, ref_dq)}

        kr = key_rows(w.B, w.Hk, w.T, W, rng)
        dkt, dveff = oracle.dkv_rows(L, qt, kt, veff, x["dO"], kr)
        ref = {"dk": [], "dv": [], "dve": [], "dgate": []}
        gk = {"dk": [], "dv": [], "dve": [], "dgate": []}
        for n, (b, hk, j) in enumerate(kr):
            _, dk, dv, dve, dg = chain_rule_row(
                L, j, x["q"][b, j, 0], x["k"][b, j, hk], None if not ve else x["ve"][b, j, hk],
                None if not ve else x["gate"][b, j, hk], np.zeros(w.D), dkt[n], dveff[n])
            ref["dk"].append(dk)
            ref["dv"].append(dv)
            gk["dk"].append(got["dk"][b, j, hk])
            gk["dv"].append(got["dv"][b, j, hk])
            if ve:
                ref["dve"].append(dve)
                ref["dgate"].append(dg)
                gk["dve"].append(got["dve"][b, j, hk])
                gk["dgate"].append(got["dgate"][b, j, hk])
        for key in ("dk", "dv", "dve", "dgate"):
            if ref[key]:
                errs[key] = rel_frob(np.array(gk[key]), np.array(ref[key]))
        bad = {k: v for k, v in errs.items() if v > TOL}
        assert not bad, (config, layer, W, errs)
