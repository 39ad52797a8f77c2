"""GPU parity of the value-embedding gate computed from the block input:
attn_prologue_gated (gate logits = x[..., :C] @ w_gate.T inside the fused
prologue) and attn_gate_bwd (dx and dw_gate from the attention backward's
dgate), against the float64 oracle on the same seeded inputs.

Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "1. GPT 모델",
value-embedding code (gate = 3*sigmoid(ve_gate(x[..., :ve_gate_channels]))).
Tolerances as elsewhere: relative Frobenius <= 2e-2 (bf16), max-abs 1e-4 (fp32).
"""
import numpy as np
import pytest
import torch

import causal_sliding_window_rope_b200 as cs
import oracle
from _helpers import TORCH_DT, f64, make_inputs, max_abs, rel_frob

pytestmark = pytest.mark.gpu


def run_case(B, T, H, Hk, D, W, X, C, dtype, seed):
    spec = cs.LayerSpec(B, T, H, Hk, D, W, has_ve=True, dtype=dtype)
    inp = make_inputs(B, T, H, Hk, D, True, dtype, config=seed)
    g = torch.Generator().manual_seed(seed)
    dt = TORCH_DT[dtype]
    x = torch.randn(B, T, X, generator=g).to(dt)
    w = (torch.randn(Hk, C, generator=g) / C ** 0.5).to(dt)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    xd, wd = x.cuda(), w.cuda()
    buf = cs.LayerBuffers(spec)
    gate = torch.empty(B, T, Hk, dtype=dt, device="cuda")
    cs.attn_prologue_gated(spec, dev["q"], dev["k"], dev["v"], dev["ve"], xd, C, wd, gate,
                           buf.q_out, buf.k_out, buf.v_out, buf.rstd_q, buf.rstd_k)
    cs.attn_fwd(spec, buf.q_out, buf.k_out, buf.v_out, buf.O, buf.lse)
    cs.attn_bwd(spec, dev["q"], dev["k"], dev["ve"], gate, buf.q_out, buf.k_out, buf.v_out,
                buf.rstd_q, buf.rstd_k, buf.O, buf.lse, dev["dO"], buf.dQ, buf.dK, buf.dV, buf.dve,
                buf.dgate, buf.workspace)
    dx = torch.empty(B, T, C, dtype=dt, device="cuda")
    dw = torch.empty(Hk, C, dtype=torch.float32, device="cuda")
    cs.attn_gate_bwd(spec, xd, C, wd, buf.dgate, dx, dw)
    cs.cswattn_sync_status()
    torch.cuda.synchronize()
    got = dict(gate=gate, O=buf.O, dq=buf.dQ, dk=buf.dK, dv=buf.dV, dve=buf.dve, dgate=buf.dgate,
               dx=dx, dw=dw)
    got = {k: f64(v) for k, v in got.items()}

    logits = oracle.gate_logits(f64(x), f64(w), C)
    L = oracle.Layer(B, T, H, Hk, D, W, True)
    ref = oracle.layer(L, *(f64(inp[k]) for k in ("q", "k", "v", "ve")), logits, f64(inp["dO"]))
    rdx, rdw = oracle.gate_bwd(f64(x), f64(w), C, ref["dgate"])
    ref = dict(gate=logits, O=ref["O"], dq=ref["dq"], dk=ref["dk"], dv=ref["dv"], dve=ref["dve"],
               dgate=ref["dgate"], dx=rdx, dw=rdw)
    return got, ref


@pytest.mark.parametrize("B,T,H,Hk,W,X,C", [(2, 300, 6, 2, 130, 96, 32), (1, 257, 4, 4, 257, 32, 32),
                                            (1, 200, 4, 1, 64, 50, 7)])
def test_gated_prologue_and_gate_backward_bf16(B, T, H, Hk, W, X, C):
    got, ref = run_case(B, T, H, Hk, 128, W, X, C, "bf16", seed=60 + C)
    errs = {k: rel_frob(got[k], ref[k]) for k in ref}
    bad = {k: v for k, v in errs.items() if not np.isfinite(v) or v > 2e-2}
    assert not bad, errs


def test_gated_prologue_and_gate_backward_f32():
    got, ref = run_case(2, 40, 4, 2, 16, 9, 24, 10, "f32", seed=66)
    for k in ref:
        assert max_abs(got[k], ref[k]) <= 1e-4, (k, max_abs(got[k], ref[k]))


def test_gate_backward_is_deterministic_and_matches_at_d24_shape():
    """dw_gate is summed in a fixed order (token lanes, then the cluster's
    blocks in rank order): two calls give the same bits. At the d24 layer
    shape (B*T = 8192 tokens, 4 KV heads, 32 and 40 gate channels: a
    partial channel group), dx and dw against the oracle."""
    B, T, Hk = 4, 2048, 4
    g = torch.Generator().manual_seed(71)
    for C in (32, 40):
        spec = cs.LayerSpec(B, T, 12, Hk, 128, 1024, has_ve=True, dtype="bf16")
        x = torch.randn(B, T, 1536, generator=g).to(torch.bfloat16)
        w = (torch.randn(Hk, C, generator=g) / C ** 0.5).to(torch.bfloat16)
        dgate = (0.1 * torch.randn(B, T, Hk, generator=g)).to(torch.bfloat16)
        xd, wd, dgd = x.cuda(), w.cuda(), dgate.cuda()
        runs = []
        for _ in range(2):
            dx = torch.empty(B, T, C, dtype=torch.bfloat16, device="cuda")
            dw = torch.empty(Hk, C, dtype=torch.float32, device="cuda")
            cs.attn_gate_bwd(spec, xd, C, wd, dgd, dx, dw)
            runs.append((dx, dw))
        cs.cswattn_sync_status()
        assert torch.equal(runs[0][1], runs[1][1]) and torch.equal(runs[0][0], runs[1][0])
        rdx, rdw = oracle.gate_bwd(f64(x), f64(w), C, f64(dgate))
        assert rel_frob(f64(runs[0][0]), rdx) <= 2e-2
        assert rel_frob(f64(runs[0][1]), rdw) <= 2e-2
