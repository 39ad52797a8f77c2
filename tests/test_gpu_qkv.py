"""GPU parity of the QKV projection fused with the prologue
(attn_qkv_prologue) and of its backward (attn_qkv_bwd), against the float64
oracle (projection, then the layer, then the projection's backward) on the
same bf16 inputs.

Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "1. GPT 모델":
the block input projected to the query, key and value heads (bias-free
Linear layers) before RoPE, QK normalisation and the value residual.
Tolerance: relative Frobenius error <= 2e-2 per tensor.
"""
import numpy as np
import pytest
import torch

import causal_sliding_window_rope_b200 as cs
import oracle
from _helpers import f64, rel_frob

pytestmark = pytest.mark.gpu
TOL = 2e-2


def draw(B, T, C, H, Hk, D, has_ve, seed):
    g = torch.Generator().manual_seed(seed)
    bf = torch.bfloat16
    x = torch.randn(B, T, C, generator=g).to(bf)
    w = (torch.randn((H + 2 * Hk) * D, C, generator=g) / C ** 0.5).to(bf)
    ve = torch.randn(B, T, Hk, D, generator=g).to(bf) if has_ve else None
    gate = torch.randn(B, T, Hk, generator=g).to(bf) if has_ve else None
    dO = torch.randn(B, T, H, D, generator=g).to(bf)
    return x, w, ve, gate, dO


def gpu_prologue(spec, x, C, w, ve, gate):
    B, T, H, Hk, D = spec.B, spec.T, spec.n_head, spec.n_kv_head, spec.head_dim
    buf = cs.LayerBuffers(spec)
    q = torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, T, Hk, D, dtype=torch.bfloat16, device="cuda")
    cs.attn_qkv_prologue(spec, x.cuda(), C, w.cuda(), ve.cuda() if ve is not None else None,
                         gate.cuda() if gate is not None else None, q, k, buf.q_out, buf.k_out,
                         buf.v_out, buf.rstd_q, buf.rstd_k)
    return q, k, buf


@pytest.mark.parametrize("B,T,C,H,Hk,D,W,has_ve", [
    (2, 300, 256, 6, 2, 128, 130, True),
    (1, 257, 96, 4, 4, 64, 257, True),
    (1, 200, 64, 2, 1, 128, 50, False),
    (1, 130, 128, 3, 1, 128, 64, True),   # 5 stacked heads: a (q, k) pair and a lone value head
    (1, 150, 64, 3, 1, 64, 64, True),     # 3 x 64 query rows: dW as three products, not one
])
def test_qkv_prologue_and_backward_match_oracle(B, T, C, H, Hk, D, W, has_ve):
    spec = cs.LayerSpec(B, T, H, Hk, D, W, has_ve=has_ve, dtype="bf16")
    x, w, ve, gate, dO = draw(B, T, C, H, Hk, D, has_ve, seed=40 + D + T)
    q, k, buf = gpu_prologue(spec, x, C, w, ve, gate)
    cs.attn_fwd(spec, buf.q_out, buf.k_out, buf.v_out, buf.O, buf.lse)
    dev_ve = ve.cuda() if ve is not None else None
    dev_gate = gate.cuda() if gate is not None else None
    cs.attn_bwd(spec, q, k, dev_ve, dev_gate, buf.q_out, buf.k_out, buf.v_out, buf.rstd_q, buf.rstd_k,
                buf.O, buf.lse, dO.cuda(), buf.dQ, buf.dK, buf.dV, buf.dve, buf.dgate, buf.workspace)
    dx = torch.empty(B, T, C, dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((H + 2 * Hk) * D, C, dtype=torch.float32, device="cuda")
    cs.attn_qkv_bwd(spec, x.cuda(), C, w.cuda(), buf.dQ, buf.dK, buf.dV, dx, dw)
    cs.cswattn_sync_status()

    L = oracle.Layer(B, T, H, Hk, D, W, has_ve)
    rq, rk, rv = oracle.qkv_projection(f64(x), f64(w), H, Hk, D)
    qt, kt, veff, rsq, rsk = oracle.prologue(L, rq, rk, rv, f64(ve), f64(gate))
    ref = oracle.layer(L, rq, rk, rv, f64(ve), f64(gate), f64(dO))
    rdx, rdw = oracle.qkv_projection_bwd(f64(x), f64(w), ref["dq"], ref["dk"], ref["dv"])
    pairs = {"q": (q, rq), "k": (k, rk), "q_out": (buf.q_out, qt), "k_out": (buf.k_out, kt),
             "v_out": (buf.v_out, veff), "rstd_q": (buf.rstd_q, rsq), "rstd_k": (buf.rstd_k, rsk),
             "O": (buf.O, ref["O"]), "dQ": (buf.dQ, ref["dq"]), "dK": (buf.dK, ref["dk"]),
             "dV": (buf.dV, ref["dv"]), "dx": (dx, rdx), "dw": (dw, rdw)}
    errs = {n: rel_frob(f64(a), r) for n, (a, r) in pairs.items()}
    bad = {n: e for n, e in errs.items() if not np.isfinite(e) or e > TOL}
    assert not bad, errs


def test_qkv_prologue_full_size_d24():
    """The d24 layer's projection (C = 1536, 12 query and 4 KV heads,
    B*T = 8192 tokens): raw projections and the prologue outputs."""
    B, T, C, H, Hk, D = 4, 2048, 1536, 12, 4, 128
    spec = cs.LayerSpec(B, T, H, Hk, D, 1024, has_ve=True, dtype="bf16")
    x, w, ve, gate, _ = draw(B, T, C, H, Hk, D, True, seed=48)
    q, k, buf = gpu_prologue(spec, x, C, w, ve, gate)
    cs.cswattn_sync_status()
    L = oracle.Layer(B, T, H, Hk, D, 1024, True)
    rq, rk, rv = oracle.qkv_projection(f64(x), f64(w), H, Hk, D)
    qt, kt, veff, rsq, rsk = oracle.prologue(L, rq, rk, rv, f64(ve), f64(gate))
    for name, a, r in (("q", q, rq), ("k", k, rk), ("q_out", buf.q_out, qt), ("k_out", buf.k_out, kt),
                       ("v_out", buf.v_out, veff), ("rstd_q", buf.rstd_q, rsq)):
        assert rel_frob(f64(a), r) <= TOL, name


def e4m3_decode(codes):
    """float64 values of E4M3 codes (torch's float8_e4m3fn conversion)."""
    return codes.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


@pytest.mark.parametrize("B,T,C,H,Hk,D,W,has_ve", [
    (2, 300, 256, 6, 2, 128, 130, True),
    (1, 257, 400, 4, 4, 64, 257, True),   # C = 3 x 128 + 16: a ragged last chunk
    (1, 200, 64, 2, 1, 128, 50, False),
    (1, 130, 128, 3, 1, 64, 64, True),    # 5 stacked heads: a (q, k) pair and a lone value head
])
def test_qkv_prologue_fp8_matches_oracle(B, T, C, H, Hk, D, W, has_ve):
    """Page section "3. 정밀도 관리" (Float8Linear, tensor-wise scaling): the
    two scales bit-exact, every E4M3 code equal to the oracle's rounding of
    t / s (both divide in float32), and the projection and prologue outputs
    within the tolerance of the bf16 path."""
    spec = cs.LayerSpec(B, T, H, Hk, D, W, has_ve=has_ve, dtype="bf16")
    x, w, ve, gate, dO = draw(B, T, C, H, Hk, D, has_ve, seed=70 + D + T)
    x = x * 3.0  # amax of x well away from 1
    buf = cs.LayerBuffers(spec)
    q = torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, T, Hk, D, dtype=torch.bfloat16, device="cuda")
    scales = torch.zeros(2, dtype=torch.float32, device="cuda")
    nbytes = cs.attn_qkv_fp8_workspace_bytes(spec, C)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    cs.attn_qkv_prologue_fp8(spec, x.cuda(), C, w.cuda(), ve.cuda() if ve is not None else None,
                             gate.cuda() if gate is not None else None, q, k, buf.q_out, buf.k_out,
                             buf.v_out, buf.rstd_q, buf.rstd_k, scales, ws)
    cs.cswattn_sync_status()

    sx, sw = oracle.fp8_tensor_scale(f64(x)), oracle.fp8_tensor_scale(f64(w))
    got = scales.cpu().numpy()
    assert got[0] == sx and got[1] == sw, (got, sx, sw)
    n_x, n_w = B * T * C, (H + 2 * Hk) * D * C
    off_w = 256 + (n_x + 255) // 256 * 256
    xq = e4m3_decode(ws[256:256 + n_x]).reshape(B, T, C)
    wq = e4m3_decode(ws[off_w:off_w + n_w]).reshape(-1, C)
    assert np.array_equal(xq, oracle.quantize_e4m3(f64(x), sx))
    assert np.array_equal(wq, oracle.quantize_e4m3(f64(w), sw))

    L = oracle.Layer(B, T, H, Hk, D, W, has_ve)
    rq, rk, rv, _ = oracle.qkv_projection_fp8(f64(x), f64(w), H, Hk, D)
    qt, kt, veff, rsq, rsk = oracle.prologue(L, rq, rk, rv, f64(ve), f64(gate))
    pairs = {"q": (q, rq), "k": (k, rk), "q_out": (buf.q_out, qt), "k_out": (buf.k_out, kt),
             "v_out": (buf.v_out, veff), "rstd_q": (buf.rstd_q, rsq), "rstd_k": (buf.rstd_k, rsk)}
    errs = {n: rel_frob(f64(a), r) for n, (a, r) in pairs.items()}
    bad = {n: e for n, e in errs.items() if not np.isfinite(e) or e > TOL}
    assert not bad, errs


def test_qkv_prologue_fp8_zero_input():
    """An all-zero x takes the scale 1 (the amax-is-zero case) and gives a
    zero projection; the value residual still adds 3 sigmoid(gate) ve."""
    B, T, C, H, Hk, D = 1, 130, 128, 2, 1, 64
    spec = cs.LayerSpec(B, T, H, Hk, D, 64, has_ve=True, dtype="bf16")
    _, w, ve, gate, _ = draw(B, T, C, H, Hk, D, True, seed=91)
    x = torch.zeros(B, T, C, dtype=torch.bfloat16)
    buf = cs.LayerBuffers(spec)
    q = torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, T, Hk, D, dtype=torch.bfloat16, device="cuda")
    scales = torch.zeros(2, dtype=torch.float32, device="cuda")
    ws = torch.empty(cs.attn_qkv_fp8_workspace_bytes(spec, C), dtype=torch.uint8, device="cuda")
    cs.attn_qkv_prologue_fp8(spec, x.cuda(), C, w.cuda(), ve.cuda(), gate.cuda(), q, k, buf.q_out, buf.k_out,
                             buf.v_out, buf.rstd_q, buf.rstd_k, scales, ws)
    cs.cswattn_sync_status()
    assert scales[0].item() == 1.0
    assert torch.count_nonzero(q).item() == 0 and torch.count_nonzero(k).item() == 0
    coef = 3.0 / (1.0 + np.exp(-f64(gate)))
    assert rel_frob(f64(buf.v_out), coef[..., None] * f64(ve)) <= TOL


def test_qkv_prologue_fp8_full_size_d24():
    """The d24 layer's projection with E4M3 operands (C = 1536, 12 query and
    4 KV heads, B*T = 8192 tokens): both scales bit-exact, the raw
    projections and the prologue outputs against the oracle."""
    B, T, C, H, Hk, D = 4, 2048, 1536, 12, 4, 128
    spec = cs.LayerSpec(B, T, H, Hk, D, 1024, has_ve=True, dtype="bf16")
    x, w, ve, gate, _ = draw(B, T, C, H, Hk, D, True, seed=49)
    buf = cs.LayerBuffers(spec)
    q = torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(B, T, Hk, D, dtype=torch.bfloat16, device="cuda")
    scales = torch.zeros(2, dtype=torch.float32, device="cuda")
    ws = torch.empty(cs.attn_qkv_fp8_workspace_bytes(spec, C), dtype=torch.uint8, device="cuda")
    cs.attn_qkv_prologue_fp8(spec, x.cuda(), C, w.cuda(), ve.cuda(), gate.cuda(), q, k, buf.q_out, buf.k_out,
                             buf.v_out, buf.rstd_q, buf.rstd_k, scales, ws)
    cs.cswattn_sync_status()
    rq, rk, rv, (sx, sw) = oracle.qkv_projection_fp8(f64(x), f64(w), H, Hk, D)
    got = scales.cpu().numpy()
    assert got[0] == np.float32(sx) and got[1] == np.float32(sw)
    L = oracle.Layer(B, T, H, Hk, D, 1024, True)
    qt, kt, veff, rsq, rsk = oracle.prologue(L, rq, rk, rv, f64(ve), f64(gate))
    for name, a, r in (("q", q, rq), ("k", k, rk), ("q_out", buf.q_out, qt), ("k_out", buf.k_out, kt),
                       ("v_out", buf.v_out, veff), ("rstd_k", buf.rstd_k, rsk)):
        assert rel_frob(f64(a), r) <= TOL, name
