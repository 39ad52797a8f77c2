"""attn_decode (one generation step with a KV cache) against the oracle's
decode step, through the C ABI.

Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "6. 추론 엔진
(nanochat/engine.py)": generation over a pre-filled KV cache. The caches
given to both sides hold the oracle prologue's k~ and v_eff rows of each
sequence's first len[b] tokens, rounded to bf16; rows from len[b] on are NaN
on the GPU side, so a kernel that read a row outside the window would show
it. Tolerance: relative Frobenius 2e-2 per output (bf16).
"""
import numpy as np
import pytest
import torch

import causal_sliding_window_rope_b200 as cs
import oracle
from _helpers import f64, make_inputs, rel_frob

pytestmark = pytest.mark.gpu

TOL = 2e-2


def run_case(B, T, H, Hk, D, W, has_ve, lens, config):
    spec = cs.LayerSpec(B, T, H, Hk, D, W, has_ve=has_ve, dtype="bf16")
    inp = make_inputs(B, T, H, Hk, D, has_ve, "bf16", config=config, layer=len(lens))
    L = oracle.Layer(B, T, H, Hk, D, W, has_ve)
    _, kt, veff, _, _ = oracle.prologue(L, f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                        f64(inp["ve"]), f64(inp["gate"]))
    kc = torch.full((B, T, Hk, D), float("nan"), dtype=torch.bfloat16)
    vc = torch.full((B, T, Hk, D), float("nan"), dtype=torch.bfloat16)
    kt16 = torch.tensor(kt).to(torch.bfloat16)
    vt16 = torch.tensor(veff).to(torch.bfloat16)
    for b, p in enumerate(lens):
        kc[b, :p] = kt16[b, :p]
        vc[b, :p] = vt16[b, :p]
    tok = {n: (torch.stack([inp[n][b, lens[b]] for b in range(B)]) if inp[n] is not None else None)
           for n in ("q", "k", "v", "ve", "gate")}
    # Oracle: same bf16 cache values (NaN rows are never read by the definition).
    O_ref, lse_ref, kc_ref, vc_ref = oracle.decode(
        L, f64(tok["q"]), f64(tok["k"]), f64(tok["v"]), f64(tok["ve"]), f64(tok["gate"]), lens,
        f64(kc), f64(vc))
    # GPU
    dev = {n: (t.cuda().contiguous() if t is not None else None) for n, t in tok.items()}
    kc_d, vc_d = kc.cuda(), vc.cuda()
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    O = torch.full((B, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(cs.attn_decode_workspace_bytes(spec), dtype=torch.uint8, device="cuda")
    cs.attn_decode(spec, dev["q"], dev["k"], dev["v"], dev["ve"], dev["gate"], lens_d, kc_d, vc_d,
                   O, lse, ws)
    cs.cswattn_sync_status()
    torch.cuda.synchronize()
    return dict(spec=spec, lens=lens, O=f64(O), lse=f64(lse), kc=kc_d.cpu(), vc=vc_d.cpu(),
                kc_in=kc, vc_in=vc, O_ref=O_ref, lse_ref=lse_ref, kc_ref=kc_ref, vc_ref=vc_ref)


def check(r):
    assert np.isfinite(r["O"]).all() and np.isfinite(r["lse"]).all()
    assert rel_frob(r["O"], r["O_ref"]) <= TOL
    assert rel_frob(r["lse"], r["lse_ref"]) <= TOL
    for b, p in enumerate(r["lens"]):
        # the new token's rows
        assert rel_frob(f64(r["kc"][b, p]), r["kc_ref"][b, p]) <= TOL
        assert rel_frob(f64(r["vc"][b, p]), r["vc_ref"][b, p]) <= TOL
        # every other row unchanged, bit for bit (NaN rows stay NaN)
        keep = [t for t in range(r["spec"].T) if t != p]
        for got, was in ((r["kc"], r["kc_in"]), (r["vc"], r["vc_in"])):
            assert torch.equal(got[b, keep].view(torch.int16), was[b, keep].view(torch.int16))


CASES = [
    # B, T, H, Hk, D, W, has_ve, lens (tokens already cached per sequence)
    (3, 300, 4, 2, 128, 100, True, [0, 150, 299]),
    (2, 200, 6, 2, 128, 200, False, [127, 128]),
    (2, 129, 3, 3, 64, 64, True, [5, 128]),
    (1, 513, 16, 1, 128, 1, True, [400]),
    (2, 1000, 8, 2, 128, 384, True, [383, 999]),
    (2, 700, 8, 1, 64, 300, True, [299, 650]),     # group of 8
    (1, 400, 10, 2, 128, 400, False, [399]),       # group of 5: three unused head slots
]


@pytest.mark.parametrize("B,T,H,Hk,D,W,has_ve,lens", CASES)
def test_decode_matches_oracle(B, T, H, Hk, D, W, has_ve, lens):
    check(run_case(B, T, H, Hk, D, W, has_ve, lens, config=93))


@pytest.mark.parametrize("W", [1024, 2048])
def test_decode_d24_shapes(W):
    """The d24 layer's shapes (B=4, 12 query heads on 4 KV heads, head_dim
    128) with a 2048-row cache, at several fill levels."""
    check(run_case(4, 2048, 12, 4, 128, W, True, [2047, 1500, 1024, 77], config=94))


def test_decode_length_out_of_range_is_reported_and_harmless():
    spec = cs.LayerSpec(2, 64, 4, 2, 128, 32, has_ve=False, dtype="bf16")
    B, T, H, Hk, D = 2, 64, 4, 2, 128
    q = torch.randn(B, H, D, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(B, Hk, D, dtype=torch.bfloat16, device="cuda")
    v = torch.randn(B, Hk, D, dtype=torch.bfloat16, device="cuda")
    kc = torch.randn(B, T, Hk, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.randn(B, T, Hk, D, dtype=torch.bfloat16, device="cuda")
    kc0, vc0 = kc.clone(), vc.clone()
    lens = torch.tensor([T, 3], dtype=torch.int32, device="cuda")  # sequence 0 is full
    O = torch.zeros(B, H, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(cs.attn_decode_workspace_bytes(spec), dtype=torch.uint8, device="cuda")
    cs.attn_decode(spec, q, k, v, None, None, lens, kc, vc, O, lse, ws)
    with pytest.raises(cs.CswattnError) as err:
        cs.cswattn_sync_status()
    assert err.value.status == cs.ERR_INVALID_ARG
    assert torch.equal(kc[0], kc0[0]) and torch.equal(vc[0], vc0[0])
    assert torch.isfinite(O[1].float()).all()
    cs.cswattn_sync_status()  # cleared
