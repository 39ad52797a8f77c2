"""Pins of the float64 oracle against things other than itself.

Each test ties one step of the oracle to a library routine, a closed form, an
invariant of the definition or finite differences, so that a dropped term, a
wrong sign or index, or a transposed operand fails at least one of them.
Definition followed: page "5만원으로 나만의 ChatGPT 훈련하는 방법"
(apidog.com), section "1. GPT 모델 (nanochat/gpt.py)" (RoPE, QK normalisation,
GQA, sliding window, value embedding code) and section "5. 플래시 어텐션 통합"
(causal attention call with a window size).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def inputs(L, seed=0):
    q = rnd((L.B, L.T, L.H, L.D), seed)
    k = rnd((L.B, L.T, L.Hk, L.D), seed + 1)
    v = rnd((L.B, L.T, L.Hk, L.D), seed + 2)
    ve = rnd((L.B, L.T, L.Hk, L.D), seed + 3)
    gate = rnd((L.B, L.T, L.Hk), seed + 4)
    dO = rnd((L.B, L.T, L.H, L.D), seed + 5)
    return q, k, v, ve, gate, dO


def band_mask(T, W):
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    return (j <= i) & (j > i - W)


# ---------------------------------------------------------------- attention core

@pytest.mark.parametrize("T,W,H,Hk,D", [(9, 9, 2, 2, 4), (9, 3, 2, 1, 4), (13, 1, 4, 2, 6),
                                        (16, 5, 6, 2, 8), (7, 100, 3, 3, 2)])
def test_core_matches_torch_sdpa_and_autograd(T, W, H, Hk, D):
    """With the norm and rotation switched off, the core is plain banded causal
    softmax attention: torch's SDPA (float64, explicit band mask, repeat
    -interleave GQA) and its autograd must agree with the oracle."""
    L = oracle.Layer(2, T, H, Hk, D, W, has_ve=False, flags=oracle.NO_NORM | oracle.NO_ROPE)
    q, k, v, _, _, dO = inputs(L, seed=T * 7 + W)
    qt, kt, veff, rq, rk = oracle.prologue(L, q, k, v)
    assert np.array_equal(qt, q) and np.array_equal(kt, k) and np.array_equal(veff, v)
    O, lse = oracle.attn_fwd(L, qt, kt, veff)
    dqt, dkt, dveff = oracle.attn_bwd(L, qt, kt, veff, O, lse, dO)

    tq = torch.tensor(q).transpose(1, 2).requires_grad_()
    tk = torch.tensor(k).transpose(1, 2).requires_grad_()
    tv = torch.tensor(v).transpose(1, 2).requires_grad_()
    ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=band_mask(T, W), enable_gqa=True)
    ref.backward(torch.tensor(dO).transpose(1, 2))
    np.testing.assert_allclose(O, ref.detach().transpose(1, 2).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dqt, tq.grad.transpose(1, 2).numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dkt, tk.grad.transpose(1, 2).numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dveff, tv.grad.transpose(1, 2).numpy(), rtol=0, atol=1e-11)

    # lse against torch.logsumexp of the masked score matrix (library routine)
    qh = torch.tensor(q).transpose(1, 2)
    kh = torch.tensor(k).transpose(1, 2).repeat_interleave(H // Hk, dim=1)
    s = qh @ kh.transpose(-1, -2) / math.sqrt(D)
    s = s.masked_fill(~band_mask(T, W), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


def test_softmax_rows_sum_to_one_and_respect_band():
    L = oracle.Layer(1, 12, 2, 1, 4, 5, has_ve=False)
    q, k, v, *_ = inputs(L, 3)
    qt, kt, *_ = oracle.prologue(L, q, k, v)
    for h in range(2):
        for i in range(12):
            p, lse = oracle.probs_row(L, qt, kt, 0, h, i)
            assert abs(p.sum() - 1.0) < 1e-12
            visible = [(j <= i and j > i - 5) for j in range(12)]
            assert all((p[j] > 0) == visible[j] for j in range(12))


def test_output_in_convex_hull_of_visible_values():
    L = oracle.Layer(1, 20, 2, 2, 4, 6, has_ve=True)
    q, k, v, ve, gate, _ = inputs(L, 4)
    qt, kt, veff, *_ = oracle.prologue(L, q, k, v, ve, gate)
    O, _ = oracle.attn_fwd(L, qt, kt, veff)
    for h in range(2):
        for i in range(20):
            win = veff[0, max(0, i - 5): i + 1, h]
            assert np.all(O[0, i, h] <= win.max(0) + 1e-12)
            assert np.all(O[0, i, h] >= win.min(0) - 1e-12)


def test_window_at_least_T_is_full_causal():
    args = dict(B=2, T=11, H=4, Hk=2, D=6, has_ve=True)
    Lw = oracle.Layer(W=11, **args)
    Lbig = oracle.Layer(W=10**6, **args)
    data = inputs(Lw, 5)
    a = oracle.layer(Lw, *data)
    b = oracle.layer(Lbig, *data)
    for key in ("O", "lse", "dq", "dk", "dv", "dve", "dgate"):
        assert np.array_equal(a[key], b[key]), key


def test_window_one_gives_value_and_zero_qk_grads():
    """W = 1: every query sees only itself, so O = v_eff, lse = s_ii and
    ds = p (dp - Delta) = 0 exactly (p = 1, Delta = dp)."""
    L = oracle.Layer(2, 9, 4, 2, 8, 1, has_ve=True)
    q, k, v, ve, gate, dO = inputs(L, 6)
    r = oracle.layer(L, q, k, v, ve, gate, dO)
    veff_rep = np.repeat(r["veff"], 2, axis=2)
    np.testing.assert_allclose(r["O"], veff_rep, rtol=0, atol=1e-14)
    kt_rep = np.repeat(r["kt"], 2, axis=2)
    s = (r["qt"] * kt_rep).sum(-1) / math.sqrt(8)
    np.testing.assert_allclose(r["lse"], s.transpose(0, 2, 1), rtol=0, atol=1e-13)
    assert np.abs(r["dq"]).max() < 1e-13 and np.abs(r["dk"]).max() < 1e-13
    np.testing.assert_allclose(r["dveff"], dO.reshape(2, 9, 2, 2, 8).sum(3), atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv():
    Lg = oracle.Layer(2, 10, 6, 2, 4, 4, has_ve=False)
    Lm = oracle.Layer(2, 10, 6, 6, 4, 4, has_ve=False)
    q, k, v, _, _, dO = inputs(Lg, 7)
    g = oracle.layer(Lg, q, k, v, None, None, dO)
    m = oracle.layer(Lm, q, np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2), None, None, dO)
    np.testing.assert_allclose(g["O"], m["O"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(g["dq"], m["dq"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(g["dk"], m["dk"].reshape(2, 10, 2, 3, 4).sum(3), atol=1e-12)
    np.testing.assert_allclose(g["dv"], m["dv"].reshape(2, 10, 2, 3, 4).sum(3), atol=1e-12)


# ---------------------------------------------------------------- prologue

def test_rope_matches_complex_rotation_and_preserves_norm():
    """RoPE on half-split pairs is multiplication of x_i + 1j*x_{i+D/2} by
    exp(1j * t * base^(-2i/D)); it keeps the norm and is the identity at t=0."""
    D, T = 8, 6
    L = oracle.Layer(1, T, 1, 1, D, T, has_ve=False, flags=oracle.NO_NORM, rope_base=500.0)
    q, k, v, *_ = inputs(L, 8)
    qt, *_ = oracle.prologue(L, q, k, v)
    z = q[0, :, 0, : D // 2] + 1j * q[0, :, 0, D // 2:]
    w = 500.0 ** (-2.0 * np.arange(D // 2) / D)
    zr = z * np.exp(1j * np.arange(T)[:, None] * w[None, :])
    np.testing.assert_allclose(qt[0, :, 0, : D // 2], zr.real, atol=1e-13)
    np.testing.assert_allclose(qt[0, :, 0, D // 2:], zr.imag, atol=1e-13)
    np.testing.assert_allclose(np.linalg.norm(qt, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-13)
    np.testing.assert_array_equal(qt[0, 0], q[0, 0])


def test_rmsnorm_matches_torch_and_closed_form():
    L = oracle.Layer(2, 5, 3, 1, 16, 5, has_ve=False, flags=oracle.NO_ROPE, eps=1e-3)
    q, k, v, *_ = inputs(L, 9)
    qt, kt, _, rq, rk = oracle.prologue(L, q, k, v)
    ref = F.rms_norm(torch.tensor(q), (16,), eps=1e-3).numpy()
    np.testing.assert_allclose(qt, ref, rtol=1e-13, atol=1e-14)
    ms = (q ** 2).mean(-1)
    np.testing.assert_allclose((qt ** 2).mean(-1), ms / (ms + 1e-3), rtol=1e-12)
    np.testing.assert_allclose(rq, 1.0 / np.sqrt(ms + 1e-3), rtol=1e-13)


def test_norm_and_rope_commute():
    base = dict(B=1, T=7, H=2, Hk=1, D=8, W=7, has_ve=False)
    q, k, v, *_ = inputs(oracle.Layer(**base), 10)
    both = oracle.prologue(oracle.Layer(**base), q, k, v)[0]
    rope_only = oracle.prologue(oracle.Layer(**base, flags=oracle.NO_NORM), q, k, v)[0]
    normed = F.rms_norm(torch.tensor(rope_only), (8,), eps=1e-6).numpy()
    np.testing.assert_allclose(both, normed, rtol=0, atol=1e-14)


def test_scores_depend_only_on_relative_position():
    base = dict(B=1, T=10, H=2, Hk=2, D=8, W=4, has_ve=True)
    data = inputs(oracle.Layer(**base), 11)
    a = oracle.layer(oracle.Layer(**base), *data)
    b = oracle.layer(oracle.Layer(**base, pos_offset=37), *data)
    for key in ("O", "lse", "dq", "dk", "dv", "dve", "dgate"):
        np.testing.assert_allclose(a[key], b[key], rtol=0, atol=1e-11, err_msg=key)
    assert not np.allclose(a["qt"], b["qt"])  # the rotation itself did change


def test_value_residual_gate_limits():
    """v_eff = v + 3 sigmoid(gate) ve (value-embedding code on the page):
    gate -> -inf gives v, gate = 0 gives v + 1.5 ve, gate -> +inf gives v + 3 ve."""
    L = oracle.Layer(1, 3, 2, 2, 4, 3, has_ve=True)
    q, k, v, ve, *_ = inputs(L, 12)
    for g, coef in ((-1e4, 0.0), (0.0, 1.5), (1e4, 3.0)):
        _, _, veff, *_ = oracle.prologue(L, q, k, v, ve, np.full((1, 3, 2), g))
        np.testing.assert_allclose(veff, v + coef * ve, rtol=0, atol=1e-15)


# ---------------------------------------------------------------- gradients

def _loss(L, q, k, v, ve, gate, dO):
    qt, kt, veff, *_ = oracle.prologue(L, q, k, v, ve, gate)
    O, _ = oracle.attn_fwd(L, qt, kt, veff)
    return float((O * dO).sum())


@pytest.mark.parametrize("W", [1, 3, 16])
def test_gradients_match_central_differences(W):
    """Every input of the layer against central differences of L = sum(O * dO)."""
    L = oracle.Layer(1, 16, 4, 2, 6, W, has_ve=True)
    q, k, v, ve, gate, dO = inputs(L, 13 + W)
    r = oracle.layer(L, q, k, v, ve, gate, dO)
    grads = dict(q=r["dq"], k=r["dk"], v=r["dv"], ve=r["dve"], gate=r["dgate"])
    data = dict(q=q, k=k, v=v, ve=ve, gate=gate)
    rng = np.random.default_rng(W)
    h = 1e-6
    for name, x in data.items():
        for _ in range(12):
            idx = tuple(rng.integers(0, s) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            fp = _loss(L, **{**data, name: xp}, dO=dO)
            fm = _loss(L, **{**data, name: xm}, dO=dO)
            fd = (fp - fm) / (2 * h)
            an = grads[name][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)


def test_layer_matches_torch_autograd_restatement():
    """The full layer written with torch library routines (rms_norm, a complex
    rotation, SDPA with a band mask and GQA), differentiated by autograd."""
    B, T, H, Hk, D, W = 2, 12, 6, 2, 8, 5
    L = oracle.Layer(B, T, H, Hk, D, W, has_ve=True, rope_base=10000.0, eps=1e-6)
    q, k, v, ve, gate, dO = inputs(L, 14)
    r = oracle.layer(L, q, k, v, ve, gate, dO)

    tq, tk, tv, tve, tg = (torch.tensor(a, requires_grad=True) for a in (q, k, v, ve, gate))

    def rope(x):
        z = torch.complex(x[..., : D // 2], x[..., D // 2:])
        w = 10000.0 ** (-2.0 * torch.arange(D // 2, dtype=torch.float64) / D)
        ang = torch.arange(T, dtype=torch.float64)[:, None] * w[None, :]
        z = z * torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
        return torch.cat([z.real, z.imag], dim=-1)

    qn = rope(F.rms_norm(tq, (D,), eps=1e-6))
    kn = rope(F.rms_norm(tk, (D,), eps=1e-6))
    vv = tv + 3 * torch.sigmoid(tg)[..., None] * tve
    o = F.scaled_dot_product_attention(qn.transpose(1, 2), kn.transpose(1, 2), vv.transpose(1, 2),
                                       attn_mask=band_mask(T, W), enable_gqa=True).transpose(1, 2)
    o.backward(torch.tensor(dO))
    np.testing.assert_allclose(r["O"], o.detach().numpy(), atol=1e-12)
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv), ("dve", tve), ("dgate", tg)):
        np.testing.assert_allclose(r[name], t.grad.numpy(), atol=1e-11, err_msg=name)


# ---------------------------------------------------------------- row entry points

def test_row_functions_match_full_layer():
    L = oracle.Layer(2, 40, 6, 2, 8, 9, has_ve=True)
    q, k, v, ve, gate, dO = inputs(L, 15)
    r = oracle.layer(L, q, k, v, ve, gate, dO)
    rows = [(0, 0, 0), (1, 5, 39), (0, 3, 17), (1, 2, 8)]
    O, lse = oracle.fwd_rows(L, r["qt"], r["kt"], r["veff"], rows)
    dq = oracle.dq_rows(L, r["qt"], r["kt"], r["veff"], dO, rows)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(O[n], r["O"][b, i, h], atol=1e-14)
        assert abs(lse[n] - r["lse"][b, h, i]) < 1e-14
        np.testing.assert_allclose(dq[n], r["dqt"][b, i, h], atol=1e-13)
    krows = [(0, 0, 0), (1, 1, 39), (0, 1, 20), (1, 0, 31)]
    dk, dv = oracle.dkv_rows(L, r["qt"], r["kt"], r["veff"], dO, krows)
    for n, (b, hk, j) in enumerate(krows):
        np.testing.assert_allclose(dk[n], r["dkt"][b, j, hk], atol=1e-13)
        np.testing.assert_allclose(dv[n], r["dveff"][b, j, hk], atol=1e-13)


# ---------------------------------------------------------------- golden values

def test_hand_worked_example():
    """A two-token case worked by hand (derivation in the fixture)."""
    with open(os.path.join(GOLDEN, "two_token_by_hand.json")) as f:
        g = json.load(f)
    L = oracle.Layer(1, 2, 1, 1, 2, 2, has_ve=False, flags=oracle.NO_NORM | oracle.NO_ROPE)
    q = np.array(g["q"]).reshape(1, 2, 1, 2)
    k = np.array(g["k"]).reshape(1, 2, 1, 2)
    v = np.array(g["v"]).reshape(1, 2, 1, 2)
    O, lse = oracle.attn_fwd(L, q, k, v)
    np.testing.assert_allclose(O.reshape(2, 2), np.array(g["O"]), atol=1e-15)
    np.testing.assert_allclose(lse.reshape(2), np.array(g["lse"]), atol=1e-15)


def test_oracle_regression_fixture():
    """Oracle outputs on a small seeded case, written by tests/golden/make_golden.py
    (which calls only the oracle). Guards against unintended oracle changes."""
    with open(os.path.join(GOLDEN, "oracle_small_case.json")) as f:
        g = json.load(f)
    c = g["case"]
    L = oracle.Layer(c["B"], c["T"], c["H"], c["Hk"], c["D"], c["W"], has_ve=True)
    data = inputs(L, c["seed"])
    r = oracle.layer(L, *data)
    for key, val in g["checksums"].items():
        assert abs(float(np.sum(r[key] * np.cos(np.arange(r[key].size)).reshape(r[key].shape))) - val) \
            <= 1e-9 * max(1.0, abs(val)), key


# ---------------------------------------------------------------- decode with a KV cache

def decode_case(L, lens, seed):
    """Raw projections for all T positions, the full-sequence oracle, and the
    decode inputs: caches holding the prologue rows of each sequence's first
    lens[b] tokens (later rows NaN, so reading them would show), and the raw
    projections of token lens[b]."""
    q, k, v, ve, gate, _ = inputs(L, seed)
    qt, kt, veff, _, _ = oracle.prologue(L, q, k, v, ve if L.has_ve else None, gate if L.has_ve else None)
    O, lse = oracle.attn_fwd(L, qt, kt, veff)
    kc = np.full_like(kt, np.nan)
    vc = np.full_like(veff, np.nan)
    B = L.B
    tok = {n: np.stack([a[b, lens[b]] for b in range(B)]) for n, a in
           (("q", q), ("k", k), ("v", v), ("ve", ve), ("gate", gate))}
    for b in range(B):
        kc[b, :lens[b]] = kt[b, :lens[b]]
        vc[b, :lens[b]] = veff[b, :lens[b]]
    return tok, kc, vc, (qt, kt, veff, O, lse)


@pytest.mark.parametrize("W,H,Hk,has_ve", [(5, 4, 2, True), (40, 3, 1, False), (1, 2, 2, True),
                                          (7, 6, 2, True)])
def test_decode_equals_last_row_of_full_forward(W, H, Hk, has_ve):
    """A decode step over a cache filled with the prologue rows of the first p
    tokens is row p of the full-sequence forward (causality: row p reads no
    later key), and the rows it writes are the prologue rows of token p."""
    L = oracle.Layer(3, 24, H, Hk, 8, W, has_ve=has_ve)
    lens = [0, 11, 23]
    tok, kc, vc, (qt, kt, veff, O, lse) = decode_case(L, lens, seed=W + 10 * H)
    Od, lsed, kc2, vc2 = oracle.decode(L, tok["q"], tok["k"], tok["v"], tok["ve"], tok["gate"],
                                       lens, kc, vc)
    for b, p in enumerate(lens):
        np.testing.assert_allclose(Od[b], O[b, p], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lsed[b], lse[b, :, p], rtol=0, atol=1e-12)
        np.testing.assert_allclose(kc2[b, p], kt[b, p], rtol=0, atol=1e-13)
        np.testing.assert_allclose(vc2[b, p], veff[b, p], rtol=0, atol=1e-13)
        assert np.isnan(kc2[b, p + 1:]).all() and np.isnan(vc2[b, p + 1:]).all()


def test_decode_window_one_returns_own_value():
    """W = 1: the new token sees only itself, so O = v_eff of the token and
    lse = c q~ . k~ of the token."""
    L = oracle.Layer(2, 10, 4, 2, 6, 1, has_ve=True)
    lens = [3, 9]
    tok, kc, vc, (qt, kt, veff, _, _) = decode_case(L, lens, seed=5)
    Od, lsed, _, _ = oracle.decode(L, tok["q"], tok["k"], tok["v"], tok["ve"], tok["gate"], lens, kc, vc)
    for b, p in enumerate(lens):
        for h in range(L.H):
            hk = h // (L.H // L.Hk)
            np.testing.assert_allclose(Od[b, h], veff[b, p, hk], rtol=0, atol=1e-12)
            assert abs(lsed[b, h] - L.scale * float(qt[b, p, h] @ kt[b, p, hk])) < 1e-12


# ---------------------------------------------------------------- value-embedding gate projection

def test_gate_projection_hand_worked():
    """Gate logits and their gradients on a hand-worked token (derivation in
    the fixture)."""
    with open(os.path.join(GOLDEN, "gate_by_hand.json")) as f:
        g = json.load(f)
    x = np.array(g["x"]).reshape(1, 1, 3)
    w = np.array(g["w"])
    logits = oracle.gate_logits(x, w, g["C"])
    np.testing.assert_allclose(logits.reshape(2), g["logits"], atol=1e-15)
    dx, dw = oracle.gate_bwd(x, w, g["C"], np.array(g["dgate"]).reshape(1, 1, 2))
    np.testing.assert_allclose(dx.reshape(2), g["dx"], atol=1e-15)
    np.testing.assert_allclose(dw, g["dw"], atol=1e-15)


def test_gate_projection_matches_torch_linear_and_autograd():
    """Against torch's float64 linear map and its autograd (library routines
    the oracle does not use)."""
    B, T, X, C, Hk = 2, 5, 9, 6, 3
    x = rnd((B, T, X), 70)
    w = rnd((Hk, C), 71)
    dg = rnd((B, T, Hk), 72)
    xt = torch.tensor(x, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    out = F.linear(xt[..., :C], wt)
    np.testing.assert_allclose(oracle.gate_logits(x, w, C), out.detach().numpy(), atol=1e-13)
    out.backward(torch.tensor(dg))
    dx, dw = oracle.gate_bwd(x, w, C, dg)
    np.testing.assert_allclose(dx, xt.grad.numpy()[..., :C], atol=1e-13)
    assert np.all(xt.grad.numpy()[..., C:] == 0)  # channels past C are not read
    np.testing.assert_allclose(dw, wt.grad.numpy(), atol=1e-13)


def test_gate_projection_gradients_match_central_differences():
    """The whole layer with its gate computed from x and w: dL/dx and dL/dw
    of L = sum(O * dO) from the layer's dgate through the projection's
    backward, against central differences of L itself."""
    L = oracle.Layer(1, 12, 4, 2, 6, 5, has_ve=True)
    q, k, v, ve, _, dO = inputs(L, 77)
    C, X = 4, 7
    x = rnd((1, L.T, X), 78)
    w = rnd((L.Hk, C), 79)

    def loss(x_, w_):
        return _loss(L, q, k, v, ve, oracle.gate_logits(x_, w_, C), dO)

    gate = oracle.gate_logits(x, w, C)
    dgate = oracle.layer(L, q, k, v, ve, gate, dO)["dgate"]
    dx, dw = oracle.gate_bwd(x, w, C, dgate)
    h = 1e-6
    rng = np.random.default_rng(5)
    for _ in range(10):
        t, c = int(rng.integers(0, L.T)), int(rng.integers(0, X))
        xp, xm = x.copy(), x.copy()
        xp[0, t, c] += h
        xm[0, t, c] -= h
        fd = (loss(xp, w) - loss(xm, w)) / (2 * h)
        an = dx[0, t, c] if c < C else 0.0
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), ("x", t, c, fd, an)
    for hh in range(L.Hk):
        for c in range(C):
            wp, wm = w.copy(), w.copy()
            wp[hh, c] += h
            wm[hh, c] -= h
            fd = (loss(x, wp) - loss(x, wm)) / (2 * h)
            assert abs(fd - dw[hh, c]) <= 1e-6 * max(1.0, abs(dw[hh, c])), ("w", hh, c, fd, dw[hh, c])


# ---------------------------------------------------------------- Muon Newton-Schulz

COEFFS = oracle.POLAR_EXPRESS_PRINTED


def test_newton_schulz_scalar_closed_form():
    """On a 1 x 1 matrix every step is the quintic x -> a x + b x^3 + c x^5."""
    x = 0.37
    want = x
    for a, b, c in COEFFS:
        want = a * want + b * want ** 3 + c * want ** 5
    got = oracle.newton_schulz(np.array([[x]]), COEFFS)
    assert abs(got[0, 0] - want) < 1e-15


def test_newton_schulz_acts_on_singular_values():
    """X = U S V^T maps to U p(S) V^T with p the composed quintic (numpy's
    SVD, a routine the oracle does not use)."""
    X = rnd((7, 5), 90)
    X /= np.linalg.norm(X)
    U, S, Vt = np.linalg.svd(X, full_matrices=False)
    for a, b, c in COEFFS:
        S = a * S + b * S ** 3 + c * S ** 5
    np.testing.assert_allclose(oracle.newton_schulz(X, COEFFS), (U * S) @ Vt, atol=1e-12)


def test_newton_schulz_orthogonal_equivariance_and_transpose():
    """NS(P X Q) = P NS(X) Q for orthogonal P, Q, and NS(X^T) = NS(X)^T."""
    X = rnd((6, 4), 91) / 4.0
    P, _ = np.linalg.qr(rnd((6, 6), 92))
    Q, _ = np.linalg.qr(rnd((4, 4), 93))
    Y = oracle.newton_schulz(X, COEFFS)
    np.testing.assert_allclose(oracle.newton_schulz(P @ X @ Q, COEFFS), P @ Y @ Q, atol=1e-12)
    np.testing.assert_allclose(oracle.newton_schulz(X.T, COEFFS), Y.T, atol=1e-12)


def test_newton_schulz_one_step_by_hand():
    """One step on a diagonal 2 x 2 matrix, worked by hand: A = diag(x^2),
    B = diag(b x^2 + c x^4), X' = diag(a x + b x^3 + c x^5)."""
    a, b, c = 2.0, -1.0, 0.5
    X = np.diag([1.0, 0.5])
    want = np.diag([2.0 - 1.0 + 0.5, 1.0 - 0.125 + 0.015625])
    np.testing.assert_allclose(oracle.newton_schulz(X, [(a, b, c)]), want, atol=1e-15)


def test_gemm_matches_explicit_sums():
    A, B, D = rnd((3, 4), 94), rnd((4, 2), 95), rnd((3, 2), 96)
    C = oracle.gemm(A, B, 0.5, D, -2.0)
    for i in range(3):
        for j in range(2):
            s = sum(A[i, k] * B[k, j] for k in range(4))
            assert abs(C[i, j] - (0.5 * s - 2.0 * D[i, j])) < 1e-13


# ---------------------------------------------------------------- QKV projection

def test_qkv_projection_matches_torch_linear_and_autograd():
    B, T, C, H, Hk, D = 2, 5, 12, 4, 2, 6
    x = rnd((B, T, C), 100)
    w = rnd(((H + 2 * Hk) * D, C), 101)
    xt = torch.tensor(x, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    y = F.linear(xt, wt)
    q, k, v = oracle.qkv_projection(x, w, H, Hk, D)
    np.testing.assert_allclose(q, y[..., :H * D].detach().numpy().reshape(B, T, H, D), atol=1e-13)
    np.testing.assert_allclose(k, y[..., H * D:(H + Hk) * D].detach().numpy().reshape(B, T, Hk, D), atol=1e-13)
    np.testing.assert_allclose(v, y[..., (H + Hk) * D:].detach().numpy().reshape(B, T, Hk, D), atol=1e-13)
    gq, gk, gv = rnd(q.shape, 102), rnd(k.shape, 103), rnd(v.shape, 104)
    y.backward(torch.cat([torch.tensor(gq).reshape(B, T, -1), torch.tensor(gk).reshape(B, T, -1),
                          torch.tensor(gv).reshape(B, T, -1)], dim=-1))
    dx, dw = oracle.qkv_projection_bwd(x, w, gq, gk, gv)
    np.testing.assert_allclose(dx, xt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dw, wt.grad.numpy(), atol=1e-12)


def test_qkv_projection_gradients_match_central_differences():
    """dL/dx and dL/dW of the whole layer fed by the projection, from the
    layer's dq, dk, dv through the projection's backward, against central
    differences of L = sum(O * dO)."""
    L = oracle.Layer(1, 10, 4, 2, 4, 4, has_ve=True)
    C = 6
    x = rnd((1, L.T, C), 105)
    w = rnd(((L.H + 2 * L.Hk) * L.D, C), 106) / 2
    _, _, _, ve, gate, dO = inputs(L, 107)

    def loss(x_, w_):
        q, k, v = oracle.qkv_projection(x_, w_, L.H, L.Hk, L.D)
        return _loss(L, q, k, v, ve, gate, dO)

    q, k, v = oracle.qkv_projection(x, w, L.H, L.Hk, L.D)
    r = oracle.layer(L, q, k, v, ve, gate, dO)
    dx, dw = oracle.qkv_projection_bwd(x, w, r["dq"], r["dk"], r["dv"])
    h = 1e-6
    rng = np.random.default_rng(9)
    for _ in range(8):
        t, c = int(rng.integers(0, L.T)), int(rng.integers(0, C))
        xp, xm = x.copy(), x.copy()
        xp[0, t, c] += h
        xm[0, t, c] -= h
        fd = (loss(xp, w) - loss(xm, w)) / (2 * h)
        assert abs(fd - dx[0, t, c]) <= 1e-6 * max(1.0, abs(dx[0, t, c])), ("x", t, c)
    for _ in range(12):
        o, c = int(rng.integers(0, w.shape[0])), int(rng.integers(0, C))
        wp, wm = w.copy(), w.copy()
        wp[o, c] += h
        wm[o, c] -= h
        fd = (loss(x, wp) - loss(x, wm)) / (2 * h)
        assert abs(fd - dw[o, c]) <= 1e-6 * max(1.0, abs(dw[o, c])), ("w", o, c)


# ---------------------------------------------------------------- FP8 E4M3

def test_e4m3_values_from_the_format_definition():
    """Codes worked from the E4M3 layout (bias 7, 3 mantissa bits): the
    largest finite value, the subnormals, exact values, ties to even and
    saturation."""
    cases = {448.0: 448.0, 500.0: 448.0, -1e6: -448.0, 2.0 ** -9: 2.0 ** -9, 2.0 ** -10: 0.0,
             3 * 2.0 ** -10: 2.0 ** -8, 1.0: 1.0, 1.0625: 1.0, 1.1875: 1.25, 1.125: 1.125,
             17.0: 16.0, 19.0: 20.0, -2.75: -2.75, 0.3: 0.3125, 240.0: 240.0, 232.0: 224.0}
    for v, want in cases.items():
        assert oracle.e4m3_round(v) == want, (v, oracle.e4m3_round(v), want)


def test_e4m3_matches_torch_float8_conversion():
    """Against torch's float8_e4m3fn conversion (a library routine the oracle
    does not use) on values inside the finite range."""
    v = np.concatenate([rnd(20000, 110) * 30, rnd(5000, 111) * 0.01, np.linspace(-448, 448, 4001)])
    t = torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(oracle.e4m3_round(np.float32(v).astype(np.float64)), t)


def test_fp8_projection_is_the_projection_of_the_dequantized_operands():
    B, T, C, H, Hk, D = 1, 6, 16, 2, 1, 8
    x = rnd((B, T, C), 112)
    w = rnd(((H + 2 * Hk) * D, C), 113) / 4
    q, k, v, (sx, sw) = oracle.qkv_projection_fp8(x, w, H, Hk, D)
    assert sx == np.float32(np.abs(np.float32(x)).max() / np.float32(448))
    xq = oracle.e4m3_round(np.float32(x) / np.float32(sx)) * sx
    wq = oracle.e4m3_round(np.float32(w) / np.float32(sw)) * sw
    assert np.all(np.abs(np.float32(x) / np.float32(sx)) <= 448.0001)
    rq, rk, rv = oracle.qkv_projection(xq, wq, H, Hk, D)
    np.testing.assert_array_equal(q, rq)
    # quantization error of the operands is small against the unquantized projection
    fq, _, _ = oracle.qkv_projection(x, w, H, Hk, D)
    assert np.linalg.norm(q - fq) / np.linalg.norm(fq) < 0.1
