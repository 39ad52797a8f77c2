"""Float64 CPU oracle for causal sliding-window RoPE attention (forward and backward).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. It shares no code
with the CUDA library and never imports it; the only thing both sides take in
common is the seeded input generator.

The arithmetic lives in ``oracle.c`` (plain C, float64, OpenMP over rows);
this module compiles it with gcc and marshals numpy float64 arrays. Every
step cites the page "5만원으로 나만의 ChatGPT 훈련하는 방법" (apidog.com),
section "1. GPT 모델 (nanochat/gpt.py)" (architecture list and the value
embedding code) and section "5. 플래시 어텐션 통합" (the causal windowed
attention call); see the header of ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

NO_NORM = 1
NO_ROPE = 2


class _Layer(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
        ("Hk", ctypes.c_int), ("D", ctypes.c_int), ("W", ctypes.c_int),
        ("has_ve", ctypes.c_int), ("flags", ctypes.c_int), ("pos_offset", ctypes.c_int),
        ("rope_base", ctypes.c_double), ("eps", ctypes.c_double), ("scale", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile oracle.c to liboracle.so with gcc (-O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _get():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        L = ctypes.POINTER(_Layer)
        _lib.oracle_prologue.argtypes = [L] + [dp] * 10
        _lib.oracle_attn_fwd.argtypes = [L] + [dp] * 5
        _lib.oracle_fwd_rows.argtypes = [L, dp, dp, dp, ctypes.c_int, ip, dp, dp]
        _lib.oracle_attn_bwd.argtypes = [L] + [dp] * 9
        _lib.oracle_dq_rows.argtypes = [L, dp, dp, dp, dp, ctypes.c_int, ip, dp]
        _lib.oracle_dkv_rows.argtypes = [L, dp, dp, dp, dp, ctypes.c_int, ip, dp, dp]
        _lib.oracle_prologue_bwd.argtypes = [L] + [dp] * 12
        _lib.oracle_probs_row.argtypes = [L, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, dp]
        _lib.oracle_probs_row.restype = ctypes.c_double
        _lib.oracle_decode.argtypes = [L] + [dp] * 5 + [ip] + [dp] * 4
        ci = ctypes.c_int
        _lib.oracle_gate_logits.argtypes = [ci] * 5 + [dp] * 3
        _lib.oracle_gate_bwd.argtypes = [ci] * 5 + [dp] * 5
    return _lib


class Layer:
    """Shape and switches of one attention layer.

    W is the number of visible keys, the query itself included; W >= T is
    plain causal attention. ``scale`` defaults to 1/sqrt(D). ``flags`` and
    ``pos_offset`` are test hooks (skip the norm / the rotation, shift the
    position origin).
    """

    def __init__(self, B, T, H, Hk, D, W, has_ve, rope_base=10000.0, eps=1e-6,
                 scale=None, flags=0, pos_offset=0):
        if H % Hk != 0:
            raise ValueError("n_head must be a multiple of n_kv_head")
        if D % 2 != 0 or D > 1024:
            raise ValueError("head_dim must be even and at most 1024")
        if W < 1:
            raise ValueError("window must be >= 1")
        self.B, self.T, self.H, self.Hk, self.D, self.W = B, T, H, Hk, D, W
        self.has_ve = bool(has_ve)
        self.rope_base, self.eps = float(rope_base), float(eps)
        self.scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
        self.flags, self.pos_offset = int(flags), int(pos_offset)

    def c(self):
        return _Layer(self.B, self.T, self.H, self.Hk, self.D, min(self.W, 2**31 - 1),
                      int(self.has_ve), self.flags, self.pos_offset,
                      self.rope_base, self.eps, self.scale)


def _f64(x, shape=None):
    if x is None:
        return None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"expected shape {tuple(shape)}, got {a.shape}")
    return a


def _p(a):
    if a is None:
        return ctypes.cast(0, ctypes.POINTER(ctypes.c_double))
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _rows(rows):
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    return r, r.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def prologue(L: Layer, q, k, v, ve=None, gate=None):
    """q~, k~, v_eff, rstd_q, rstd_k."""
    lib = _get()
    sq, skv = (L.B, L.T, L.H, L.D), (L.B, L.T, L.Hk, L.D)
    q, k, v = _f64(q, sq), _f64(k, skv), _f64(v, skv)
    if L.has_ve and (ve is None or gate is None):
        raise ValueError("has_ve layer needs ve and gate")
    ve = _f64(ve, skv) if L.has_ve else None
    gate = _f64(gate, (L.B, L.T, L.Hk)) if L.has_ve else None
    qt, kt, veff = np.empty(sq), np.empty(skv), np.empty(skv)
    rq, rk = np.empty((L.B, L.T, L.H)), np.empty((L.B, L.T, L.Hk))
    lib.oracle_prologue(ctypes.byref(L.c()), _p(q), _p(k), _p(v), _p(ve), _p(gate),
                        _p(qt), _p(kt), _p(veff), _p(rq), _p(rk))
    return qt, kt, veff, rq, rk


def attn_fwd(L: Layer, qt, kt, veff):
    """O (B,T,H,D) and lse (B,H,T), natural log."""
    lib = _get()
    qt, kt, veff = _f64(qt), _f64(kt), _f64(veff)
    O, lse = np.empty((L.B, L.T, L.H, L.D)), np.empty((L.B, L.H, L.T))
    lib.oracle_attn_fwd(ctypes.byref(L.c()), _p(qt), _p(kt), _p(veff), _p(O), _p(lse))
    return O, lse


def fwd_rows(L: Layer, qt, kt, veff, rows):
    """O and lse of selected rows; rows is a sequence of (b, h, i)."""
    lib = _get()
    qt, kt, veff = _f64(qt), _f64(kt), _f64(veff)
    r, rp = _rows(rows)
    O, lse = np.empty((len(r), L.D)), np.empty(len(r))
    lib.oracle_fwd_rows(ctypes.byref(L.c()), _p(qt), _p(kt), _p(veff), len(r), rp, _p(O), _p(lse))
    return O, lse


def attn_bwd(L: Layer, qt, kt, veff, O, lse, dO):
    """dq~ (B,T,H,D), dk~ and dv_eff (B,T,Hk,D)."""
    lib = _get()
    args = [_f64(a) for a in (qt, kt, veff, O, lse, dO)]
    dqt = np.empty((L.B, L.T, L.H, L.D))
    dkt, dveff = np.empty((L.B, L.T, L.Hk, L.D)), np.empty((L.B, L.T, L.Hk, L.D))
    lib.oracle_attn_bwd(ctypes.byref(L.c()), *[_p(a) for a in args], _p(dqt), _p(dkt), _p(dveff))
    return dqt, dkt, dveff


def dq_rows(L: Layer, qt, kt, veff, dO, rows):
    """dq~ of selected query rows (b, h, i), computed from scratch."""
    lib = _get()
    qt, kt, veff, dO = _f64(qt), _f64(kt), _f64(veff), _f64(dO)
    r, rp = _rows(rows)
    out = np.empty((len(r), L.D))
    lib.oracle_dq_rows(ctypes.byref(L.c()), _p(qt), _p(kt), _p(veff), _p(dO), len(r), rp, _p(out))
    return out


def dkv_rows(L: Layer, qt, kt, veff, dO, rows):
    """dk~ and dv_eff of selected key rows (b, hk, j), computed from scratch."""
    lib = _get()
    qt, kt, veff, dO = _f64(qt), _f64(kt), _f64(veff), _f64(dO)
    r, rp = _rows(rows)
    dk, dv = np.empty((len(r), L.D)), np.empty((len(r), L.D))
    lib.oracle_dkv_rows(ctypes.byref(L.c()), _p(qt), _p(kt), _p(veff), _p(dO), len(r), rp,
                        _p(dk), _p(dv))
    return dk, dv


def prologue_bwd(L: Layer, q, k, ve, gate, dqt, dkt, dveff):
    """dQ, dK, dV, dve, dgate (dve/dgate are None without a value embedding)."""
    lib = _get()
    q, k, dqt, dkt, dveff = (_f64(a) for a in (q, k, dqt, dkt, dveff))
    if L.has_ve and (ve is None or gate is None):
        raise ValueError("has_ve layer needs ve and gate")
    ve = _f64(ve) if L.has_ve else None
    gate = _f64(gate) if L.has_ve else None
    dq, dk, dv = np.empty(q.shape), np.empty(k.shape), np.empty(k.shape)
    dve = np.empty(k.shape) if L.has_ve else None
    dgate = np.empty((L.B, L.T, L.Hk)) if L.has_ve else None
    lib.oracle_prologue_bwd(ctypes.byref(L.c()), _p(q), _p(k), _p(ve), _p(gate), _p(dqt),
                            _p(dkt), _p(dveff), _p(dq), _p(dk), _p(dv), _p(dve), _p(dgate))
    return dq, dk, dv, dve, dgate


def probs_row(L: Layer, qt, kt, b, h, i):
    """Softmax row p_i. (length T, zeros where masked) and lse_i."""
    lib = _get()
    qt, kt = _f64(qt), _f64(kt)
    p = np.empty(L.T)
    lse = lib.oracle_probs_row(ctypes.byref(L.c()), _p(qt), _p(kt), b, h, i, _p(p))
    return p, lse


def layer(L: Layer, q, k, v, ve, gate, dO):
    """Whole layer, forward and backward. Returns a dict of float64 arrays."""
    qt, kt, veff, rq, rk = prologue(L, q, k, v, ve, gate)
    O, lse = attn_fwd(L, qt, kt, veff)
    dqt, dkt, dveff = attn_bwd(L, qt, kt, veff, O, lse, dO)
    dq, dk, dv, dve, dgate = prologue_bwd(L, q, k, ve, gate, dqt, dkt, dveff)
    return dict(qt=qt, kt=kt, veff=veff, rstd_q=rq, rstd_k=rk, O=O, lse=lse,
                dqt=dqt, dkt=dkt, dveff=dveff, dq=dq, dk=dk, dv=dv, dve=dve, dgate=dgate)


def decode(L: Layer, q, k, v, ve, gate, lens, kcache, vcache):
    """One decode step with a KV cache (L.T = cache capacity). q (B,H,D);
    k, v, ve (B,Hk,D); gate (B,Hk); lens (B,) tokens already cached; the
    caches (B,T,Hk,D) hold k~ and v_eff rows. Returns (O (B,H,D), lse (B,H),
    kcache', vcache') with the new token's rows written at position lens[b]."""
    if L.has_ve and (ve is None or gate is None):
        raise ValueError("layer has a value embedding: ve and gate are required")
    B, H, Hk, D = L.B, L.H, L.Hk, L.D
    q, k, v = _f64(q, (B, H, D)), _f64(k, (B, Hk, D)), _f64(v, (B, Hk, D))
    ve = _f64(ve, (B, Hk, D)) if L.has_ve else np.zeros((B, Hk, D))
    gate = _f64(gate, (B, Hk)) if L.has_ve else np.zeros((B, Hk))
    lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32).reshape(B))
    if (lens < 0).any() or (lens >= L.T).any():
        raise ValueError("cache lengths must lie in [0, T)")
    kc = _f64(kcache, (B, L.T, Hk, D)).copy()
    vc = _f64(vcache, (B, L.T, Hk, D)).copy()
    O = np.zeros((B, H, D))
    lse = np.zeros((B, H))
    _get().oracle_decode(L.c(), _p(q), _p(k), _p(v), _p(ve), _p(gate),
                         lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), _p(kc), _p(vc), _p(O), _p(lse))
    return O, lse, kc, vc


def gate_logits(x, w, C):
    """Gate logits of the value-embedding gate: x[..., :C] @ w.T, x (B, T, X)
    with X >= C, w (Hk, C); returns (B, T, Hk)."""
    x = _f64(x)
    w = _f64(w)
    B, T, X = x.shape
    Hk = w.shape[0]
    if w.shape[1] != C or X < C:
        raise ValueError("w must be (Hk, C) and x must have at least C channels")
    out = np.empty((B, T, Hk))
    _get().oracle_gate_logits(B, T, Hk, C, X, _p(x), _p(w), _p(out))
    return out


def gate_bwd(x, w, C, dgate):
    """dx (B, T, C) and dw (Hk, C) of the gate projection given dL/dgate."""
    x, w, dgate = _f64(x), _f64(w), _f64(dgate)
    B, T, X = x.shape
    Hk = w.shape[0]
    dx = np.empty((B, T, C))
    dw = np.empty((Hk, C))
    _get().oracle_gate_bwd(B, T, Hk, C, X, _p(x), _p(w), _p(dgate), _p(dx), _p(dw))
    return dx, dw


# ---------------------------------------------------------------- Muon orthogonalisation

# The coefficient triples (a, b, c) the page prints for the first two steps of
# the "Polar Express" iteration (page "5만원으로 나만의 ChatGPT 훈련하는 방법",
# section "2. Muon 옵티마이저 (nanochat/optim.py)"); the rest of its list is
# elided there, so callers pass the triples they want to apply.
POLAR_EXPRESS_PRINTED = ((8.156, -22.483, 15.879), (4.043, -2.809, 0.500))


def newton_schulz(X, coeffs):
    """The quintic Newton-Schulz iteration of the same section, in float64,
    one step per (a, b, c) triple, in the page's order and notation:
        A = X^T X;  B = b A + c A A;  X = a X + X B.
    X is (m, n); returns the iterate after len(coeffs) steps."""
    X = np.array(X, dtype=np.float64, copy=True)
    for a, b, c in coeffs:
        A = X.T @ X
        B = b * A + c * (A @ A)
        X = a * X + X @ B
    return X


def gemm(A, B, alpha=1.0, D=None, beta=0.0):
    """C = alpha A B + beta D in float64 (the product the iteration's steps
    are made of)."""
    C = alpha * (np.asarray(A, np.float64) @ np.asarray(B, np.float64))
    if D is not None and beta != 0.0:
        C = C + beta * np.asarray(D, np.float64)
    return C


# ---------------------------------------------------------------- QKV projection

def qkv_projection(x, w_qkv, H, Hk, D):
    """q, k, v of the layer from the block input x (B, T, C) and the stacked
    bias-free projection weight w_qkv ((H + 2 Hk) D, C) (rows: the H query
    heads, then the Hk key heads, then the Hk value heads), float64:
    q = x w_q^T viewed (B, T, H, D), likewise k and v with Hk heads."""
    x = _f64(x)
    w = _f64(w_qkv)
    B, T, C = x.shape
    if w.shape != ((H + 2 * Hk) * D, C):
        raise ValueError("w_qkv must be ((H + 2 Hk) D, C)")
    y = x.reshape(B * T, C) @ w.T
    q = y[:, :H * D].reshape(B, T, H, D)
    k = y[:, H * D:(H + Hk) * D].reshape(B, T, Hk, D)
    v = y[:, (H + Hk) * D:].reshape(B, T, Hk, D)
    return q, k, v


def qkv_projection_bwd(x, w_qkv, dq, dk, dv):
    """dx (B, T, C) and dw_qkv of the projection given the gradients of q, k, v."""
    x = _f64(x)
    w = _f64(w_qkv)
    B, T, C = x.shape
    dy = np.concatenate([_f64(dq).reshape(B * T, -1), _f64(dk).reshape(B * T, -1),
                         _f64(dv).reshape(B * T, -1)], axis=1)
    return (dy @ w).reshape(B, T, C), dy.T @ x.reshape(B * T, C)


# ---------------------------------------------------------------- FP8 (E4M3) projection

E4M3_MAX = 448.0


def e4m3_round(v):
    """Nearest FP8 E4M3 value (OCP 8-bit floating point: 1 sign, 4 exponent
    bits with bias 7, 3 mantissa bits; largest finite 448, smallest subnormal
    2^-9), ties to even, magnitudes above 448 saturated to 448."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    out = np.zeros_like(a)
    sub = a < 2.0 ** -6                      # subnormal range: steps of 2^-9
    out[sub] = np.round(a[sub] / 2.0 ** -9) * 2.0 ** -9   # numpy rounds halves to even
    nrm = ~sub
    e = np.floor(np.log2(np.where(nrm, a, 1.0)))
    step = 2.0 ** (e - 3)                    # 3 mantissa bits below the leading one
    out[nrm] = (np.round(a / step) * step)[nrm]
    out = np.minimum(out, E4M3_MAX)
    return np.sign(v) * out


def fp8_tensor_scale(x):
    """Tensor-wise scale of a tensor for E4M3: amax / 448 in float32 (1 when
    the tensor is zero)."""
    amax = np.float32(np.max(np.abs(np.asarray(x, dtype=np.float32))))
    return np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(E4M3_MAX))


def quantize_e4m3(x, scale):
    """E4M3 values of x / scale, the division in float32 (returns float64
    copies of the FP8 values)."""
    return e4m3_round(np.asarray(x, dtype=np.float32) / np.float32(scale))


def qkv_projection_fp8(x, w_qkv, H, Hk, D):
    """The QKV projection with both operands quantized to E4M3 with
    tensor-wise scales (a Float8Linear with tensor-wise scaling):
    y = (Q(x / sx) Q(w / sw)^T) sx sw. Returns q, k, v and (sx, sw)."""
    sx, sw = fp8_tensor_scale(x), fp8_tensor_scale(w_qkv)
    xq = quantize_e4m3(x, sx) * np.float64(sx)
    wq = quantize_e4m3(w_qkv, sw) * np.float64(sw)
    q, k, v = qkv_projection(xq, wq, H, Hk, D)
    return q, k, v, (float(sx), float(sw))
