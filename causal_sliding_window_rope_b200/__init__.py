"""B200-native causal sliding-window RoPE attention (forward and backward).

A thin ctypes binding over libcswattn.so, the C ABI declared in
``include/cswattn.h``. Every step of the computation runs in the library's
CUDA kernels; this module only marshals pointers, sizes and the stream.
PyTorch provides device memory and streams.

The layer is the attention of a nanochat-style GPT block (page
"5만원으로 나만의 ChatGPT 훈련하는 방법", section "1. GPT 모델"): RoPE,
parameter-free QK RMSNorm, GQA, a per-layer sliding window ("SSSL") and the
value-embedding residual v + 3*sigmoid(gate)*ve.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

from .configs import WORKLOADS, Workload, alternating_ve, window_pattern  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
# CSWATTN_CHECK=1 in the environment selects the checked build (device-side
# bounds checks that report CSWATTN_ERR_BOUNDS instead of faulting); build it
# with `python -m causal_sliding_window_rope_b200.build --check`.
CHECKED = os.environ.get("CSWATTN_CHECK", "0") == "1"
LIB_PATH = os.path.join(_HERE, "libcswattn_check.so" if CHECKED else "libcswattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = 0, 1, 2, 3, 4, 5
F32, BF16 = 0, 1

# Every symbol the header declares; the CPU tests check the library exports them.
EXPORTS = ("attn_prologue", "attn_prologue_gated", "attn_gate_bwd", "attn_qkv_prologue",
           "attn_qkv_fp8_workspace_bytes", "attn_qkv_prologue_fp8", "attn_qkv_bwd", "attn_fwd",
           "attn_bwd_workspace_bytes", "attn_bwd", "attn_bwd_noalloc",
           "attn_decode_workspace_bytes", "attn_decode", "cswattn_gemm_bf16",
           "muon_ns_workspace_bytes", "muon_newton_schulz",
           "cswattn_sync_status", "cswattn_set_wait_limit_ns", "cswattn_set_timing",
           "cswattn_kernel_times", "cswattn_selftest_wait_timeout", "cswattn_last_error",
           "cswattn_version")
KERNEL_KINDS = ("prologue", "fwd", "bwd_pre", "bwd", "bwd_epi", "decode", "gate_bwd", "gemm")


class CswattnLayer(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("n_head", ctypes.c_int),
        ("n_kv_head", ctypes.c_int), ("head_dim", ctypes.c_int), ("window", ctypes.c_int),
        ("rope_base", ctypes.c_float), ("eps", ctypes.c_float), ("softmax_scale", ctypes.c_float),
        ("has_ve", ctypes.c_int), ("dtype", ctypes.c_int),
    ]


class CswattnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"cswattn status {status}: {message}")
        self.status = status


_lib = None


def lib():
    """The loaded library. Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m causal_sliding_window_rope_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
        lp = ctypes.POINTER(CswattnLayer)
        L.attn_prologue.argtypes = [lp] + [vp] * 8 + [fp, fp, vp]
        L.attn_fwd.argtypes = [lp, vp, vp, vp, vp, fp, vp]
        ll, ci = ctypes.c_longlong, ctypes.c_int
        L.attn_prologue_gated.argtypes = [lp] + [vp] * 5 + [ll, ci, vp, vp, vp, vp, vp, fp, fp, vp]
        L.attn_gate_bwd.argtypes = [lp, vp, ll, ci, vp, vp, vp, fp, vp]
        L.attn_qkv_prologue.argtypes = [lp, vp, ll, ci] + [vp] * 8 + [fp, fp, vp]
        L.attn_qkv_prologue.restype = ci
        L.attn_qkv_fp8_workspace_bytes.argtypes = [lp, ci]
        L.attn_qkv_fp8_workspace_bytes.restype = sz
        L.attn_qkv_prologue_fp8.argtypes = [lp, vp, ll, ci] + [vp] * 8 + [fp, fp, fp, vp, sz, vp]
        L.attn_qkv_prologue_fp8.restype = ci
        L.attn_qkv_bwd.argtypes = [lp, vp, ll, ci] + [vp] * 5 + [fp, vp]
        L.attn_qkv_bwd.restype = ci
        cf = ctypes.c_float
        L.cswattn_gemm_bf16.argtypes = [ci, ci, ci, ci, vp, ll, ci, vp, ll, cf, cf, vp, ll, vp, ll, vp]
        L.cswattn_gemm_bf16.restype = ci
        L.muon_ns_workspace_bytes.argtypes = [ci, ci]
        L.muon_ns_workspace_bytes.restype = sz
        L.muon_newton_schulz.argtypes = [ci, ci, ctypes.POINTER(cf), ci, vp, vp, vp, sz, vp]
        L.muon_newton_schulz.restype = ci
        L.attn_bwd_workspace_bytes.argtypes = [lp]
        L.attn_bwd_workspace_bytes.restype = sz
        L.attn_bwd.argtypes = [lp] + [vp] * 7 + [fp, fp, vp, fp, vp] + [vp] * 6 + [sz, vp]
        L.cswattn_sync_status.argtypes = [vp]
        L.cswattn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.cswattn_set_wait_limit_ns.restype = ctypes.c_uint64
        L.cswattn_last_error.restype = ctypes.c_char_p
        L.cswattn_set_timing.argtypes = [ctypes.c_int]
        L.cswattn_set_timing.restype = None
        L.cswattn_kernel_times.argtypes = [ctypes.POINTER(ctypes.c_double),
                                           ctypes.POINTER(ctypes.c_int)]
        L.cswattn_kernel_times.restype = ctypes.c_int
        L.cswattn_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
        L.cswattn_selftest_wait_timeout.restype = ctypes.c_int
        L.attn_bwd_noalloc.argtypes = [lp] + [vp] * 7 + [fp, fp, vp, fp, vp] + [vp] * 5 + [vp]
        L.attn_decode_workspace_bytes.argtypes = [lp]
        L.attn_decode_workspace_bytes.restype = sz
        L.attn_decode.argtypes = [lp] + [vp] * 5 + [vp, vp, vp, vp, fp, vp, sz, vp]
        for name in ("attn_prologue", "attn_prologue_gated", "attn_gate_bwd", "attn_fwd", "attn_bwd",
                     "attn_bwd_noalloc", "cswattn_sync_status"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


@dataclass
class LayerSpec:
    """Arguments of one layer, as in the C struct ``cswattn_layer``."""
    B: int
    T: int
    n_head: int
    n_kv_head: int
    head_dim: int
    window: int
    has_ve: bool = True
    dtype: str = "bf16"          # "bf16" or "f32"
    rope_base: float = 10000.0
    eps: float = 1e-6
    softmax_scale: float = 0.0   # 0: 1/sqrt(head_dim)

    def c(self) -> CswattnLayer:
        return CswattnLayer(self.B, self.T, self.n_head, self.n_kv_head, self.head_dim,
                            self.window, self.rope_base, self.eps, self.softmax_scale,
                            int(bool(self.has_ve)), BF16 if self.dtype == "bf16" else F32)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_contiguous():
        raise ValueError("tensors passed to cswattn must be contiguous")
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != OK:
        raise CswattnError(status, lib().cswattn_last_error().decode())


def attn_prologue(spec: LayerSpec, q, k, v, ve, gate, q_out, k_out, v_out, rstd_q, rstd_k,
                  stream=None):
    layer = spec.c()
    _check(lib().attn_prologue(ctypes.byref(layer), _ptr(q), _ptr(k), _ptr(v), _ptr(ve),
                               _ptr(gate), _ptr(q_out), _ptr(k_out), _ptr(v_out),
                               _ptr(rstd_q), _ptr(rstd_k), _stream(stream)))


def attn_prologue_gated(spec: LayerSpec, q, k, v, ve, x, gate_channels, w_gate, gate_out, q_out,
                        k_out, v_out, rstd_q, rstd_k, stream=None):
    """attn_prologue with the gate logits computed from the block input:
    gate_out = x[..., :gate_channels] @ w_gate.T (x (B, T, X) contiguous)."""
    layer = spec.c()
    _check(lib().attn_prologue_gated(ctypes.byref(layer), _ptr(q), _ptr(k), _ptr(v), _ptr(ve),
                                     _ptr(x), int(x.shape[-1]), int(gate_channels), _ptr(w_gate),
                                     _ptr(gate_out), _ptr(q_out), _ptr(k_out), _ptr(v_out),
                                     _ptr(rstd_q), _ptr(rstd_k), _stream(stream)))


def attn_gate_bwd(spec: LayerSpec, x, gate_channels, w_gate, dgate, dx, dw_gate, stream=None):
    """dx (B, T, gate_channels) and float32 dw_gate (Hk, gate_channels) of the
    gate projection, from dgate (the attention backward's dgate)."""
    layer = spec.c()
    _check(lib().attn_gate_bwd(ctypes.byref(layer), _ptr(x), int(x.shape[-1]), int(gate_channels),
                               _ptr(w_gate), _ptr(dgate), _ptr(dx), _ptr(dw_gate), _stream(stream)))


def attn_qkv_prologue(spec: LayerSpec, x, C, w_qkv, ve, gate, q, k, q_out, k_out, v_out, rstd_q,
                      rstd_k, stream=None):
    """The QKV projection of x[..., :C] by the stacked weight w_qkv, fused with
    the prologue (see the C header); q and k receive the raw projections."""
    layer = spec.c()
    _check(lib().attn_qkv_prologue(ctypes.byref(layer), _ptr(x), int(x.shape[-1]), int(C), _ptr(w_qkv),
                                   _ptr(ve), _ptr(gate), _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out),
                                   _ptr(v_out), _ptr(rstd_q), _ptr(rstd_k), _stream(stream)))


def attn_qkv_fp8_workspace_bytes(spec: LayerSpec, C) -> int:
    layer = spec.c()
    return int(lib().attn_qkv_fp8_workspace_bytes(ctypes.byref(layer), int(C)))


def attn_qkv_prologue_fp8(spec: LayerSpec, x, C, w_qkv, ve, gate, q, k, q_out, k_out, v_out, rstd_q,
                          rstd_k, scales, workspace, workspace_bytes=None, stream=None):
    """attn_qkv_prologue with both operands quantized to E4M3 with tensor-wise
    scales (written to `scales`); `workspace` holds the codes afterwards."""
    layer = spec.c()
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(lib().attn_qkv_prologue_fp8(ctypes.byref(layer), _ptr(x), int(x.shape[-1]), int(C), _ptr(w_qkv),
                                       _ptr(ve), _ptr(gate), _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out),
                                       _ptr(v_out), _ptr(rstd_q), _ptr(rstd_k), _ptr(scales), _ptr(workspace),
                                       int(nbytes), _stream(stream)))


def attn_qkv_bwd(spec: LayerSpec, x, C, w_qkv, dQ, dK, dV, dx, dw_qkv, stream=None):
    """dx (B, T, C) and float32 dw_qkv of the projection from attn_bwd's dQ, dK, dV."""
    layer = spec.c()
    _check(lib().attn_qkv_bwd(ctypes.byref(layer), _ptr(x), int(x.shape[-1]), int(C), _ptr(w_qkv),
                              _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dx), _ptr(dw_qkv), _stream(stream)))


def attn_fwd(spec: LayerSpec, q_out, k_out, v_out, O, lse, stream=None):
    layer = spec.c()
    _check(lib().attn_fwd(ctypes.byref(layer), _ptr(q_out), _ptr(k_out), _ptr(v_out),
                          _ptr(O), _ptr(lse), _stream(stream)))


def attn_bwd_workspace_bytes(spec: LayerSpec) -> int:
    layer = spec.c()
    return int(lib().attn_bwd_workspace_bytes(ctypes.byref(layer)))


def attn_bwd(spec: LayerSpec, q, k, ve, gate, q_out, k_out, v_out, rstd_q, rstd_k, O, lse,
             dO, dQ, dK, dV, dve, dgate, workspace, workspace_bytes=None, stream=None):
    layer = spec.c()
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().attn_bwd(ctypes.byref(layer), _ptr(q), _ptr(k), _ptr(ve), _ptr(gate),
                          _ptr(q_out), _ptr(k_out), _ptr(v_out), _ptr(rstd_q), _ptr(rstd_k),
                          _ptr(O), _ptr(lse), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV),
                          _ptr(dve), _ptr(dgate), _ptr(workspace), workspace_bytes,
                          _stream(stream)))


# Size of the fixed scratch array behind attn_bwd_noalloc (bytes).
NOALLOC_SCRATCH_BYTES = 32 << 20


def attn_bwd_noalloc(spec: LayerSpec, q, k, ve, gate, q_out, k_out, v_out, rstd_q, rstd_k, O,
                     lse, dO, dQ, dK, dV, dve, dgate, stream=None):
    """attn_bwd for callers that cannot allocate device memory: the scratch is
    a fixed array inside the library (see the C header for the limit and for
    why overlapping calls must be ordered)."""
    layer = spec.c()
    _check(lib().attn_bwd_noalloc(ctypes.byref(layer), _ptr(q), _ptr(k), _ptr(ve), _ptr(gate),
                                  _ptr(q_out), _ptr(k_out), _ptr(v_out), _ptr(rstd_q),
                                  _ptr(rstd_k), _ptr(O), _ptr(lse), _ptr(dO), _ptr(dQ), _ptr(dK),
                                  _ptr(dV), _ptr(dve), _ptr(dgate), _stream(stream)))


def attn_decode_workspace_bytes(spec: LayerSpec) -> int:
    """Scratch bytes of attn_decode; spec.T is the cache capacity."""
    layer = spec.c()
    return int(lib().attn_decode_workspace_bytes(ctypes.byref(layer)))


def attn_decode(spec: LayerSpec, q, k, v, ve, gate, cache_len, k_cache, v_cache, O, lse,
                workspace, workspace_bytes=None, stream=None):
    """One decode step with a KV cache (spec.T = cache capacity, cache_len an
    int32 device tensor of B lengths): writes the new token's k~ / v_eff rows
    into the caches and its attention output O (B,H,D) and lse (B,H)."""
    layer = spec.c()
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().attn_decode(ctypes.byref(layer), _ptr(q), _ptr(k), _ptr(v), _ptr(ve), _ptr(gate),
                             _ptr(cache_len), _ptr(k_cache), _ptr(v_cache), _ptr(O), _ptr(lse),
                             _ptr(workspace), workspace_bytes, _stream(stream)))


def cswattn_sync_status(stream=None):
    _check(lib().cswattn_sync_status(_stream(stream)))


def cswattn_set_wait_limit_ns(ns: int) -> int:
    """Sets the device-side wait limit; returns the limit applied (>= 1 ms)."""
    return int(lib().cswattn_set_wait_limit_ns(int(ns)))


def cswattn_set_timing(enable: bool):
    lib().cswattn_set_timing(1 if enable else 0)


def cswattn_kernel_times():
    """{kind: (total_ms, launches)} since the last read, for the kernel kinds."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int * n)()
    _check(lib().cswattn_kernel_times(ms, cnt))
    return {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_KINDS)}


def cswattn_selftest_wait_timeout(limit_ns: int, stream=None):
    """Launch the bounded-wait self-test kernel (its wait always runs out)."""
    _check(lib().cswattn_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def cswattn_version() -> int:
    return int(lib().cswattn_version())


# ------------------------------------------------------------------ convenience

class LayerBuffers:
    """Device buffers of one layer (torch tensors), allocated once and reused."""

    def __init__(self, spec: LayerSpec, device="cuda"):
        import torch
        dt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
        B, T, H, Hk, D = spec.B, spec.T, spec.n_head, spec.n_kv_head, spec.head_dim
        e = dict(device=device, dtype=dt)
        f = dict(device=device, dtype=torch.float32)
        self.spec = spec
        self.q_out = torch.empty(B, T, H, D, **e)
        self.k_out = torch.empty(B, T, Hk, D, **e)
        self.v_out = torch.empty(B, T, Hk, D, **e)
        self.rstd_q = torch.empty(B, T, H, **f)
        self.rstd_k = torch.empty(B, T, Hk, **f)
        self.O = torch.empty(B, T, H, D, **e)
        self.lse = torch.empty(B, H, T, **f)
        self.dQ = torch.empty(B, T, H, D, **e)
        self.dK = torch.empty(B, T, Hk, D, **e)
        self.dV = torch.empty(B, T, Hk, D, **e)
        self.dve = torch.empty(B, T, Hk, D, **e) if spec.has_ve else None
        self.dgate = torch.empty(B, T, Hk, **e) if spec.has_ve else None
        nbytes = attn_bwd_workspace_bytes(spec)
        self.workspace = torch.empty(max(nbytes, 256), device=device, dtype=torch.uint8)


def layer_forward(spec: LayerSpec, buf: LayerBuffers, q, k, v, ve=None, gate=None, stream=None):
    attn_prologue(spec, q, k, v, ve, gate, buf.q_out, buf.k_out, buf.v_out, buf.rstd_q,
                  buf.rstd_k, stream)
    attn_fwd(spec, buf.q_out, buf.k_out, buf.v_out, buf.O, buf.lse, stream)


def layer_backward(spec: LayerSpec, buf: LayerBuffers, q, k, ve, gate, dO, stream=None):
    attn_bwd(spec, q, k, ve, gate, buf.q_out, buf.k_out, buf.v_out, buf.rstd_q, buf.rstd_k,
             buf.O, buf.lse, dO, buf.dQ, buf.dK, buf.dV, buf.dve, buf.dgate, buf.workspace,
             stream=stream)


# ------------------------------------------------------------------ Muon

def gemm_bf16(A, B, C, alpha=1.0, beta=0.0, D=None, a_mn=False, b_mn=True, stream=None):
    """C = alpha Aop Bop^T + beta D on the tensor cores (see the C header for
    Aop/Bop). Defaults: the plain product of row-major A (M x K), B (K x N)."""
    M, N = C.shape
    K = A.shape[0] if a_mn else A.shape[1]
    _check(lib().cswattn_gemm_bf16(M, N, K, int(a_mn), _ptr(A), A.stride(0), int(b_mn), _ptr(B),
                                   B.stride(0), float(alpha), float(beta), _ptr(D),
                                   D.stride(0) if D is not None else N, _ptr(C), C.stride(0),
                                   _stream(stream)))


def muon_ns_workspace_bytes(m: int, n: int) -> int:
    return int(lib().muon_ns_workspace_bytes(m, n))


def muon_newton_schulz(X, Y, coeffs, workspace, stream=None):
    """Muon's Newton-Schulz iteration, one step per (a, b, c) triple, from the
    bf16 m x n matrix X into Y (see the C header)."""
    m, n = X.shape
    flat = [float(v) for t in coeffs for v in t]
    arr = (ctypes.c_float * len(flat))(*flat)
    _check(lib().muon_newton_schulz(m, n, arr, len(coeffs), _ptr(X), _ptr(Y), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))
