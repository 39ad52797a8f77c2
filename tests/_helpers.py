"""Shared test helpers: run one layer through the C ABI and through the oracle."""
from __future__ import annotations

import numpy as np
import torch

import causal_sliding_window_rope_b200 as cs
import oracle
from causal_sliding_window_rope_b200 import synth

TORCH_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def make_inputs(B, T, H, Hk, D, has_ve, dtype, config=0, layer=0, dO_std=1.0):
    return synth.layer_inputs(B, T, H, Hk, D, has_ve, TORCH_DT[dtype], config, layer, dO_std)


def to_dev(x):
    return None if x is None else x.cuda()


def f64(x):
    return None if x is None else x.detach().double().cpu().numpy()


def run_gpu(spec: cs.LayerSpec, inp):
    """Prologue, forward and backward through the C ABI. Returns host float64 arrays."""
    dev = {k: to_dev(v) for k, v in inp.items()}
    buf = cs.LayerBuffers(spec)
    cs.layer_forward(spec, buf, dev["q"], dev["k"], dev["v"], dev["ve"], dev["gate"])
    cs.layer_backward(spec, buf, dev["q"], dev["k"], dev["ve"], dev["gate"], dev["dO"])
    cs.cswattn_sync_status()
    torch.cuda.synchronize()
    out = dict(qt=buf.q_out, kt=buf.k_out, veff=buf.v_out, rstd_q=buf.rstd_q, rstd_k=buf.rstd_k,
               O=buf.O, lse=buf.lse, dq=buf.dQ, dk=buf.dK, dv=buf.dV, dve=buf.dve, dgate=buf.dgate)
    return {k: f64(v) for k, v in out.items()}, buf


def oracle_layer(spec: cs.LayerSpec, inp):
    L = oracle.Layer(spec.B, spec.T, spec.n_head, spec.n_kv_head, spec.head_dim, spec.window,
                     spec.has_ve, rope_base=spec.rope_base, eps=spec.eps)
    return L, oracle.layer(L, f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["ve"]),
                           f64(inp["gate"]), f64(inp["dO"]))


def rel_frob(a, ref):
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / den) if den > 0 else float(np.linalg.norm(a))


def max_abs(a, ref):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(ref, np.float64))))


OUT_KEYS = ("O", "lse", "dq", "dk", "dv", "dve", "dgate")
