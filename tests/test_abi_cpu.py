"""C ABI checks that need no GPU: the library loads, exports what the header
declares, and rejects bad arguments on the host with the documented codes
before anything is enqueued."""
import ctypes
import os
import re

import pytest

import causal_sliding_window_rope_b200 as cs
from causal_sliding_window_rope_b200 import build as cs_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "cswattn.h")


@pytest.fixture(scope="module")
def lib():
    cs_build.build()
    return cs.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:cswattn_status|size_t|uint64_t|void|const char\s*\*|int)\s+(\w+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(cs.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), n


def test_version(lib):
    assert cs.cswattn_version() >> 16 == 1


def call_fwd(spec, ptrs=(16, 32, 48, 64, 80)):
    layer = spec.c() if spec is not None else None
    ref = ctypes.byref(layer) if layer is not None else None
    return cs.lib().attn_fwd(ref, *ptrs, None)


@pytest.mark.parametrize("change,code", [
    (dict(B=0), cs.ERR_INVALID_ARG),
    (dict(T=0), cs.ERR_INVALID_ARG),
    (dict(window=0), cs.ERR_INVALID_ARG),
    (dict(n_kv_head=3), cs.ERR_INVALID_ARG),
    (dict(has_ve=2), cs.ERR_INVALID_ARG),
    (dict(rope_base=0.0), cs.ERR_INVALID_ARG),
    (dict(rope_base=float("inf")), cs.ERR_INVALID_ARG),
    (dict(eps=-1.0), cs.ERR_INVALID_ARG),
    (dict(softmax_scale=-0.5), cs.ERR_INVALID_ARG),
    (dict(head_dim=32), cs.ERR_UNSUPPORTED),
    (dict(head_dim=96), cs.ERR_UNSUPPORTED),
    (dict(head_dim=6, dtype="f32"), cs.ERR_UNSUPPORTED),
    (dict(T=(1 << 20) + 1), cs.ERR_UNSUPPORTED),
])
def test_layer_validation(lib, change, code):
    base = dict(B=2, T=64, n_head=4, n_kv_head=2, head_dim=128, window=32)
    spec = cs.LayerSpec(**{**base, **change})
    layer = spec.c()
    if "has_ve" in change:
        layer.has_ve = change["has_ve"]
    assert lib.attn_fwd(ctypes.byref(layer), 16, 32, 48, 64, 80, None) == code
    assert lib.cswattn_last_error().decode() != ""
    assert lib.attn_bwd_workspace_bytes(ctypes.byref(layer)) == 0


@pytest.mark.parametrize("D,dtype", [(64, "bf16"), (128, "bf16"), (4, "f32"), (64, "f32")])
def test_supported_head_dims_pass_validation(lib, D, dtype):
    # A supported shape fails only on its (deliberately misaligned) pointers.
    spec = cs.LayerSpec(2, 64, 4, 2, D, 32, dtype=dtype)
    layer = spec.c()
    assert lib.attn_bwd_workspace_bytes(ctypes.byref(layer)) > 0
    assert lib.attn_fwd(ctypes.byref(layer), 16 + 8, 32, 48, 64, 80, None) == cs.ERR_INVALID_ARG
    assert b"aligned" in lib.cswattn_last_error()


def test_bad_dtype_and_null_layer(lib):
    spec = cs.LayerSpec(2, 64, 4, 2, 128, 32)
    layer = spec.c()
    layer.dtype = 7
    assert lib.attn_fwd(ctypes.byref(layer), 16, 32, 48, 64, 80, None) == cs.ERR_INVALID_ARG
    assert lib.attn_fwd(None, 16, 32, 48, 64, 80, None) == cs.ERR_INVALID_ARG


def test_pointer_validation(lib):
    spec = cs.LayerSpec(2, 64, 4, 2, 128, 32)
    layer = ctypes.byref(spec.c())
    assert lib.attn_fwd(layer, None, 32, 48, 64, 80, None) == cs.ERR_INVALID_ARG
    assert b"q_out" in lib.cswattn_last_error()
    assert lib.attn_fwd(layer, 16 + 8, 32, 48, 64, 80, None) == cs.ERR_INVALID_ARG
    assert b"aligned" in lib.cswattn_last_error()
    assert lib.attn_fwd(layer, 16, 32, 48, 64, 82, None) == cs.ERR_INVALID_ARG  # lse 4-byte
    # prologue: outputs may not alias inputs; ve/gate required with has_ve
    args = [16, 32, 48, 64, 80, 16, 112, 128, 144, 160, None]
    assert lib.attn_prologue(layer, *args) == cs.ERR_INVALID_ARG
    assert b"alias" in lib.cswattn_last_error()
    args = [16, 32, 48, None, 80, 96, 112, 128, 144, 160, None]
    assert lib.attn_prologue(layer, *args) == cs.ERR_INVALID_ARG
    assert b"ve" in lib.cswattn_last_error()


def test_workspace_size_and_check(lib):
    spec = cs.LayerSpec(2, 100, 6, 2, 128, 32)
    n = cs.attn_bwd_workspace_bytes(spec)
    pad = lambda x: (x + 255) // 256 * 256  # noqa: E731
    B, T, H, Hk, D = 2, 100, 6, 2, 128
    Tpad = (T + 63) // 64 * 64
    # dq accumulator, P partial-sum slots each for dk and dv (1 <= P <= 8), two row terms
    fixed = pad(4 * B * H * T * D) + 2 * pad(4 * B * H * Tpad)
    assert any(n == fixed + 2 * pad(P * 4 * B * T * Hk * D) for P in range(1, 9))
    f32 = cs.LayerSpec(2, 100, 6, 2, 128, 32, dtype="f32")
    assert cs.attn_bwd_workspace_bytes(f32) == fixed + 2 * pad(4 * B * T * Hk * D)  # P = 1
    layer = ctypes.byref(spec.c())
    ptrs = [256 * (i + 1) for i in range(17)]
    st = lib.attn_bwd(layer, *ptrs[:12], *ptrs[12:17], 256 * 40, n - 1, None)
    assert st == cs.ERR_INVALID_ARG
    assert b"workspace" in lib.cswattn_last_error()


def test_decode_validation(lib):
    spec = cs.LayerSpec(2, 256, 12, 4, 128, 100, has_ve=True)
    n = cs.attn_decode_workspace_bytes(spec)
    # per split (max, sum) and partial O of every query head; 2 x 4 (sequence,
    # KV head) pairs would take 18 splits to cover 148 SMs, but a window of
    # 100 keys straddles at most 2 chunks of 128 (and the cache has 2)
    rows, chunks = 2 * 12, 2
    def pad(x):
        return (x + 255) // 256 * 256
    assert n == pad(rows * chunks * 2 * 4) + pad(rows * chunks * 128 * 4)
    assert cs.attn_decode_workspace_bytes(cs.LayerSpec(2, 256, 4, 2, 128, 64, dtype="f32")) == 0
    assert cs.attn_decode_workspace_bytes(cs.LayerSpec(2, 256, 34, 2, 128, 64)) == 0  # group 17
    assert cs.attn_decode_workspace_bytes(cs.LayerSpec(70000, 16, 4, 2, 128, 8)) == 0  # grid limit
    layer = ctypes.byref(spec.c())
    good = [256 * (i + 1) for i in range(5)]  # q k v ve gate
    args = good + [4096, 8192, 12288, 16384, 20480, 24576, n, None]
    assert lib.attn_decode(layer, *args[:5], 4096 + 2, *args[6:]) == cs.ERR_INVALID_ARG  # cache_len
    assert b"cache_len" in lib.cswattn_last_error()
    assert lib.attn_decode(layer, *args[:11], n - 1, None) == cs.ERR_INVALID_ARG
    assert b"workspace" in lib.cswattn_last_error()
    same = args[:7] + [args[6]] + args[8:]
    assert lib.attn_decode(layer, *same) == cs.ERR_INVALID_ARG


def test_header_enums_match_the_binding():
    """Status codes and kernel kinds in the header are the ones the Python
    binding uses (ctypes cannot check enums)."""
    text = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                             "include", "cswattn.h")).read()
    codes = dict(re.findall(r"CSWATTN_(OK|ERR_\w+)\s*=\s*(\d+)", text))
    assert int(codes["OK"]) == cs.OK
    for name in ("INVALID_ARG", "UNSUPPORTED", "CUDA", "TIMEOUT"):
        assert int(codes["ERR_" + name]) == getattr(cs, "ERR_" + name)
    kinds = re.findall(r"CSWATTN_K_(\w+)\s*=\s*(\d+)", text)
    assert [k.lower() for k, _ in sorted(kinds, key=lambda kv: int(kv[1]))] == list(cs.KERNEL_KINDS)
    assert int(re.search(r"CSWATTN_NUM_KERNELS\s*=\s*(\d+)", text).group(1)) == len(cs.KERNEL_KINDS)


def test_wait_limit_floor(lib):
    # Short limits are raised to 1 ms, far above any copy or product latency;
    # the kernels' final waits for their own copies have a fixed bound.
    assert cs.cswattn_set_wait_limit_ns(5) == 1_000_000
    assert cs.cswattn_set_wait_limit_ns(999_999) == 1_000_000
    assert cs.cswattn_set_wait_limit_ns(3_000_000) == 3_000_000
    assert cs.cswattn_set_wait_limit_ns(2_000_000_000) == 2_000_000_000


def test_build_tracks_every_kernel_source(tmp_path, monkeypatch):
    """Editing any kernel header, the translation unit or the public header
    makes the library stale, so build() recompiles it."""
    import shutil
    csrc = tmp_path / "csrc"
    shutil.copytree(cs_build.CSRC, csrc)
    header = tmp_path / "cswattn.h"
    shutil.copy(cs_build.HEADER, header)
    libf = tmp_path / "libcswattn.so"
    libf.write_bytes(b"")
    monkeypatch.setattr(cs_build, "CSRC", str(csrc))
    monkeypatch.setattr(cs_build, "HEADER", str(header))
    monkeypatch.setattr(cs_build, "LIB", str(libf))
    deps = cs_build.deps()
    names = {os.path.basename(d) for d in deps}
    assert {"decode.cuh", "bwd_sm100.cuh", "fwd_sm100.cuh", "cswattn.cu", "cswattn.h"} <= names
    copied = [d for d in deps if d.startswith(str(tmp_path))]  # never touch the real tree
    assert len(copied) == len(deps) - 1
    t_lib = 2_000_000_000
    for d in copied:
        os.utime(d, (t_lib - 10, t_lib - 10))
    os.utime(libf, (t_lib, t_lib))
    assert not cs_build.stale()
    for d in copied:
        os.utime(d, (t_lib + 10, t_lib + 10))
        assert cs_build.stale(), d
        os.utime(d, (t_lib - 10, t_lib - 10))


def test_gate_entry_point_validation(lib):
    """The gate projection needs a value embedding and 1 <= C <= x_stride."""
    ptrs = [256 * (i + 1) for i in range(12)]
    no_ve = cs.LayerSpec(1, 16, 2, 1, 128, 16, has_ve=False)
    st = lib.attn_prologue_gated(ctypes.byref(no_ve.c()), *ptrs[:5], 32, 32, *ptrs[5:12], None)
    assert st == cs.ERR_INVALID_ARG and b"value embedding" in lib.cswattn_last_error()
    spec = cs.LayerSpec(1, 16, 2, 1, 128, 16, has_ve=True)
    st = lib.attn_prologue_gated(ctypes.byref(spec.c()), *ptrs[:5], 16, 32, *ptrs[5:12], None)
    assert st == cs.ERR_INVALID_ARG and b"gate_channels" in lib.cswattn_last_error()
    st = lib.attn_gate_bwd(ctypes.byref(spec.c()), ptrs[0], 64, 0, *ptrs[1:5], None)
    assert st == cs.ERR_INVALID_ARG
    st = lib.attn_gate_bwd(ctypes.byref(no_ve.c()), ptrs[0], 64, 32, *ptrs[1:5], None)
    assert st == cs.ERR_INVALID_ARG


def test_gemm_and_newton_schulz_validation(lib):
    g = lib.cswattn_gemm_bf16
    ok_args = dict(M=128, N=128, K=64, a_mn=0, A=256, lda=64, b_mn=1, B=512, ldb=128,
                   alpha=1.0, beta=0.0, D=None, ldd=128, C=768, ldc=128)

    def call(**kw):
        a = {**ok_args, **kw}
        return g(a["M"], a["N"], a["K"], a["a_mn"], a["A"], a["lda"], a["b_mn"], a["B"], a["ldb"],
                 a["alpha"], a["beta"], a["D"], a["ldd"], a["C"], a["ldc"], None)

    assert call(N=12, ldb=16, ldc=16) == cs.ERR_UNSUPPORTED          # N not a multiple of 8
    assert call(lda=32) == cs.ERR_INVALID_ARG                        # row shorter than K
    assert call(lda=68) == cs.ERR_INVALID_ARG                        # not a multiple of 8
    assert call(C=256) == cs.ERR_INVALID_ARG                         # C aliases A
    assert call(beta=1.0, D=None) == cs.ERR_INVALID_ARG              # beta needs D
    assert call(M=0) == cs.ERR_INVALID_ARG
    coeffs = (ctypes.c_float * 6)(8.156, -22.483, 15.879, 4.043, -2.809, 0.5)
    n = lib.muon_ns_workspace_bytes(256, 128)
    assert n == 2 * 128 * 128 * 2 + 256 * 128 * 2
    ns = lib.muon_newton_schulz
    assert ns(256, 128, coeffs, 2, 256, 256, 1024, n, None) == cs.ERR_INVALID_ARG      # X == Y
    assert ns(256, 128, coeffs, 2, 256, 512, 1024, n - 1, None) == cs.ERR_INVALID_ARG  # workspace
    assert ns(256, 128, coeffs, 0, 256, 512, 1024, n, None) == cs.ERR_INVALID_ARG      # steps
    assert ns(256, 12, coeffs, 2, 256, 512, 1024, n, None) == cs.ERR_UNSUPPORTED       # n % 8


def test_checked_build_compiles_and_exports_the_same_symbols():
    """The CSWATTN_CHECK=1 build (device-side bounds checks that report
    CSWATTN_ERR_BOUNDS) compiles and exports what the header declares."""
    path = cs_build.build(check=True)
    assert path.endswith("libcswattn_check.so")
    checked = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(checked, n), n


def test_qkv_entry_point_validation(lib):
    ptrs = [256 * (i + 1) for i in range(12)]
    spec = cs.LayerSpec(1, 16, 2, 1, 128, 16, has_ve=False)
    f32 = cs.LayerSpec(1, 16, 2, 1, 64, 16, has_ve=False, dtype="f32")
    qp = lib.attn_qkv_prologue
    assert qp(ctypes.byref(f32.c()), ptrs[0], 64, 64, *ptrs[1:11], None) == cs.ERR_UNSUPPORTED
    assert qp(ctypes.byref(spec.c()), ptrs[0], 64, 60, *ptrs[1:11], None) == cs.ERR_INVALID_ARG  # C % 8
    assert qp(ctypes.byref(spec.c()), ptrs[0], 32, 64, *ptrs[1:11], None) == cs.ERR_INVALID_ARG  # stride < C
    qb = lib.attn_qkv_bwd
    assert qb(ctypes.byref(f32.c()), ptrs[0], 64, 64, *ptrs[1:7], None) == cs.ERR_UNSUPPORTED
    assert qb(ctypes.byref(spec.c()), ptrs[0], 64, 60, *ptrs[1:7], None) == cs.ERR_INVALID_ARG


def test_qkv_fp8_entry_point_validation(lib):
    """Host checks of the FP8 projection and its workspace size: 256 bytes of
    amax state, then the x codes (B*T*C bytes) and the weight codes
    ((H + 2 Hk) D C bytes), each padded to 256."""
    ptrs = [256 * (i + 1) for i in range(13)]
    spec = cs.LayerSpec(2, 100, 6, 2, 128, 16, has_ve=False)
    pad = lambda n: (n + 255) // 256 * 256
    C = 96
    assert lib.attn_qkv_fp8_workspace_bytes(ctypes.byref(spec.c()), C) == \
        256 + pad(2 * 100 * C) + pad(10 * 128 * C)
    assert lib.attn_qkv_fp8_workspace_bytes(ctypes.byref(spec.c()), 0) == 0
    ws = lib.attn_qkv_fp8_workspace_bytes(ctypes.byref(spec.c()), C)
    qp = lib.attn_qkv_prologue_fp8
    f32 = cs.LayerSpec(2, 100, 6, 2, 64, 16, has_ve=False, dtype="f32")
    assert qp(ctypes.byref(f32.c()), ptrs[0], C, C, *ptrs[1:12], ptrs[12], ws, None) == cs.ERR_UNSUPPORTED
    # C a multiple of 8 but not of 16: E4M3 rows must be whole 16-byte units
    assert qp(ctypes.byref(spec.c()), ptrs[0], 104, 104, *ptrs[1:12], ptrs[12], ws, None) == cs.ERR_INVALID_ARG
    # workspace one byte short
    assert qp(ctypes.byref(spec.c()), ptrs[0], C, C, *ptrs[1:12], ptrs[12], ws - 1, None) == cs.ERR_INVALID_ARG
    # workspace not 256-byte aligned
    assert qp(ctypes.byref(spec.c()), ptrs[0], C, C, *ptrs[1:12], 16, ws, None) == cs.ERR_INVALID_ARG
