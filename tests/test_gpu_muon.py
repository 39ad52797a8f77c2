"""GPU parity of the tensor-core matrix product and of Muon's Newton-Schulz
orthogonalisation built from it, through the C ABI, against the float64
oracle on the same bf16 inputs.

Page "5만원으로 나만의 ChatGPT 훈련하는 방법", section "2. Muon 옵티마이저
(nanochat/optim.py)": A = X^T X; B = b A + c A A; X = a X + X B, with the
printed coefficient triples.

Tolerance: relative Frobenius error <= 1e-2 for one product (bf16 output
rounding is ~2e-3) and <= 2e-2 for the whole iteration (bf16 intermediates
after every product; a bf16 emulation of the same steps on the CPU stays
below 4e-3 at these sizes).
"""
import numpy as np
import pytest
import torch

import causal_sliding_window_rope_b200 as cs
import oracle

pytestmark = pytest.mark.gpu


def bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


def rel(a, b):
    a = a.double().cpu().numpy() if torch.is_tensor(a) else a
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("a_mn,b_mn", [(False, False), (False, True), (True, False), (True, True)])
# Every contiguous extent a multiple of 8 (16-byte rows); tiles ragged
# against the 128 x 128 output tile and the 64-wide K chunk; the last shape
# has enough tiles (17 x 9 = 153 >= 148 SMs) for the 128 x 256 tile, ragged
# in all three extents.
@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (296, 136, 200), (136, 8, 24), (640, 384, 1000),
                                   (2056, 2200, 200)])
def test_gemm_layouts_and_ragged_tiles(M, N, K, a_mn, b_mn):
    A = bf16((K, M) if a_mn else (M, K), 1 + M)
    B = bf16((K, N) if b_mn else (N, K), 2 + N)
    D = bf16((M, N), 3 + K)
    C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    cs.gemm_bf16(A.cuda(), B.cuda(), C, alpha=0.5, beta=-2.0, D=D.cuda(), a_mn=a_mn, b_mn=b_mn)
    cs.cswattn_sync_status()
    Aop = A.double().numpy().T if a_mn else A.double().numpy()
    Bop = B.double().numpy() if b_mn else B.double().numpy().T
    ref = oracle.gemm(Aop, Bop, 0.5, D.double().numpy(), -2.0)
    assert torch.isfinite(C.float()).all()
    assert rel(C, ref) <= 1e-2


def test_gemm_in_place_axpby():
    """D may be C: C = alpha A B + beta C."""
    M, N, K = 256, 192, 320
    A, B, C0 = bf16((M, K), 11), bf16((K, N), 12), bf16((M, N), 13)
    C = C0.cuda()
    cs.gemm_bf16(A.cuda(), B.cuda(), C, alpha=1.0, beta=3.0, D=C)
    cs.cswattn_sync_status()
    ref = oracle.gemm(A.double().numpy(), B.double().numpy(), 1.0, C0.double().numpy(), 3.0)
    assert rel(C, ref) <= 1e-2


CUBIC = [(1.5, -0.5, 0.0)] * 5  # the textbook cubic Newton-Schulz step for the polar factor


@pytest.mark.parametrize("m,n,name", [(256, 128, "printed"), (384, 512, "printed"), (1000, 264, "printed"),
                                      (6144, 1536, "printed"), (256, 128, "cubic"), (1000, 264, "cubic")])
def test_newton_schulz_matches_oracle(m, n, name):
    coeffs = oracle.POLAR_EXPRESS_PRINTED if name == "printed" else CUBIC
    X = bf16((m, n), 20 + m)
    X = (X.double() / X.double().norm()).to(torch.bfloat16)
    Y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(cs.muon_ns_workspace_bytes(m, n), dtype=torch.uint8, device="cuda")
    cs.muon_newton_schulz(X.cuda(), Y, coeffs, ws)
    cs.cswattn_sync_status()
    ref = oracle.newton_schulz(X.double().numpy(), coeffs)
    assert torch.isfinite(Y.float()).all()
    assert rel(Y, ref) <= 2e-2


def test_newton_schulz_twice_in_a_row_is_identical():
    m, n = 512, 256
    X = bf16((m, n), 31)
    X = (X.double() / X.double().norm()).to(torch.bfloat16).cuda()
    ws = torch.empty(cs.muon_ns_workspace_bytes(m, n), dtype=torch.uint8, device="cuda")
    Y1 = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    Y2 = torch.empty_like(Y1)
    cs.muon_newton_schulz(X, Y1, oracle.POLAR_EXPRESS_PRINTED, ws)
    cs.muon_newton_schulz(X, Y2, oracle.POLAR_EXPRESS_PRINTED, ws)
    cs.cswattn_sync_status()
    assert torch.equal(Y1, Y2)
