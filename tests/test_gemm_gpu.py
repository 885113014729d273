"""Parity of the tcgen05 GEMM D = alpha A^T B (the backward pass's dy^T zl and x^T dz) with a float64 product.

The operands are binary16, so every product a*b is exact in float64 and the
reference is the exact sum; the kernel accumulates in float32 on the tensor
cores.  Each element is compared against the float32-summation bound
|D - ref| <= (Kc + 1) * 2^-22 * alpha * sum_k |A[k][i] B[k][j]| (a generous
multiple of the unit roundoff 2^-24 per addition): a wrong index, a dropped
k block or a misplaced tile gives errors of the order of the sum itself.
Shapes cover ragged k (not a multiple of the 64-row stage), ragged i (a last
tile with fewer than 64 rows, so one of its two 64-wide slices is never
loaded), ragged j (last tiles 32, 64, 96 columns wide), more tiles than SMs
(the persistent loop and both accumulators), and a row pitch wider than the
matrix.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sub_bit_weight_b200 import lib as _lib
    return _lib


def _ref(A, B, alpha):
    a, b = A.astype(np.float64), B.astype(np.float64)
    return alpha * (a.T @ b), abs(alpha) * (np.abs(a).T @ np.abs(b))


def _check(D, A, B, alpha):
    ref, absdot = _ref(A, B, alpha)
    tol = (A.shape[0] + 1) * 2.0 ** -22 * absdot + 1e-30
    err = np.abs(D.astype(np.float64) - ref)
    bad = err > tol
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5], float((err / tol).max()))


def _operands(seed, Kc, Mr, Nc):
    rng = np.random.default_rng(seed)
    A = (rng.standard_normal((Kc, Mr)) * 0.5).astype(np.float16)
    B = (rng.standard_normal((Kc, Nc)) * 0.5).astype(np.float16)
    return A, B


@pytest.mark.parametrize("Kc,Mr,Nc,alpha", [
    (1, 8, 32, 1.0),             # smallest: one k row, a partial slice each way
    (64, 136, 96, 0.25),         # one stage; second i tile of 8 rows (one slice); j tile 96 wide
    (300, 1000, 2368, 2.0 ** -5),   # ragged k (4 stages + 44 rows), 104-row last i tile, 64-wide last j tile
    (200, 5120, 2048, 0.37),     # 320 tiles: more than the SMs, both accumulators, the ring wraps
    (2048, 520, 288, 1.0),       # 32 stages per tile, 32-wide last j tile
])
def test_gemm_parity(lib, Kc, Mr, Nc, alpha):
    A, B = _operands(Kc * 7 + Mr, Kc, Mr, Nc)
    dev = torch.device("cuda")
    At = torch.from_numpy(A).to(dev)
    Bt = torch.from_numpy(B).to(dev)
    al = torch.tensor([alpha], dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    D = lib.lb_gemm_at_b(At, Bt, al, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert lib.lb_last_launch_count() == 1
    _check(D.cpu().numpy(), A, B, alpha)


def test_gemm_pitched_and_padding_untouched(lib):
    """lda, ldb > the used widths, ldd > Nc: only the used columns are read, padding columns of D stay as they were."""
    Kc, Mr, Nc, lda, ldb, ldd = 130, 200, 160, 264, 200, 196
    rng = np.random.default_rng(5)
    A = (rng.standard_normal((Kc, lda))).astype(np.float16)
    B = (rng.standard_normal((Kc, ldb))).astype(np.float16)
    A[:, Mr:] = np.float16(np.nan)          # never read
    B[:, Nc:] = np.float16(np.nan)
    dev = torch.device("cuda")
    At, Bt = torch.from_numpy(A).to(dev), torch.from_numpy(B).to(dev)
    D = torch.full((Mr, ldd), -7.0, dtype=torch.float32, device=dev)
    al = torch.tensor([1.5], dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    st = lib._lib.lb_gemm_at_b(At.data_ptr(), lda, Bt.data_ptr(), ldb, D.data_ptr(), ldd, Kc, Mr, Nc,
                               al.data_ptr(), err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == lib.LB_OK
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    Dn = D.cpu().numpy()
    assert (Dn[:, Nc:] == -7.0).all()
    _check(Dn[:, :Nc], A[:, :Mr], B[:, :Nc], 1.5)


def test_gemm_non_finite_stays_in_its_row_and_column(lib):
    """An Inf in A column i and a NaN in B column j reach only D row i and column j."""
    Kc, Mr, Nc = 96, 256, 256
    A, B = _operands(11, Kc, Mr, Nc)
    A[40, 17] = np.float16(np.inf)
    B[3, 200] = np.float16(np.nan)
    dev = torch.device("cuda")
    al = torch.tensor([1.0], dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    D = lib.lb_gemm_at_b(torch.from_numpy(A).to(dev), torch.from_numpy(B).to(dev), al, err).cpu().numpy()
    finite = np.isfinite(D)
    expect = np.ones_like(finite)
    expect[17, :] = False
    expect[:, 200] = False
    assert (finite == expect).all()
    keep_i = np.ones(Mr, bool)
    keep_i[17] = False
    keep_j = np.ones(Nc, bool)
    keep_j[200] = False
    _check(D[keep_i][:, keep_j], A[:, keep_i], B[:, keep_j], 1.0)
