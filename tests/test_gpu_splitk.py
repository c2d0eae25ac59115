"""GPU parity of kq_gemv_splitk: tall-skinny matrices (fewer row pairs than
SMs) split K across CTAs, write partial sums to a caller workspace and add
them in a fixed order.  Checked against the oracle; deterministic; column c
of a k-column call equals column c of an 8-column call bitwise."""
import numpy as np
import pytest
import torch

import oracle
from kqtest import assert_close, dev, matrix, oracle_gemv, x_vec

pytestmark = pytest.mark.gpu
kq = pytest.importorskip("dequant_quant_gemv_b200.kq")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


SHAPES = [("q4_k", 1, 4096), ("q4_k", 2, 4096), ("q4_k", 17, 4096), ("q4_k", 64, 32768), ("q4_k", 100, 2048),
          ("q4_k", 5, 768), ("q6_k", 3, 14336), ("q6_k", 64, 28672), ("q6_k", 9, 2048), ("q5_k", 17, 4096),
          ("q5_k", 3, 14336), ("q2_k", 17, 4096), ("q2_k", 3, 14336), ("q3_k", 17, 4096), ("q3_k", 3, 14336),
          ("q8_0", 17, 4096), ("q8_0", 3, 14336), ("q8_0", 5, 768)]


@pytest.mark.parametrize("fmt,N,K", SHAPES)
def test_splitk_parity(fmt, N, K):
    W = matrix(fmt, 900 + N, N, K)
    x = x_vec(901 + K, K)
    Wt, xt = dev(W), dev(x)
    # Q6_K ranges are multiples of 8 blocks, so K = 2048 cannot split (as
    # are Q3_K's; Q2_K's are multiples of 4)
    splits = kq.splitk_workspace_bytes(fmt, N, K, 1) > 0
    assert splits or (fmt == "q6_k" and K // 256 < 16)
    y = kq.gemv_splitk(Wt, fmt, N, K, xt)
    y_ref, s_ref = oracle_gemv(fmt, W, N, K, x)
    assert_close(y[0], y_ref, s_ref, f"splitk {fmt} {N}x{K}")
    y2 = kq.gemv_splitk(Wt, fmt, N, K, xt)
    assert torch.equal(y, y2)


@pytest.mark.parametrize("k", [2, 3, 8])
def test_splitk_multi_columns_independent(k):
    fmt, N, K = "q4_k", 40, 8192
    W = matrix(fmt, 950, N, K)
    X = np.stack([x_vec(960 + c, K) for c in range(8)])
    Wt, Xt = dev(W), dev(X)
    Y8 = kq.gemv_splitk(Wt, fmt, N, K, Xt)
    Y = kq.gemv_splitk(Wt, fmt, N, K, Xt[:k].contiguous())
    assert torch.equal(Y, Y8[:k])
    y_ref, s_ref = oracle.gemv_multi(fmt, W, N, K, X[:k], nthreads=0)
    for c in range(k):
        assert_close(Y[c], y_ref[c], s_ref[c])


def test_splitk_wide_matrix_is_plain_gemv():
    fmt, N, K = "q4_k", 1000, 4096
    assert kq.splitk_workspace_bytes(fmt, N, K, 1) == 0
    W, x = dev(matrix(fmt, 970, N, K)), dev(x_vec(971, K))
    assert torch.equal(kq.gemv_splitk(W, fmt, N, K, x)[0], kq.gemv(W, fmt, N, K, x))


def test_splitk_rejects_small_workspace():
    fmt, N, K = "q4_k", 8, 4096
    need = kq.splitk_workspace_bytes(fmt, N, K, 1)
    assert need > 0
    ws = torch.empty(need // 4 - 1, dtype=torch.float32, device="cuda")
    with pytest.raises(kq.KQError) as e:
        kq.gemv_splitk(dev(matrix(fmt, 980, N, K)), fmt, N, K, dev(x_vec(981, K)), workspace=ws)
    assert e.value.status == 1
