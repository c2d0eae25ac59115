"""GPU parity of kq_gemv_fused: the RMSNorm and SiLU-gated prologues applied
while the activations are staged, against the fp64 oracle of prologue then
GEMV on identical seeded inputs.  The tolerance is the usual
1e-3 * sum|w x'| + 1e-6 over the transformed activations x'.  Shapes cover
the single-column kernels (integer Q4_K, fp32 Q6_K), the tensor-core kernel
(unsplit and cluster-split over K) and ragged N."""
import numpy as np
import pytest
import torch

import oracle
from kqtest import assert_close, dev, matrix, x_vec

pytestmark = pytest.mark.gpu
kq = pytest.importorskip("dequant_quant_gemv_b200.kq")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


SHAPES = [("q4_k", 300, 4096), ("q6_k", 66, 14336), ("q6_k", 130, 2048), ("q4_k", 40, 768), ("q5_k", 200, 4096),
          ("q5_k", 24, 14336), ("q2_k", 200, 4096), ("q2_k", 24, 14336), ("q3_k", 200, 4096), ("q3_k", 24, 14336),
          ("q8_0", 200, 4096), ("q8_0", 24, 14336)]


@pytest.mark.parametrize("fmt,N,K", SHAPES)
@pytest.mark.parametrize("k", [1, 2, 5, 8])
def test_rmsnorm_parity(fmt, N, K, k):
    W = matrix(fmt, 500 + k, N, K)
    X = np.stack([x_vec(510 + c, K) * np.float32(3.0) for c in range(k)])
    g = x_vec(520, K)
    Y = kq.gemv_fused(dev(W), fmt, N, K, dev(X), "rmsnorm", dev(g), 1e-5)
    y_ref, s_ref = oracle.gemv_fused(fmt, W, N, K, X, "rmsnorm", g, 1e-5, nthreads=0)
    for c in range(k):
        assert_close(Y[c], y_ref[c], s_ref[c], f"rmsnorm col {c}")


@pytest.mark.parametrize("fmt,N,K", SHAPES)
@pytest.mark.parametrize("k", [1, 3, 8])
def test_swiglu_parity(fmt, N, K, k):
    W = matrix(fmt, 600 + k, N, K)
    GU = np.stack([x_vec(610 + c, 2 * K) for c in range(k)])
    Y = kq.gemv_fused(dev(W), fmt, N, K, dev(GU), "swiglu")
    y_ref, s_ref = oracle.gemv_fused(fmt, W, N, K, GU, "swiglu", nthreads=0)
    for c in range(k):
        assert_close(Y[c], y_ref[c], s_ref[c], f"swiglu col {c}")


@pytest.mark.parametrize("k", [1, 4])
def test_no_prologue_equals_multi_bitwise(k):
    fmt, N, K = "q4_k", 200, 4096
    W = dev(matrix(fmt, 700, N, K))
    X = dev(np.stack([x_vec(701 + c, K) for c in range(k)]))
    assert torch.equal(kq.gemv_fused(W, fmt, N, K, X, "none"), kq.gemv_multi(W, fmt, N, K, X))


@pytest.mark.parametrize("fmt,K", [("q4_k", 4096), ("q6_k", 2048)])
@pytest.mark.parametrize("k", [1, 4])
def test_exact_zeros(fmt, K, k):
    """SwiGLU with up = 0 and RMSNorm of a zero vector give y = 0 exactly."""
    N = 64
    W = dev(matrix(fmt, 710, N, K))
    GU = np.stack([x_vec(711 + c, 2 * K) for c in range(k)])
    GU[:, K:] = 0.0
    assert torch.all(kq.gemv_fused(W, fmt, N, K, dev(GU), "swiglu") == 0)
    X = torch.zeros((k, K), device="cuda")
    g = dev(x_vec(712, K))
    assert torch.all(kq.gemv_fused(W, fmt, N, K, X, "rmsnorm", g, 1e-5) == 0)


def test_invalid_prologues_are_rejected():
    fmt, N, K = "q4_k", 16, 256
    W = dev(matrix(fmt, 720, N, K))
    x = dev(x_vec(721, K))
    g = dev(x_vec(722, K))
    L = kq.lib()
    y = torch.empty(N, device="cuda")
    for kind, gamma, eps in [(7, g.data_ptr(), 1e-5), (1, None, 1e-5), (1, g.data_ptr(), 0.0),
                             (1, g.data_ptr(), -1.0)]:
        pro = kq.Prologue(kind, gamma, eps)
        st = L.kq_gemv_fused(W.data_ptr(), 1, N, K, x.data_ptr(), K, 1, pro, y.data_ptr(), N, None)
        assert st == 1, (kind, eps)
    # SwiGLU columns must hold 2K floats
    X = torch.zeros((2, K), device="cuda")
    Y = torch.empty((2, N), device="cuda")
    pro = kq.Prologue(2, None, 0.0)
    st = L.kq_gemv_fused(W.data_ptr(), 1, N, K, X.data_ptr(), K, 2, pro, Y.data_ptr(), N, None)
    assert st == 1


@pytest.mark.parametrize("H,F", [(512, 2048), (4096, 14336)])
def test_chained_ffn_each_stage_matches_oracle(H, F):
    """The decode FFN as the fused path runs it: gate|up (2F x H, Q4_K) with
    RMSNorm on x, then down (H x F, Q6_K) reading gate|up's device output
    [g; u] through the SiLU-gated prologue.  Each stage is compared with the
    oracle on that stage's own inputs (down on the device's [g; u])."""
    Wgu = matrix("q4_k", 730, 2 * F, H)
    Wdn = matrix("q6_k", 731, H, F)
    x = x_vec(732, H)
    g = x_vec(733, H) * np.float32(0.1) + np.float32(1.0)
    GU = kq.gemv_fused(dev(Wgu), "q4_k", 2 * F, H, dev(x), "rmsnorm", dev(g), 1e-5)
    Y = kq.gemv_fused(dev(Wdn), "q6_k", H, F, GU, "swiglu")
    gu_host = GU.cpu().numpy()
    gu_ref, gu_s = oracle.gemv_fused("q4_k", Wgu, 2 * F, H, x[None, :], "rmsnorm", g, 1e-5, nthreads=0)
    assert_close(GU[0], gu_ref[0], gu_s[0], "gate|up")
    y_ref, y_s = oracle.gemv_fused("q6_k", Wdn, H, F, gu_host, "swiglu", nthreads=0)
    assert_close(Y[0], y_ref[0], y_s[0], "down")
