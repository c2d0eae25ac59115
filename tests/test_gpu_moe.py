"""GPU parity of kq_moe_gemv: routed expert ids select which expert
matrices are read ("RunNburn - Run a 295B MoE ...": the selected experts of
each token; "Out-of-core LLM inference engine ...", Results: a resident 30B
MoE).  Output i must equal kq_gemv on expert ids[i] bitwise and the oracle
within tolerance; invalid ids give zeros and a device status, never a trap."""
import numpy as np
import pytest
import torch

import kqgen
import oracle
from kqtest import assert_close, dev, matrix, x_vec

pytestmark = pytest.mark.gpu
kq = pytest.importorskip("dequant_quant_gemv_b200.kq")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("fmt,E,N,K,per_id", [
    ("q4_k", 16, 768, 2048, False),   # gate/up shape, shared x
    ("q4_k", 16, 2048, 768, True),    # down shape, one x per routed id
    ("q6_k", 6, 130, 2048, True),
    ("q4_k", 5, 33, 256, True),       # odd rows per expert
    ("q5_k", 16, 768, 2048, False),
    ("q5_k", 8, 2048, 768, True),
    ("q2_k", 16, 768, 2048, False),
    ("q2_k", 8, 2048, 1024, True),
    ("q3_k", 8, 512, 2048, True),
    ("q3_k", 6, 130, 4096, False),
    ("q8_0", 16, 768, 2048, False),
    ("q8_0", 8, 2048, 768, True),
])
def test_moe_parity(fmt, E, N, K, per_id):
    W = matrix(fmt, 300 + E + N, E * N, K)
    ids = kqgen.topk_ids(17 + N, E, min(8, E))
    n = ids.size
    X = np.stack([x_vec(400 + i, K) for i in range(n)]) if per_id else x_vec(399, K)
    Wt, idt, Xt = dev(W), dev(ids), dev(X)
    y = kq.moe_gemv(Wt, fmt, E, N, K, idt, Xt)
    y_ref, s_ref = oracle.moe_gemv(fmt, W, E, N, K, ids, X, nthreads=0)
    stride = N * kq.row_bytes(fmt, K)
    for i, e in enumerate(ids.tolist()):
        assert_close(y[i], y_ref[i], s_ref[i], f"id {i} -> expert {e}")
        xi = Xt[i] if per_id else Xt
        ye = kq.gemv(Wt[e * stride:(e + 1) * stride], fmt, N, K, xi.contiguous())
        assert torch.equal(y[i], ye), i


def test_moe_invalid_ids_zero_and_flag():
    E, N, K = 4, 64, 2048
    W = matrix("q4_k", 500, E * N, K)
    ids = np.array([3, 4, -1, 0], np.int32)
    x = x_vec(501, K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = kq.moe_gemv(dev(W), "q4_k", E, N, K, dev(ids), dev(x), status=status)
    assert int(status.item()) == 7
    assert torch.all(y[1] == 0) and torch.all(y[2] == 0)
    y_ref, s_ref = oracle.moe_gemv("q4_k", W, E, N, K, ids[[0, 3]], x)
    assert_close(y[0], y_ref[0], s_ref[0])
    assert_close(y[3], y_ref[1], s_ref[1])


def test_moe_repeated_ids():
    E, N, K = 8, 96, 2048
    W = matrix("q4_k", 502, E * N, K)
    ids = np.array([2, 2, 7, 2], np.int32)
    X = np.stack([x_vec(600 + i, K) for i in range(4)])
    y = kq.moe_gemv(dev(W), "q4_k", E, N, K, dev(ids), dev(X))
    y_ref, s_ref = oracle.moe_gemv("q4_k", W, E, N, K, ids, X, nthreads=0)
    for i in range(4):
        assert_close(y[i], y_ref[i], s_ref[i])
