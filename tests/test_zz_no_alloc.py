"""kq_gemv_splitk_noalloc: the split-K GEMV for callers that cannot allocate
device memory -- a real-time or callback thread that must stay out of the
allocator, an engine that owns every byte of device memory through its own
arena, a plugin handed only its inputs and outputs.  Instead of a
caller-provided workspace it keeps its partial sums in a small array built
into the library.

The test drives it through the C ABI on two calls in a row with different
inputs (the built-in array keeps the previous call's contents).  It runs the
same kernels in the same summation order as kq_gemv_splitk fed a workspace
allocated here, so the two outputs must be equal bit for bit; each output is
also checked against the oracle within the parity tolerance.  It lives in
its own file, collected last, and sets up everything it needs, so it passes
alone in a fresh process or after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
from kqtest import ABS, REL, dev, matrix, x_vec

pytestmark = pytest.mark.gpu
kq = pytest.importorskip("dequant_quant_gemv_b200.kq")

# (format, N, K, columns): all tall-skinny, so every call really splits K
CASES = [("q4_k", 17, 4096, 1), ("q6_k", 64, 28672, 1), ("q4_k", 40, 8192, 3), ("q4_k", 3, 32768, 2)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("fmt,N,K,k", CASES)
def test_noalloc_matches_workspace_entry_point_twice(fmt, N, K, k):
    assert kq.splitk_workspace_bytes(fmt, N, K, k) > 0     # the split really happens
    W = matrix(fmt, 4000 + N, N, K)
    Wt = dev(W)
    for call in range(2):                                 # two calls in a row
        X = np.stack([x_vec(4100 + 10 * call + c, K) for c in range(k)])
        Xt = dev(X)
        Y_na = torch.full((k, N), float("nan"), device="cuda")
        kq.gemv_splitk_noalloc(Wt, fmt, N, K, Xt, Y_na)
        ws = torch.empty(kq.splitk_workspace_bytes(fmt, N, K, k) // 4, dtype=torch.float32, device="cuda")
        Y_ws = kq.gemv_splitk(Wt, fmt, N, K, Xt, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(Y_na, Y_ws), (call, float((Y_na - Y_ws).abs().max()))
        y_ref, s = oracle.gemv_multi(fmt, W, N, K, X, nthreads=0)
        err = np.abs(Y_na.double().cpu().numpy() - y_ref)
        assert np.all(err <= REL * s + ABS), (call, float((err / (REL * s + ABS)).max()))
