"""Failure detection on the device: a bounded wait that runs out.

Every wait of the GEMV kernels (a consumer waiting for a weight stage to
land, the producer waiting for a ring slot to be released) is bounded; when
the limit passes, the kernel records KQ_ERR_TIMEOUT in the device fault word
and stops instead of hanging.  The test hook kq_inject("hold@S") makes the
next single-column launch withhold one weight stage of its first CTA and
shortens the limit to 1 ms, so the consumers waiting for that stage time
out.  No fault, trap or hang is involved: the launch completes, the host
reads the fault word, and the context stays usable (the next launch is
checked against the oracle).
"""
import pytest
import torch

from kqtest import assert_close, dev, matrix, oracle_gemv, x_vec

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("dequant_quant_gemv_b200.kq")

KQ_ERR_TIMEOUT = 6


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()
    kq.device_fault()          # start from a clear fault word
    yield
    kq.inject(None)


@pytest.mark.parametrize("fmt,N,K,hold", [("q4_k", 4096, 4096, 1), ("q4_k", 28672, 4096, 3),
                                          ("q6_k", 4096, 14336, 2), ("q8_0", 2048, 4096, 1)])
def test_withheld_stage_times_out_and_context_survives(fmt, N, K, hold):
    W = matrix(fmt, 0x71 + N, N, K)
    x = x_vec(0x72 + K, K)
    Wt, xt = dev(W), dev(x)
    torch.cuda.synchronize()                     # nothing queued ahead of the launch
    assert kq.device_fault() == 0
    kq.inject(f"hold@{hold}")
    kq.gemv(Wt, fmt, N, K, xt)
    torch.cuda.synchronize()                     # the launch ends: no hang
    assert kq.device_fault() == KQ_ERR_TIMEOUT
    assert kq.device_fault() == 0                # read and cleared
    # the hook was one-shot and the context is intact
    y = kq.gemv(Wt, fmt, N, K, xt)
    torch.cuda.synchronize()
    assert kq.device_fault() == 0
    y_ref, s_ref = oracle_gemv(fmt, W, N, K, x)
    assert_close(y, y_ref, s_ref, f"{fmt} after the timeout")


def test_inject_rejects_unknown_specs():
    with pytest.raises(kq.KQError):
        kq.inject("hold@0")
    with pytest.raises(kq.KQError):
        kq.inject("drop")
    kq.inject(None)
