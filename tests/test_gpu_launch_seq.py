"""Sequences of single-column launches, as the decode chain issues them.

Every launch programs its successor to start early (programmatic dependent
launch): a CTA of launch i+1 starts on an SM as soon as launch i's CTA
there has finished, streams its weights at once and waits only before it
reads its activations.  So:

* every output is written (outputs start as NaN) and matches the oracle,
  including a last stage of a single row (odd N) and Q6_K rows off the
  16-byte grid;
* back-to-back launches on one stream equal isolated launches bit for bit;
* replays of a CUDA graph of such launches equal the eager results bit for
  bit each time.

Tolerance: |y - y_ref| <= 1e-3 * sum_i |w_i x_i| + 1e-6 per output.
"""
import pytest
import torch

import kqgen
from kqtest import assert_close, dev, matrix, oracle_gemv, x_vec

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("dequant_quant_gemv_b200.kq")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


@pytest.mark.parametrize("fmt,N,K", [("q4_k", 30001, 4096),     # the last stage holds one row
                                     ("q6_k", 4097, 14592),     # rows of 11970 bytes (off the grid)
                                     ("q5_k", 20000, 4096),
                                     ("q8_0", 16384, 4096),
                                     ("q2_k", 24576, 4096),
                                     ("q3_k", 12288, 8192)])
def test_large_launch_every_output_against_oracle(fmt, N, K):
    W = matrix(fmt, 0x9001 + N, N, K)
    x = x_vec(0x9002 + K, K)
    y = torch.full((N,), float("nan"), device="cuda")
    kq.gemv(dev(W), fmt, N, K, dev(x), y)
    torch.cuda.synchronize()
    assert not torch.isnan(y).any()
    y_ref, s_ref = oracle_gemv(fmt, W, N, K, x)
    assert_close(y, y_ref, s_ref, f"{fmt} {N}x{K}")
    assert kq.device_fault() == 0


SEQ = [("q4_k", 6144, 4096), ("q4_k", 4096, 4096), ("q4_k", 28672, 4096), ("q6_k", 4096, 14336)] * 3


def _inputs():
    Ws, xs = [], []
    for i, (fmt, N, K) in enumerate(SEQ):
        Ws.append(dev(matrix(fmt, kqgen.tensor_seed(0x9003, i, 0), N, K)))
        xs.append(dev(x_vec(kqgen.tensor_seed(0x9004, i, 0), K)))
    return Ws, xs


def _isolated(Ws, xs):
    out = []
    for (fmt, N, K), W, x in zip(SEQ, Ws, xs):
        out.append(kq.gemv(W, fmt, N, K, x))
        torch.cuda.synchronize()
    return out


def test_back_to_back_equals_isolated():
    Ws, xs = _inputs()
    ref = _isolated(Ws, xs)
    s = torch.cuda.Stream()
    ys = [torch.full((N,), float("nan"), device="cuda") for (_, N, _) in SEQ]
    torch.cuda.synchronize()
    for rep in range(3):
        for y in ys:
            y.fill_(float("nan"))
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            for (fmt, N, K), W, x, y in zip(SEQ, Ws, xs, ys):
                kq.gemv(W, fmt, N, K, x, y, stream=s)
        torch.cuda.synchronize()
        for i, (y, r) in enumerate(zip(ys, ref)):
            assert torch.equal(y, r), (rep, i, SEQ[i])
    assert kq.device_fault() == 0
    fmt, N, K = SEQ[3]
    y_ref, s_ref = oracle_gemv(fmt, Ws[3].cpu().numpy(), N, K, xs[3].cpu().numpy())
    assert_close(ys[3], y_ref, s_ref, "down after back-to-back launches")


def test_graph_replays_equal_eager():
    Ws, xs = _inputs()
    ref = _isolated(Ws, xs)
    ys = [torch.empty(N, device="cuda") for (_, N, _) in SEQ]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):  # warm-up outside the capture
        for (fmt, N, K), W, x, y in zip(SEQ, Ws, xs, ys):
            kq.gemv(W, fmt, N, K, x, y, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for (fmt, N, K), W, x, y in zip(SEQ, Ws, xs, ys):
            kq.gemv(W, fmt, N, K, x, y, stream=s)
    for rep in range(5):
        for y in ys:
            y.fill_(float("nan"))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        for i, (y, r) in enumerate(zip(ys, ref)):
            assert torch.equal(y, r), (rep, i, SEQ[i])
    del g
    assert kq.device_fault() == 0
