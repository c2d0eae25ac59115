"""Streamed MoE (kq_moe_stream_*): routed experts copied from pinned host
memory on demand.  Every run must equal, bitwise, the routed GEMV over the
same experts resident in device memory (kq_moe_gemv), which the MoE parity
tests pin to the oracle; one run is also compared with the oracle directly.
Runs in flight share the slot sets in turn (n_sets), so several runs are
enqueued before any is waited for."""
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


def pinned(a: np.ndarray) -> torch.Tensor:
    t = torch.empty(a.nbytes, dtype=torch.uint8, pin_memory=True)
    t.numpy()[:] = a
    return t


@pytest.mark.parametrize("fmt,E,N,K,per_id", [
    ("q4_k", 16, 1536, 2048, False),   # MoE gate|up shape, shared x
    ("q4_k", 16, 2048, 768, True),     # down shape, one x per routed id
    ("q6_k", 6, 130, 2048, True),
    ("q8_0", 12, 256, 1024, False),
])
@pytest.mark.parametrize("n_sets", [1, 2, 3])
def test_runs_equal_resident_routed_gemv_bitwise(fmt, E, N, K, per_id, n_sets):
    W = matrix(fmt, 1300 + E, E * N, K)
    Wh, Wd = pinned(W), dev(W)
    top = min(8, E)
    ms = kq.MoEStream(Wh, fmt, E, N, K, max_ids=top, n_sets=n_sets)
    runs = []
    for r in range(5):                  # all enqueued before any wait
        ids = kqgen.topk_ids(1310 + r, E, top)
        X = dev(np.stack([x_vec(1320 + 10 * r + i, K) for i in range(top)]) if per_id else x_vec(1320 + r, K))
        y = ms.run(ids, X, K if per_id else 0)
        runs.append((ids, X, y))
    ms.wait(60000)
    for ids, X, y in runs:
        yr = kq.moe_gemv(Wd, fmt, E, N, K, dev(ids), X)
        assert torch.equal(y, yr)
    ms.close()


def test_one_run_against_oracle():
    fmt, E, N, K = "q4_k", 8, 512, 2048
    W = matrix(fmt, 1400, E * N, K)
    ms = kq.MoEStream(pinned(W), fmt, E, N, K, max_ids=4, n_sets=2)
    ids = np.array([5, 0, 7, 2], np.int32)
    x = x_vec(1401, K)
    y = ms.run(ids, dev(x))
    ms.wait(60000)
    y_ref, s_ref = oracle.moe_gemv(fmt, W, E, N, K, ids, x, nthreads=0)
    for i in range(4):
        assert_close(y[i], y_ref[i], s_ref[i], f"id {i}")
    ms.close()


def test_invalid_arguments_enqueue_nothing():
    fmt, E, N, K = "q4_k", 4, 64, 256
    W = matrix(fmt, 1500, E * N, K)
    ms = kq.MoEStream(pinned(W), fmt, E, N, K, max_ids=2, n_sets=1)
    x = dev(x_vec(1501, K))
    y = torch.full((2, N), float("nan"), device="cuda")
    for ids in ([0, 4], [-1, 1], [0, 1, 2]):          # out of range, negative, more than max_ids
        with pytest.raises(kq.KQError) as e:
            ms.run(np.array(ids, np.int32), x, y=y)
        assert e.value.status == 1
    ms.run(np.zeros(0, np.int32), x, y=y)             # n_ids = 0: nothing
    ms.wait(60000)
    assert torch.isnan(y).all()
    ms.close()
    with pytest.raises(kq.KQError) as e:               # weights not page-locked
        kq.MoEStream(torch.from_numpy(W.copy()), fmt, E, N, K, max_ids=2)
    assert e.value.status == 3
    with pytest.raises(kq.KQError) as e:               # stride below one expert
        kq.MoEStream(pinned(W), fmt, E, N, K, max_ids=2, stride=N * kq.row_bytes(fmt, K) - 16)
    assert e.value.status == 1
