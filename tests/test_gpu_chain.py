"""GPU tests of the streamed layer chain (kq_chain_*): weights in pinned
host memory stream through a ring of device slots ("Out-of-core LLM
inference engine written from scratch in Rust", Approach; "Kortex: Streaming
70B Models on Consumer GPUs", Key components 2).  The pages' own check that
streamed execution matches fully resident execution becomes a bitwise
comparison with kq_gemv on resident copies of the same weights."""
import os

import numpy as np
import pytest
import torch

import kqgen
from kqtest import assert_close, oracle_gemv

pytestmark = pytest.mark.gpu
kq = pytest.importorskip("dequant_quant_gemv_b200.kq")

SHAPES = [("q4_k", 300, 4096), ("q4_k", 64, 768), ("q6_k", 48, 14336)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def make_layers(n_layers, seed=7):
    layers = []
    for l in range(n_layers):
        mats = []
        for m, (fmt, N, K) in enumerate(SHAPES):
            W = torch.empty(N * kq.row_bytes(fmt, K), dtype=torch.uint8, pin_memory=True)
            kqgen.matrix(fmt, kqgen.tensor_seed(seed, l, m), N, K, out=W.numpy())
            mats.append((W, fmt, N, K))
        layers.append(mats)
    xs = [torch.from_numpy(kqgen.normal_f32(1000 + i, K)).cuda()
          for i, (_, _, _, K) in enumerate(m for layer in layers for m in layer)]
    return layers, xs


@pytest.mark.parametrize("n_slots", [1, 2, 4])
def test_streamed_equals_resident_bitwise(n_slots):
    layers, xs = make_layers(7)
    flat = [m for layer in layers for m in layer]
    ys = [torch.full((N,), float("nan"), device="cuda") for (_, _, N, _) in flat]
    ch = kq.Chain(layers, n_slots=n_slots)
    assert ch.slot_bytes >= sum(N * kq.row_bytes(f, K) for (_, f, N, K) in layers[0])
    ch.run(xs, ys)
    ch.wait(60000)
    for i, (W, fmt, N, K) in enumerate(flat):
        y_res = kq.gemv(W.cuda(), fmt, N, K, xs[i])
        assert torch.equal(ys[i], y_res), i
    # and one matrix against the oracle
    W, fmt, N, K = flat[-1]
    y_ref, s_ref = oracle_gemv(fmt, W.numpy(), N, K, xs[-1].cpu().numpy())
    assert_close(ys[-1], y_ref, s_ref)
    # a second run on the same chain gives the same bits
    ys2 = [torch.empty_like(y) for y in ys]
    ch.run(xs, ys2)
    ch.wait(60000)
    assert all(torch.equal(a, b) for a, b in zip(ys, ys2))
    ch.close()


def test_pageable_weights_are_rejected():
    layers, _ = make_layers(2)
    bad = [[(torch.from_numpy(W.numpy().copy()), f, N, K) for (W, f, N, K) in layer] for layer in layers]
    with pytest.raises(kq.KQError) as e:
        kq.Chain(bad, n_slots=2)
    assert e.value.status == 3


def test_injected_copy_fault_drains(monkeypatch):
    layers, xs = make_layers(6)
    flat = [m for layer in layers for m in layer]
    ys = [torch.zeros(N, device="cuda") for (_, _, N, _) in flat]
    monkeypatch.setenv("KQ_FAULT", "copy@3")
    ch = kq.Chain(layers, n_slots=2)
    with pytest.raises(kq.KQError) as e:
        ch.run(xs, ys)
    assert e.value.status == 8
    ch.wait(60000)                      # what was queued completes
    per = len(SHAPES)
    for i, (W, fmt, N, K) in enumerate(flat[: 3 * per]):
        assert torch.equal(ys[i], kq.gemv(W.cuda(), fmt, N, K, xs[i]))
    for i in range(3 * per, len(flat)):
        assert torch.all(ys[i] == 0)    # never computed
    ch.close()


def test_wait_timeout_is_reported_then_completes():
    layers, xs = make_layers(12)
    flat = [m for layer in layers for m in layer]
    ys = [torch.empty(N, device="cuda") for (_, _, N, _) in flat]
    ch = kq.Chain(layers, n_slots=2)
    torch.cuda.synchronize()
    ch.run(xs, ys)
    try:
        ch.wait(0)
        finished_early = True
    except kq.KQError as e:
        assert e.status == 6
        finished_early = False
    ch.wait(60000)
    ch.close()
    assert finished_early in (True, False)


@pytest.mark.parametrize("n_resident,n_slots", [(2, 1), (5, 2), (7, 1), (0, 3)])
def test_resident_prefix_then_stream_equals_resident_bitwise(n_resident, n_slots):
    """The first n_resident layers stay in device memory, the rest stream
    ("Kortex: Streaming 70B Models on Consumer GPUs", Key components): the
    outputs equal resident kq_gemv calls bit for bit, on two runs."""
    layers, xs = make_layers(7, seed=11)
    flat = [m for layer in layers for m in layer]
    ch = kq.Chain(layers, n_slots=n_slots, n_resident=n_resident)
    assert ch.resident_layers == n_resident
    for _ in range(2):
        ys = [torch.full((N,), float("nan"), device="cuda") for (_, _, N, _) in flat]
        ch.run(xs, ys)
        ch.wait(60000)
        for i, (W, fmt, N, K) in enumerate(flat):
            assert torch.equal(ys[i], kq.gemv(W.cuda(), fmt, N, K, xs[i])), i


def test_resident_counts_are_checked():
    layers, _ = make_layers(3, seed=12)
    with pytest.raises(kq.KQError):
        kq.Chain(layers, n_slots=0, n_resident=1)      # streamed layers need a slot
    with pytest.raises(kq.KQError):
        kq.Chain(layers, n_slots=1, n_resident=4)      # more than the layers
    ch = kq.Chain(layers, n_slots=0, n_resident=3)     # everything resident: no ring
    assert ch.resident_layers == 3
