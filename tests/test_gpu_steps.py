"""kq_gemv_steps: several single-column GEMVs in one persistent launch.

Every step is computed exactly as the single-column kernel computes it, so
the outputs must equal, bit for bit, the same steps run one by one through
kq_gemv_fused (k = 1), which the other GPU tests pin to the oracle.  The
cases mix formats and prologues, chain a step's input to an earlier step's
output (the decode FFN: gate|up with RMSNorm, then down reading gate|up's
[g; u] through the SiLU-gated prologue), run more steps than one launch
takes, and cover the empty cases and rejected arguments.  One chained case
is also compared with the oracle directly.
"""
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


def nan(n):
    return torch.full((n,), float("nan"), device="cuda")


def one_by_one(specs):
    """The same steps through kq_gemv_fused, one call each, in order."""
    ys = []
    for (W, fmt, N, K, x, kind, gamma) in specs:
        y = nan(N)
        kq.gemv_fused(W, fmt, N, K, x() if callable(x) else x, kind, gamma, 1e-5, Y=y[None, :])
        ys.append(y)
    return ys


# (format, N, K, prologue): the 8B layer's shapes, a ragged and a tiny matrix
LAYER = [("q4_k", 6144, 4096, "rmsnorm"), ("q4_k", 4096, 4096, "none"), ("q4_k", 300, 4096, "none"),
         ("q6_k", 4096, 14336, "swiglu"), ("q4_k", 64, 768, "none"), ("q6_k", 48, 14336, "none"),
         ("q4_k", 1, 256, "rmsnorm"), ("q4_k", 2048, 8192, "none"), ("q5_k", 1024, 4096, "rmsnorm"),
         ("q5_k", 96, 14336, "swiglu"), ("q2_k", 1024, 4096, "rmsnorm"), ("q3_k", 96, 14336, "swiglu"),
         ("q2_k", 40, 14336, "none"), ("q3_k", 300, 4096, "none"), ("q8_0", 512, 4096, "rmsnorm"),
         ("q8_0", 64, 14336, "swiglu")]


def build(seed, shapes):
    specs = []
    for i, (fmt, N, K, kind) in enumerate(shapes):
        W = dev(matrix(fmt, seed + i, N, K))
        x = dev(x_vec(seed + 100 + i, 2 * K if kind == "swiglu" else K))
        g = dev(x_vec(seed + 200 + i, K) * np.float32(0.1) + np.float32(1.0)) if kind == "rmsnorm" else None
        specs.append((W, fmt, N, K, x, kind, g))
    return specs


@pytest.mark.parametrize("after", [False, True])
def test_independent_steps_equal_single_calls_bitwise(after):
    specs = build(900, LAYER)
    ys = [nan(N) for (_, _, N, _, _, _, _) in specs]
    kq.gemv_steps([kq.make_step(W, f, N, K, x, y, kind, g, 1e-5, after)
                   for (W, f, N, K, x, kind, g), y in zip(specs, ys)])
    ref = one_by_one(specs)
    for i, (y, r) in enumerate(zip(ys, ref)):
        assert torch.equal(y, r), i


# Q6_K in the block-parity lane order, each of its layouts (24, 36, 80, 96
# and 128 blocks: lone warps, part-filled warp pairs, both, two pairs)
@pytest.mark.parametrize("K", [6144, 9216, 20480, 24576, 32768])
def test_q6k_parity_layouts_steps_equal_single_calls(K):
    specs = build(1300 + K // 256, [("q6_k", 37, K, "none"), ("q6_k", 6, K, "rmsnorm"), ("q6_k", 21, K, "swiglu")])
    ys = [nan(N) for (_, _, N, _, _, _, _) in specs]
    kq.gemv_steps([kq.make_step(W, f, N, K_, x, y, kind, g, 1e-5, True)
                   for (W, f, N, K_, x, kind, g), y in zip(specs, ys)])
    ref = one_by_one(specs)
    for i, (y, r) in enumerate(zip(ys, ref)):
        assert torch.equal(y, r), i


def test_chained_ffn_steps_equal_single_calls_and_oracle():
    """gate|up (RMSNorm) -> down (SiLU-gated [g; u] read from gate|up's
    output), three layers deep, in one call: each down step waits for its
    gate|up step."""
    H, F = 4096, 14336
    Wgu = [dev(matrix("q4_k", 950 + l, 2 * F, H)) for l in range(3)]
    Wdn = [dev(matrix("q6_k", 960 + l, H, F)) for l in range(3)]
    g = dev(x_vec(970, H) * np.float32(0.1) + np.float32(1.0))
    xs = [dev(x_vec(971 + l, H)) for l in range(3)]
    gu = [nan(2 * F) for _ in range(3)]
    out = [nan(H) for _ in range(3)]
    steps = []
    for l in range(3):
        steps.append(kq.make_step(Wgu[l], "q4_k", 2 * F, H, xs[l], gu[l], "rmsnorm", g, 1e-5, after=True))
        steps.append(kq.make_step(Wdn[l], "q6_k", H, F, gu[l], out[l], "swiglu", after=True))
    kq.gemv_steps(steps)
    for l in range(3):
        gu_ref = nan(2 * F)
        kq.gemv_fused(Wgu[l], "q4_k", 2 * F, H, xs[l], "rmsnorm", g, 1e-5, Y=gu_ref[None, :])
        dn_ref = nan(H)
        kq.gemv_fused(Wdn[l], "q6_k", H, F, gu_ref, "swiglu", Y=dn_ref[None, :])
        assert torch.equal(gu[l], gu_ref), l
        assert torch.equal(out[l], dn_ref), l
    # the last down step against the oracle on its own inputs
    y_ref, s_ref = oracle.gemv_fused("q6_k", Wdn[2].cpu().numpy(), H, F, gu[2].cpu().numpy()[None, :], "swiglu",
                                     nthreads=0)
    assert_close(out[2], y_ref[0], s_ref[0], "down after gate|up")


def test_more_steps_than_one_launch_takes():
    shapes = [("q4_k", 512 + 64 * (i % 5), 4096, "none") for i in range(37)]
    specs = build(1000, shapes)
    ys = [nan(N) for (_, _, N, _, _, _, _) in specs]
    kq.gemv_steps([kq.make_step(W, f, N, K, x, y, kind, g) for (W, f, N, K, x, kind, g), y in zip(specs, ys)])
    ref = one_by_one(specs)
    for i, (y, r) in enumerate(zip(ys, ref)):
        assert torch.equal(y, r), i


def test_empty_steps_and_zero_k():
    specs = build(1100, [("q4_k", 300, 4096, "none"), ("q4_k", 128, 2048, "none")])
    ys = [nan(N) for (_, _, N, _, _, _, _) in specs]
    yk0 = nan(77)
    W0 = torch.empty(0, dtype=torch.uint8, device="cuda")
    xk0 = torch.empty(1, device="cuda")
    steps = [kq.make_step(*specs[0][:5], ys[0]),
             kq.make_step(W0, "q4_k", 0, 4096, xk0, nan(1)),     # N = 0: nothing
             kq.make_step(W0, "q6_k", 77, 0, xk0, yk0),          # K = 0: zeros
             kq.make_step(*specs[1][:5], ys[1])]
    kq.gemv_steps(steps)
    kq.gemv_steps([])
    ref = one_by_one(specs)
    assert torch.equal(ys[0], ref[0]) and torch.equal(ys[1], ref[1])
    assert torch.all(yk0 == 0)


def test_invalid_step_launches_nothing():
    specs = build(1200, [("q4_k", 300, 4096, "none"), ("q6_k", 64, 2048, "none")])
    ys = [nan(N) for (_, _, N, _, _, _, _) in specs]
    good = [kq.make_step(*sp[:5], y) for sp, y in zip(specs, ys)]
    L = kq.lib()
    bad_fmt = kq.make_step(*specs[0][:5], ys[0])
    bad_fmt.fmt = 9
    bad_k = kq.make_step(*specs[1][:5], ys[1])
    bad_k.K = 3000                                   # not a multiple of 256
    bad_q6 = kq.make_step(*specs[1][:5], ys[1])
    bad_q6.x = None                                  # NULL activations
    bad_pro = kq.make_step(*specs[0][:5], ys[0], "rmsnorm", specs[0][4], 0.0)  # eps = 0
    for bad in (bad_fmt, bad_k, bad_q6, bad_pro):
        arr = (kq.Step * 3)(good[0], bad, good[1])
        st = L.kq_gemv_steps(arr, 3, None)
        assert st != 0
        assert b"step 1" in L.kq_last_error()
    assert L.kq_gemv_steps(None, 2, None) == 1
    assert L.kq_gemv_steps(None, -1, None) == 1
    torch.cuda.synchronize()
    assert all(torch.isnan(y).all() for y in ys)     # nothing ran
