"""GPU parity of the fused K-quant GEMV (kq_gemv, kq_gemv_multi, kq_unpack)
against the CPU oracle, on identical seeded inputs.

Acceptance: integer fields bit-exact; every output within
|y - y_ref| <= 1e-3 * sum_i |w_i x_i| + 1e-6 (the bound stated for the
method's decode GEMV); cross-API equalities bitwise.
"""
import numpy as np
import pytest
import torch

import kqgen
import oracle
from kqtest import ABS, assert_close, dev, matrix, oracle_gemv, x_vec

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("dequant_quant_gemv_b200.kq")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


# ------------------------------------------------------------ bit-exact
@pytest.mark.parametrize("fmt,N,K", [("q4_k", 4096, 4096), ("q6_k", 64, 14336), ("q6_k", 3, 2048),
                                     ("q5_k", 2048, 4096), ("q5_k", 3, 256), ("q2_k", 512, 4096),
                                     ("q2_k", 3, 1024), ("q3_k", 512, 4096), ("q3_k", 3, 2048),
                                     ("q3_k", 1, 256), ("q8_0", 512, 4096), ("q8_0", 3, 256)])
def test_unpack_bit_exact(fmt, N, K):
    W = matrix(fmt, 1000 + N, N, K)
    nb = N * K // 256
    q, sc, d = kq.unpack(dev(W), fmt, nb)
    torch.cuda.synchronize()
    q0, sc0, d0 = oracle.unpack(fmt, W, nb)
    assert np.array_equal(q.cpu().numpy(), q0)
    assert np.array_equal(sc.cpu().numpy(), sc0)
    assert np.array_equal(d.cpu().numpy().view(np.uint32), d0.view(np.uint32))


@pytest.mark.parametrize("fmt,N,K", [("q4_k", 512, 4096), ("q6_k", 64, 14336), ("q5_k", 256, 4096),
                                     ("q2_k", 128, 4096), ("q3_k", 128, 4096), ("q8_0", 128, 4096)])
def test_unpack_separate_arrays_bit_exact(fmt, N, K):
    """kq_unpack (q, sc_or_s, m, d, dmin as separate arrays) against the
    oracle's unpacker, field by field."""
    W = matrix(fmt, 2000 + N, N, K)
    nb = N * K // 256
    q, sc, m, d, dmin = (t.cpu().numpy() for t in kq.unpack_split(dev(W), fmt, nb))
    q0, sc0, d0 = oracle.unpack(fmt, W, nb)
    sc0 = sc0.reshape(nb, 16)
    assert np.array_equal(q.view(np.uint8), q0)
    z8 = np.zeros((nb, 8), np.uint8)
    if fmt in ("q4_k", "q5_k"):
        want_sc, want_m = np.hstack([sc0[:, :8], z8]), np.hstack([sc0[:, 8:], z8])
    elif fmt == "q2_k":
        want_sc, want_m = sc0 & 15, sc0 >> 4
    else:
        want_sc, want_m = sc0, np.zeros_like(sc0)
    assert np.array_equal(sc.reshape(nb, 16), want_sc)
    assert np.array_equal(m.reshape(nb, 16), want_m)
    d0 = d0.reshape(nb, 2)
    assert np.array_equal(d.view(np.uint32), np.ascontiguousarray(d0[:, 0]).view(np.uint32))
    assert np.array_equal(dmin.view(np.uint32), np.ascontiguousarray(d0[:, 1]).view(np.uint32))


# -------------------------------------------------- parity, many shapes
SHAPES = [
    ("q4_k", 1, 256), ("q4_k", 3, 256), ("q4_k", 7, 768), ("q4_k", 33, 2048), ("q4_k", 64, 4096),
    ("q4_k", 257, 4096), ("q4_k", 301, 8192), ("q4_k", 5, 1280), ("q4_k", 9, 32768), ("q4_k", 2, 5120),
    ("q6_k", 1, 2048), ("q6_k", 5, 2048), ("q6_k", 64, 14336), ("q6_k", 37, 28672), ("q6_k", 300, 4096),
    ("q6_k", 11, 16384),
    # the block-parity lane order's layouts: one lone warp per parity (24
    # blocks), warp pairs over part-filled chunks (36), a pair and a lone
    # warp (80), a full lone warp (96), two pairs (128, the largest K)
    ("q6_k", 9, 6144), ("q6_k", 13, 9216), ("q6_k", 7, 20480), ("q6_k", 5, 24576), ("q6_k", 3, 32768),
    ("q5_k", 1, 256), ("q5_k", 7, 768), ("q5_k", 257, 4096), ("q5_k", 301, 8192), ("q5_k", 9, 32768),
    ("q5_k", 5, 1280), ("q5_k", 4096, 4096), ("q5_k", 2, 14336),
    ("q2_k", 1, 1024), ("q2_k", 3, 1024), ("q2_k", 257, 4096), ("q2_k", 301, 8192), ("q2_k", 9, 32768),
    ("q2_k", 5, 3072), ("q2_k", 4096, 4096), ("q2_k", 2, 14336),
    ("q3_k", 1, 2048), ("q3_k", 5, 2048), ("q3_k", 257, 4096), ("q3_k", 301, 8192), ("q3_k", 9, 32768),
    ("q3_k", 37, 6144), ("q3_k", 4096, 4096), ("q3_k", 2, 14336),
    ("q8_0", 1, 256), ("q8_0", 7, 768), ("q8_0", 257, 4096), ("q8_0", 301, 8192), ("q8_0", 9, 32768),
    ("q8_0", 5, 1280), ("q8_0", 4096, 4096), ("q8_0", 2, 14336),
]


@pytest.mark.parametrize("fmt,N,K", SHAPES)
def test_gemv_parity(fmt, N, K):
    W = matrix(fmt, 7 * N + K, N, K)
    x = x_vec(N + 3 * K, K)
    y = kq.gemv(dev(W), fmt, N, K, dev(x))
    y_ref, s_ref = oracle_gemv(fmt, W, N, K, x)
    assert_close(y, y_ref, s_ref, f"{fmt} {N}x{K}")


# Lane layouts whose row pairs do not fill a consumer group's 256 lanes (96,
# 160, 192 or 224 lanes per row pair): the warps past a stage's row pairs
# must stay out of the units and the partial-sum reductions.  Enough rows
# that every CTA takes several stages; no bounded wait may run out.
IDLE_WARP_SHAPES = [("q4_k", 1000, 10240), ("q4_k", 600, 20480), ("q4_k", 500, 24576), ("q4_k", 400, 28672),
                    ("q6_k", 700, 20480), ("q6_k", 500, 24576), ("q5_k", 400, 28672), ("q8_0", 600, 20480),
                    ("q2_k", 500, 20480), ("q3_k", 500, 24576)]


@pytest.mark.parametrize("fmt,N,K", IDLE_WARP_SHAPES)
def test_gemv_idle_warp_layouts(fmt, N, K):
    kq.device_fault()  # read and clear
    W = matrix(fmt, 11 * N + K, N, K)
    x = x_vec(N + 5 * K, K)
    y = kq.gemv(dev(W), fmt, N, K, dev(x))
    y_ref, s_ref = oracle_gemv(fmt, W, N, K, x)
    assert_close(y, y_ref, s_ref, f"{fmt} {N}x{K}")
    assert kq.device_fault() == 0


def test_gemv_single_q4k_4096_full():
    """The 4096 x 4096 Q4_K GEMV, every output against the oracle."""
    N = K = 4096
    W = matrix("q4_k", 0xC0FFEE, N, K)
    x = x_vec(0xC0FFEE + 1, K)
    y = kq.gemv(dev(W), "q4_k", N, K, dev(x))
    y_ref, s_ref = oracle_gemv("q4_k", W, N, K, x)
    worst = assert_close(y, y_ref, s_ref, "cfg 4096x4096")
    assert worst < 0.05   # typical error is far inside the bound


def test_deterministic():
    N, K = 1000, 4096
    Wd = dev(matrix("q4_k", 5, N, K))
    xd = dev(x_vec(6, K))
    a = kq.gemv(Wd, "q4_k", N, K, xd)
    b = kq.gemv(Wd, "q4_k", N, K, xd)
    assert torch.equal(a, b)


# --------------------------------------------------- degenerate cases
def test_q4k_zero_quants_and_zero_mins_give_exact_zero():
    N, K = 70, 4096
    nb = N * K // 256
    lg = kqgen.q4k_draw(21, nb)
    W = kqgen.q4k_pack(np.zeros_like(lg["q"]), lg["sc"], np.zeros_like(lg["m"]), lg["d"], lg["dmin"])
    y = kq.gemv(dev(W), "q4_k", N, K, dev(x_vec(22, K)))
    assert torch.all(y == 0)


def test_q5k_zero_quants_and_zero_mins_give_exact_zero():
    N, K = 70, 4096
    nb = N * K // 256
    lg = kqgen.q5k_draw(121, nb)
    W = kqgen.q5k_pack(np.zeros_like(lg["q"]), lg["sc"], np.zeros_like(lg["m"]), lg["d"], lg["dmin"])
    y = kq.gemv(dev(W), "q5_k", N, K, dev(x_vec(122, K)))
    assert torch.all(y == 0)
    Y = kq.gemv_multi(dev(W), "q5_k", N, K, dev(np.stack([x_vec(123 + c, K) for c in range(3)])))
    assert torch.all(Y == 0)


def test_q5k_zero_quants_closed_form():
    """All-zero Q5_K quants: y = -sum_j dmin*m_j*(sum of x over sub-block j),
    as for Q4_K (the 5th bits all zero too)."""
    N, K = 70, 4096
    nb = N * K // 256
    lg = kqgen.q5k_draw(124, nb)
    W = kqgen.q5k_pack(np.zeros_like(lg["q"]), lg["sc"], lg["m"], lg["d"], lg["dmin"])
    x = x_vec(125, K)
    y = kq.gemv(dev(W), "q5_k", N, K, dev(x))
    X = x.astype(np.float64).reshape(K // 32, 32).sum(axis=1).reshape(K // 256, 8)
    dmin = lg["dmin"].view(np.float16).astype(np.float64).reshape(N, K // 256)
    m = lg["m"].astype(np.float64).reshape(N, K // 256, 8)
    want = -np.einsum("rb,rbj,bj->r", dmin, m, X)
    s = np.einsum("rb,rbj,bj->r", dmin, m, np.abs(x.astype(np.float64)).reshape(K // 32, 32).sum(1).reshape(K // 256, 8))
    assert_close(y, want, s, "q5k zero quants")


def test_q2k_zero_quants_closed_form():
    """All-zero Q2_K quants: y = -sum_g dmin*m_g*(sum of x over 16-weight
    group g); with zero mins as well, y = 0 exactly."""
    N, K = 70, 4096
    nb = N * K // 256
    lg = kqgen.q2k_draw(126, nb)
    W = kqgen.q2k_pack(np.zeros_like(lg["q"]), lg["sc"], lg["m"], lg["d"], lg["dmin"])
    x = x_vec(127, K)
    y = kq.gemv(dev(W), "q2_k", N, K, dev(x))
    X = x.astype(np.float64).reshape(K // 256, 16, 16).sum(axis=2)
    A = np.abs(x.astype(np.float64)).reshape(K // 256, 16, 16).sum(axis=2)
    dmin = lg["dmin"].view(np.float16).astype(np.float64).reshape(N, K // 256)
    m = lg["m"].astype(np.float64).reshape(N, K // 256, 16)
    want = -np.einsum("rb,rbg,bg->r", dmin, m, X)
    assert_close(y, want, np.einsum("rb,rbg,bg->r", dmin, m, A), "q2k zero quants")
    W0 = kqgen.q2k_pack(np.zeros_like(lg["q"]), lg["sc"], np.zeros_like(lg["m"]), lg["d"], lg["dmin"])
    assert torch.all(kq.gemv(dev(W0), "q2_k", N, K, dev(x)) == 0)


def test_q3k_zero_values_and_scales_give_exact_zero():
    """Q3_K quants of value 0 (third bit set, low bits 0), or every scale at
    its offset v = 32, give y = 0 exactly."""
    N, K = 70, 4096
    nb = N * K // 256
    lg = kqgen.q3k_draw(128, nb)
    x = dev(x_vec(129, K))
    W = kqgen.q3k_pack(np.zeros_like(lg["q"]), lg["v"], lg["d"])
    assert torch.all(kq.gemv(dev(W), "q3_k", N, K, x) == 0)
    W = kqgen.q3k_pack(lg["q"], np.full_like(lg["v"], 32), lg["d"])
    assert torch.all(kq.gemv(dev(W), "q3_k", N, K, x) == 0)


def test_q80_zero_quants_or_scales_give_exact_zero():
    """Q8_0 with every quant 0, or every block scale 0, gives y = 0 exactly."""
    N, K = 70, 4096
    nu = N * K // 256
    lg = kqgen.q80_draw(130, nu)
    x = dev(x_vec(131, K))
    W = kqgen.q80_pack(np.zeros_like(lg["q"]), lg["d"])
    assert torch.all(kq.gemv(dev(W), "q8_0", N, K, x) == 0)
    W = kqgen.q80_pack(lg["q"], np.zeros_like(lg["d"]))
    assert torch.all(kq.gemv(dev(W), "q8_0", N, K, x) == 0)


def test_q4k_zero_quants_closed_form():
    N, K = 70, 4096
    nb = N * K // 256
    lg = kqgen.q4k_draw(23, nb)
    W = kqgen.q4k_pack(np.zeros_like(lg["q"]), lg["sc"], lg["m"], lg["d"], lg["dmin"])
    x = x_vec(24, K)
    y = kq.gemv(dev(W), "q4_k", N, K, dev(x))
    X = x.astype(np.float64).reshape(K // 32, 32).sum(axis=1).reshape(K // 256, 8)
    dmin = lg["dmin"].view(np.float16).astype(np.float64).reshape(N, K // 256)
    m = lg["m"].astype(np.float64).reshape(N, K // 256, 8)
    want = -np.einsum("rb,rbj,bj->r", dmin, m, X)
    s = np.einsum("rb,rbj,bj->r", dmin, m, np.abs(x.astype(np.float64)).reshape(K // 32, 32).sum(1).reshape(K // 256, 8))
    assert_close(y, want, s, "zero quants")


def test_q6k_mid_quants_give_exact_zero():
    N, K = 40, 14336
    nb = N * K // 256
    lg = kqgen.q6k_draw(25, nb)
    W = kqgen.q6k_pack(np.full_like(lg["q"], 32), lg["s"], lg["d"])
    y = kq.gemv(dev(W), "q6_k", N, K, dev(x_vec(26, K)))
    assert torch.all(y == 0)


def test_unit_scales_integer_matvec():
    N, K = 50, 4096
    nb = N * K // 256
    lg = kqgen.q4k_draw(27, nb)
    W = kqgen.q4k_pack(lg["q"], np.ones((nb, 8), np.uint8), np.zeros((nb, 8), np.uint8),
                       np.full(nb, 0x3C00, np.uint16), np.zeros(nb, np.uint16))
    x = x_vec(28, K)
    Q = lg["q"].reshape(N, K).astype(np.float64)
    y = kq.gemv(dev(W), "q4_k", N, K, dev(x))
    assert_close(y, Q @ x.astype(np.float64), np.abs(Q) @ np.abs(x.astype(np.float64)), "unit scales")


@pytest.mark.parametrize("fmt,K", [("q4_k", 4096), ("q6_k", 14336), ("q5_k", 4096)])
def test_one_hot_extracts_column(fmt, K):
    N = 16
    W = matrix(fmt, 29, N, K)
    Wd = oracle.dequant(fmt, W, N, K)
    Wt = dev(W)
    for i in (0, 1, 31, 32, 33, 255, 256, K - 1):
        x = np.zeros(K, np.float32)
        x[i] = 1.0
        y = kq.gemv(Wt, fmt, N, K, dev(x)).cpu().numpy().astype(np.float64)
        assert np.all(np.abs(y - Wd[:, i]) <= 1e-6 * np.abs(Wd[:, i]) + ABS), i


def test_linearity():
    N, K = 128, 4096
    Wt = dev(matrix("q4_k", 30, N, K))
    rng = np.random.default_rng(0)
    x1 = rng.integers(-8, 8, K).astype(np.float32)
    x2 = rng.integers(-8, 8, K).astype(np.float32)
    y1 = kq.gemv(Wt, "q4_k", N, K, dev(x1)).double()
    y2 = kq.gemv(Wt, "q4_k", N, K, dev(x2)).double()
    yc = kq.gemv(Wt, "q4_k", N, K, dev(2 * x1 - 3 * x2)).double()
    _, s1 = oracle_gemv("q4_k", matrix("q4_k", 30, N, K), N, K, x1)
    _, s2 = oracle_gemv("q4_k", matrix("q4_k", 30, N, K), N, K, x2)
    bound = torch.from_numpy(2 * (2 * 1e-3 * s1 + 3 * 1e-3 * s2) + 1e-5).cuda()
    assert torch.all((yc - (2 * y1 - 3 * y2)).abs() <= bound)


# ---------------------------------------------------------- multi column
@pytest.mark.parametrize("fmt,N,K", [("q4_k", 300, 4096), ("q6_k", 66, 14336), ("q4_k", 17, 768),
                                     ("q4_k", 4096, 4096), ("q4_k", 33, 14336), ("q6_k", 64, 4096),
                                     ("q6_k", 41, 2048), ("q6_k", 4096, 2048), ("q6_k", 3, 14336),
                                     ("q5_k", 300, 4096), ("q5_k", 33, 14336), ("q5_k", 4096, 4096),
                                     ("q5_k", 17, 768), ("q2_k", 300, 4096), ("q2_k", 33, 14336),
                                     ("q3_k", 300, 4096), ("q3_k", 33, 14336), ("q8_0", 300, 4096),
                                     ("q8_0", 17, 768)])
@pytest.mark.parametrize("k", [2, 3, 4, 5, 8])
def test_multi_columns_independent_and_match_oracle(fmt, N, K, k):
    """Each column of a k-column call equals the same column of an 8-column
    call bitwise (a column's value never depends on the other columns or
    on k) and is within the bound of the oracle."""
    W = matrix(fmt, 31, N, K)
    Wt = dev(W)
    X = np.stack([x_vec(100 + c, K) for c in range(8)])
    Xt = dev(X)
    Y8 = kq.gemv_multi(Wt, fmt, N, K, Xt)
    Y = kq.gemv_multi(Wt, fmt, N, K, Xt[:k].contiguous())
    assert torch.equal(Y, Y8[:k])
    y_ref, s_ref = oracle.gemv_multi(fmt, W, N, K, X[:k], nthreads=0)
    for c in range(k):
        assert_close(Y[c], y_ref[c], s_ref[c], f"col {c}")


# Several columns at the K of the single-column idle-warp layouts (and of
# the larger K-range splits of the tensor-core kernel): every format, 8
# columns, against the oracle; no bounded wait may run out.
@pytest.mark.parametrize("fmt,N,K", [("q4_k", 300, 10240), ("q4_k", 200, 20480), ("q6_k", 300, 20480),
                                     ("q6_k", 200, 24576), ("q5_k", 200, 28672), ("q8_0", 300, 20480),
                                     ("q2_k", 300, 20480), ("q3_k", 200, 24576)])
def test_multi_columns_large_k_match_oracle(fmt, N, K):
    kq.device_fault()  # read and clear
    W = matrix(fmt, 37 + K // 256, N, K)
    X = np.stack([x_vec(200 + c + K, K) for c in range(8)])
    Y = kq.gemv_multi(dev(W), fmt, N, K, dev(X))
    y_ref, s_ref = oracle.gemv_multi(fmt, W, N, K, X, nthreads=0)
    for c in range(8):
        assert_close(Y[c], y_ref[c], s_ref[c], f"{fmt} {N}x{K} col {c}")
    assert kq.device_fault() == 0


@pytest.mark.parametrize("fmt,N,K", [("q4_k", 300, 4096), ("q6_k", 66, 14336), ("q5_k", 300, 4096),
                                     ("q2_k", 300, 4096), ("q3_k", 300, 4096), ("q8_0", 300, 4096)])
def test_single_column_of_multi_call_matches_oracle(fmt, N, K):
    """k = 1 through gemv_multi is the single-column kernel, bitwise."""
    W = matrix(fmt, 32, N, K)
    Wt = dev(W)
    x = x_vec(150, K)
    xt = dev(x)
    Y = kq.gemv_multi(Wt, fmt, N, K, xt[None, :].contiguous())
    assert torch.equal(Y[0], kq.gemv(Wt, fmt, N, K, xt))
    y_ref, s_ref = oracle_gemv(fmt, W, N, K, x)
    assert_close(Y[0], y_ref, s_ref)


@pytest.mark.parametrize("fmt", ["q4_k", "q6_k", "q5_k", "q2_k", "q3_k", "q8_0"])
@pytest.mark.parametrize("scale", [1e-30, 1e-6, 1.0, 3e3, 1e20])
def test_multi_column_scale_range(fmt, scale):
    """Activations far from 1 in either direction (the kernel rescales each
    column and super-block by a power of two before splitting it into fp16
    terms); one column of zeros."""
    N, K, k = 48, 4096, 3
    W = matrix(fmt, 33, N, K)
    X = np.stack([x_vec(160 + c, K) for c in range(k)]) * np.float32(scale)
    X[1] = 0.0
    X = X.astype(np.float32)
    Y = kq.gemv_multi(dev(W), fmt, N, K, dev(X))
    y_ref, s_ref = oracle.gemv_multi(fmt, W, N, K, X, nthreads=0)
    for c in range(k):
        assert_close(Y[c], y_ref[c], s_ref[c], f"col {c} scale {scale}")
    assert torch.all(Y[1] == 0)


def test_multi_strided_columns():
    N, K, k = 100, 4096, 4
    W = matrix("q4_k", 40, N, K)
    big = np.zeros((k, K + 64), np.float32)
    for c in range(k):
        big[c, :K] = x_vec(200 + c, K)
    Xt = dev(big)[:, :K]
    Yb = torch.full((k, N + 8), 7.0, device="cuda")
    Y = kq.gemv_multi(dev(W), "q4_k", N, K, Xt, Yb[:, :N])
    assert torch.all(Yb[:, N:] == 7.0)   # padding untouched
    y_ref, s_ref = oracle.gemv_multi("q4_k", W, N, K, big[:, :K], nthreads=0)
    for c in range(k):
        assert_close(Y[c], y_ref[c], s_ref[c])


# ----------------------------------------------------------------- edges
def test_empty_and_degenerate_sizes():
    x = torch.zeros(256, device="cuda")
    y = torch.full((4,), 5.0, device="cuda")
    W = torch.zeros(144 * 4, dtype=torch.uint8, device="cuda")
    kq.gemv(W, "q4_k", 0, 256, x, y)               # N = 0: no-op
    assert torch.all(y == 5.0)
    kq.gemv(W, "q4_k", 4, 0, x, y)                 # K = 0: empty sums
    assert torch.all(y == 0.0)


def test_invalid_arguments_are_rejected():
    W = torch.zeros(144 * 4, dtype=torch.uint8, device="cuda")
    x = torch.zeros(256, device="cuda")
    y = torch.zeros(4, device="cuda")
    with pytest.raises(kq.KQError) as e:
        kq.gemv(W, 9, 4, 256, x, y)
    assert e.value.status == 1
    with pytest.raises(kq.KQError) as e:
        kq.gemv(W, "q4_k", 4, 300, x, y)
    assert e.value.status == 1
    with pytest.raises(kq.KQError) as e:
        kq.gemv(W[1:], "q4_k", 1, 256, x, y)    # misaligned W
    assert e.value.status == 1
    with pytest.raises(kq.KQError):
        kq.gemv_multi(W, "q4_k", 4, 256, torch.zeros((9, 256), device="cuda"))
    assert kq.device_fault() == 0


# ------------------------------------------- single-column integer path
@pytest.mark.parametrize("fmt", ["q4_k", "q5_k", "q2_k", "q3_k", "q6_k", "q8_0"])
def test_single_column_within_activation_rounding_bound(fmt):
    """A single column (every format) rounds each activation to a 14-bit integer
    on a power-of-two grid per group of 32, so |x - x'| <= 2^-14 * (largest
    |x| of the group).  The error must stay within that bound (plus fp32
    rounding slack), computed from the oracle's dequantised weights."""
    N, K = 256, 4096
    W = matrix(fmt, 77, N, K)
    x = x_vec(78, K)
    y = kq.gemv(dev(W), fmt, N, K, dev(x)).cpu().numpy().astype(np.float64)
    Wd = oracle.dequant(fmt, W, N, K).reshape(N, K)
    xd = x.astype(np.float64)
    err = np.abs(y - Wd @ xd)
    gmax = np.abs(xd).reshape(-1, 32).max(axis=1)
    bound = 2.0 ** -14 * (np.abs(Wd).reshape(N, -1, 32).sum(axis=2) * gmax[None, :]).sum(axis=1)
    slack = 1e-5 * (np.abs(Wd) @ np.abs(xd)) + 1e-6
    assert np.all(err <= bound + slack), float(np.max(err / (bound + slack)))


@pytest.mark.parametrize("fmt", ["q4_k", "q6_k", "q5_k", "q2_k", "q3_k", "q8_0"])
@pytest.mark.parametrize("scale", [1e-30, 1e-6, 3e3, 1e20])
def test_single_column_scale_range(fmt, scale):
    """Single column with activations far from 1: the integer path scales
    each group of 32 by its own power of two."""
    N, K = 96, 4096
    W = matrix(fmt, 79, N, K)
    x = (x_vec(80, K) * np.float32(scale)).astype(np.float32)
    x[:64] = 0.0                                   # two all-zero groups
    y = kq.gemv(dev(W), fmt, N, K, dev(x))
    y_ref, s_ref = oracle_gemv(fmt, W, N, K, x)
    assert_close(y, y_ref, s_ref, f"scale {scale}")


# ------------------------------------------- rows off the 16-byte grid
# Real K-quant files have hidden sizes such as 2560, 3584 or 5120 with Q6_K
# tensors ("RunNburn - Run a 295B MoE from a 98GB GGUF ...": native Q2_K-Q6_K
# kernels on the files as they are), whose rows are not multiples of 16
# bytes (or even of 4 bytes when K/256 is odd).
UNALIGNED = [("q6_k", 37, 2560), ("q6_k", 301, 3584), ("q6_k", 64, 5120), ("q6_k", 33, 2304),
             ("q6_k", 257, 6400), ("q6_k", 130, 6656), ("q6_k", 3, 256), ("q6_k", 4096, 5120),
             ("q3_k", 37, 2304), ("q3_k", 300, 256), ("q3_k", 65, 3328), ("q3_k", 2048, 2304),
             ("q2_k", 37, 768), ("q2_k", 301, 2304), ("q2_k", 5, 256), ("q2_k", 2048, 5376)]


@pytest.mark.parametrize("fmt,N,K", UNALIGNED)
@pytest.mark.parametrize("k", [1, 8])
def test_rows_off_the_16_byte_grid(fmt, N, K, k):
    W = matrix(fmt, 0xA11 + N + K, N, K)
    X = np.stack([x_vec(0xA12 + K + c, K) for c in range(k)])
    Wt = dev(W)
    Y = kq.gemv_multi(Wt, fmt, N, K, dev(X))
    y_ref, s_ref = oracle.gemv_multi(fmt, W, N, K, X, nthreads=0)
    for c in range(k):
        assert_close(Y[c], y_ref[c], s_ref[c], f"{fmt} {N}x{K} col {c}")
    if k == 1:
        assert torch.equal(Y[0], kq.gemv(Wt, fmt, N, K, dev(X[0])))


@pytest.mark.parametrize("fmt,K", [("q6_k", 2304), ("q3_k", 2304), ("q2_k", 768), ("q6_k", 6656)])
def test_rows_off_the_grid_moe_and_steps(fmt, K):
    """Routed experts and the multi-step launch on such rows equal kq_gemv
    bit for bit (experts 16-byte aligned, their rows not)."""
    N, E = 96, 5
    rb = kq.row_bytes(fmt, K)
    stride = (N * rb + 15) // 16 * 16
    Wall = np.zeros(E * stride, np.uint8)
    for e in range(E):
        Wall[e * stride:e * stride + N * rb] = matrix(fmt, 0xB00 + e, N, K)
    Wt = dev(Wall)
    x = dev(x_vec(0xB10, K))
    ids = torch.tensor([3, 0, 4], dtype=torch.int32, device="cuda")
    Y = kq.moe_gemv(Wt, fmt, E, N, K, ids, x, expert_stride=stride)
    for i, e in enumerate([3, 0, 4]):
        ref = kq.gemv(Wt[e * stride:], fmt, N, K, x)
        assert torch.equal(Y[i], ref), (fmt, e)
    ys = [torch.full((N,), float("nan"), device="cuda") for _ in range(2)]
    kq.gemv_steps([kq.make_step(Wt[e * stride:], fmt, N, K, x, ys[j]) for j, e in enumerate([1, 2])])
    for j, e in enumerate([1, 2]):
        assert torch.equal(ys[j], kq.gemv(Wt[e * stride:], fmt, N, K, x))
