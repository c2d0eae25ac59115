"""Pins for the CPU oracle: checks against values fixed by something other
than the oracle itself — hand-worked blocks, library routines, closed forms,
invariants and exhaustive round trips.

Formats: GGUF K-quants Q4_K and Q5_K (w = d*sc_j*q - dmin*m_j per 32-weight
sub-block, q of 4 or 5 bits), Q6_K (w = d*s_g*(q-32) per 16-weight group),
Q2_K, Q3_K, and the 8-bit Q8_0 (w = d*q per block of 32),
the formats the pages name ("Out-of-core LLM inference engine written from scratch in Rust",
Results: Q4_K_M; "RunNburn - Run a 295B MoE ...": K-quants Q2_K..Q6_K).
"""
import os

import numpy as np
import pytest

import kqgen
import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _read_golden(path):
    rec = {"w": []}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        if key == "w":
            rec["w"].append((int(vals[0]), int(vals[1]), float(vals[2])))
        else:
            rec[key] = vals
    return rec


# ------------------------------------------------------------------ fp16
def test_f16_decode_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_generator_f16_encode_matches_numpy():
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.standard_normal(20000) * 1e-3,
        rng.standard_normal(5000) * 1e-6,           # subnormal range
        rng.standard_normal(5000) * 1e4,
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, 2.0**-24, 2.0**-25, 3 * 2.0**-26,
                  2.0**-14, 2.0**-14 - 2.0**-25, 1.0 + 2.0**-11, 1.0 + 3 * 2.0**-11]),
    ])
    for v in vals:
        want = int(np.array(v, np.float64).astype(np.float16).view(np.uint16))
        assert kqgen.f16_bits(float(v)) == want, v


# ----------------------------------------------------- hand-worked blocks
def test_q4k_hand_worked_block(golden_dir):
    g = _read_golden(os.path.join(golden_dir, "q4k_block_worked.txt"))
    blk = np.array([int(h, 16) for h in g["header"]] + list(range(128)), np.uint8)
    assert blk.size == 144
    q, sc, d = oracle.unpack("q4_k", blk, 1)
    assert sc[:8].tolist() == [int(v) for v in g["sc"]]
    assert sc[8:].tolist() == [int(v) for v in g["m"]]
    assert d.tolist() == [1.0, 0.5]
    w = oracle.dequant("q4_k", blk, 1, 256)[0]
    for i, qi, wi in g["w"]:
        assert q[i] == qi, i
        assert w[i] == wi, i
    y, _ = oracle.gemv("q4_k", blk, 1, 256, np.ones(256, np.float32))
    assert y[0] == float(g["y_ones"][0])


def test_q6k_hand_worked_block(golden_dir):
    g = _read_golden(os.path.join(golden_dir, "q6k_block_worked.txt"))
    s = np.array([int(v) for v in g["s"]], np.int8)
    blk = np.concatenate([np.arange(128, dtype=np.uint8),
                          np.full(64, int(g["qh_fill"][0], 16), np.uint8),
                          s.view(np.uint8),
                          np.array([int(h, 16) for h in g["d"]], np.uint8)])
    assert blk.size == 210
    q, sc, d = oracle.unpack("q6_k", blk, 1)
    assert sc.view(np.int8).tolist() == s.tolist()
    assert d[0] == 1.0
    w = oracle.dequant("q6_k", blk, 1, 256)[0]
    for i, qi, wi in g["w"]:
        assert q[i] == qi, i
        assert w[i] == wi, i


def test_q5k_hand_worked_block(golden_dir):
    g = _read_golden(os.path.join(golden_dir, "q5k_block_worked.txt"))
    qh = np.arange(32, dtype=np.uint8)
    qh[31] = 0xFF
    blk = np.concatenate([np.array([int(h, 16) for h in g["header"]], np.uint8), qh,
                          np.arange(128, dtype=np.uint8)])
    assert blk.size == 176
    q, sc, d = oracle.unpack("q5_k", blk, 1)
    assert sc[:8].tolist() == [int(v) for v in g["sc"]]
    assert sc[8:].tolist() == [int(v) for v in g["m"]]
    assert d.tolist() == [1.0, 0.5]
    w = oracle.dequant("q5_k", blk, 1, 256)[0]
    for i, qi, wi in g["w"]:
        assert q[i] == qi, i
        assert w[i] == wi, i
    y, _ = oracle.gemv("q5_k", blk, 1, 256, np.ones(256, np.float32))
    assert y[0] == float(g["y_ones"][0])


def test_q2k_hand_worked_block(golden_dir):
    g = _read_golden(os.path.join(golden_dir, "q2k_block_worked.txt"))
    scales = np.array([j | ((15 - j) << 4) for j in range(16)], np.uint8)
    blk = np.concatenate([scales, np.arange(64, dtype=np.uint8), np.array([int(h, 16) for h in g["d"]], np.uint8),
                          np.array([int(h, 16) for h in g["dmin"]], np.uint8)])
    assert blk.size == 84
    q, sc, d = oracle.unpack("q2_k", blk, 1)
    assert (sc & 15).tolist() == list(range(16)) and (sc >> 4).tolist() == [15 - j for j in range(16)]
    assert d.tolist() == [1.0, 0.5]
    w = oracle.dequant("q2_k", blk, 1, 256)[0]
    for i, qi, wi in g["w"]:
        assert q[i] == qi, i
        assert w[i] == wi, i
    y, _ = oracle.gemv("q2_k", blk, 1, 256, np.ones(256, np.float32))
    assert y[0] == float(g["y_ones"][0])


def test_q3k_hand_worked_block(golden_dir):
    g = _read_golden(os.path.join(golden_dir, "q3k_block_worked.txt"))
    blk = np.concatenate([np.arange(32, dtype=np.uint8), np.arange(64, dtype=np.uint8),
                          np.array([int(h, 16) for h in g["scales"]], np.uint8),
                          np.array([int(h, 16) for h in g["d"]], np.uint8)])
    assert blk.size == 110
    q, sc, d = oracle.unpack("q3_k", blk, 1)
    assert sc.tolist() == [int(v) for v in g["v"]]
    assert d.tolist() == [1.0, 0.0]
    w = oracle.dequant("q3_k", blk, 1, 256)[0]
    qs = q.view(np.int8)
    for i, qi, wi in g["w"]:
        assert qs[i] == qi, i
        assert w[i] == wi, i
    y, _ = oracle.gemv("q3_k", blk, 1, 256, np.ones(256, np.float32))
    assert y[0] == float(g["y_ones"][0])


def _q80_golden_unit(g):
    """The worked unit's bytes, from its stated d bytes and quant rules."""
    dbytes = [int(h, 16) for h in g["d"]]
    out = []
    for j in range(8):
        q = [i - 16 for i in range(32)] if j % 2 == 0 else [8 * i - 128 for i in range(31)] + [127]
        out += dbytes[2 * j:2 * j + 2] + [v & 0xFF for v in q]
    return np.array(out, np.uint8)


def test_q80_hand_worked_unit(golden_dir):
    g = _read_golden(os.path.join(golden_dir, "q80_unit_worked.txt"))
    blk = _q80_golden_unit(g)
    assert blk.size == 272
    q, sc, d = oracle.unpack("q8_0", blk, 1)
    assert sc.tolist() == [int(h, 16) for h in g["d"]]   # the raw fp16 scales
    assert d.tolist() == [0.0, 0.0]
    w = oracle.dequant("q8_0", blk, 1, 256)[0]
    qs = q.view(np.int8)
    for i, qi, wi in g["w"]:
        assert qs[i] == qi, i
        assert w[i] == wi, i
    y, _ = oracle.gemv("q8_0", blk, 1, 256, np.ones(256, np.float32))
    assert y[0] == float(g["y_ones"][0])


# ----------------------------------------------- exhaustive round trips
def test_q80_roundtrip_all_values_all_positions():
    """Every int8 value in every quant position, and each block's scale,
    survive generator packing and oracle unpacking."""
    nu = 256
    u, i = np.meshgrid(np.arange(nu), np.arange(256), indexing="ij")
    q = ((i * 7 + u) % 256 - 128).astype(np.int8)
    d = ((np.arange(nu)[:, None] * 8 + np.arange(8)[None, :]) * 37 % 0x7C00).astype(np.uint16)
    W = kqgen.q80_pack(q, d)
    qo, sc, _ = oracle.unpack("q8_0", W, nu)
    assert np.array_equal(qo.view(np.int8).reshape(nu, 256), q)
    assert np.array_equal(sc.reshape(nu, 16).view(np.uint16).reshape(nu, 8), d)
    assert all(len(set(q[:, k].tolist())) == 256 for k in range(256))
    wd = oracle.dequant("q8_0", W, nu, 256)
    want = d.view(np.float16).astype(np.float64).repeat(32, axis=1) * q.astype(np.float64)
    assert np.array_equal(wd, want)


def test_q2k_q3k_roundtrip_all_values_all_positions():
    """Every quant value in every position and every scale (and Q2_K min)
    value in every slot survive generator packing and oracle unpacking."""
    nb = 64
    b, i = np.meshgrid(np.arange(nb), np.arange(256), indexing="ij")
    b16, j16 = np.meshgrid(np.arange(nb), np.arange(16), indexing="ij")
    q2 = ((i * 5 + b) % 4).astype(np.uint8)
    sc2 = ((b16 + 3 * j16) % 16).astype(np.uint8)
    m2 = ((15 - b16 + j16) % 16).astype(np.uint8)
    W2 = kqgen.q2k_pack(q2, sc2, m2, np.full(nb, 0x3C00, np.uint16), np.full(nb, 0x3800, np.uint16))
    q, sc, d = oracle.unpack("q2_k", W2, nb)
    assert np.array_equal(q.reshape(nb, 256), q2)
    assert np.array_equal(sc.reshape(nb, 16) & 15, sc2) and np.array_equal(sc.reshape(nb, 16) >> 4, m2)
    assert all(len(set(q2[:, k].tolist())) == 4 for k in range(256))
    assert all(len(set(sc2[:, k].tolist())) == 16 and len(set(m2[:, k].tolist())) == 16 for k in range(16))
    q3 = ((i * 3 + b) % 8 - 4).astype(np.int8)
    v3 = ((b16 + 5 * j16) % 64).astype(np.uint8)
    W3 = kqgen.q3k_pack(q3, v3, np.full(nb, 0x3C00, np.uint16))
    q, sc, d = oracle.unpack("q3_k", W3, nb)
    assert np.array_equal(q.view(np.int8).reshape(nb, 256), q3)
    assert np.array_equal(sc.reshape(nb, 16), v3)
    assert all(len(set(q3[:, k].tolist())) == 8 for k in range(256))
    assert all(len(set(v3[:, k].tolist())) == 64 for k in range(16))


def test_q5k_quant_and_scale_roundtrip_all_positions():
    """Every 5-bit value in every quant position, and every 6-bit value in
    every scale and min slot, survive generator packing and oracle unpacking."""
    nb = 64
    q = ((np.arange(nb * 256).reshape(nb, 256) * 11 + np.arange(nb)[:, None] * 5) % 32).astype(np.uint8)
    b, j = np.meshgrid(np.arange(nb), np.arange(8), indexing="ij")
    sc = ((b + 5 * j) % 64).astype(np.uint8)
    m = ((63 - b + 3 * j) % 64).astype(np.uint8)
    W = kqgen.q5k_pack(q, sc, m, np.full(nb, 0x3C00, np.uint16), np.full(nb, 0x3800, np.uint16))
    q2, sc2, d2 = oracle.unpack("q5_k", W, nb)
    assert np.array_equal(q2.reshape(nb, 256), q)
    sc2 = sc2.reshape(nb, 16)
    assert np.array_equal(sc2[:, :8], sc) and np.array_equal(sc2[:, 8:], m)
    # each position takes all 32 values across the blocks
    assert all(len(set(q[:, i].tolist())) == 32 for i in range(256))
    assert all(len(set(sc[:, j].tolist())) == 64 and len(set(m[:, j].tolist())) == 64 for j in range(8))


def test_q5k_fifth_bit_alone():
    """Quants 16 everywhere (only the 5th bit set), d=1, sc=1, m=0: y = 16 sum x;
    and quants 15 (no 5th bit) give 15 sum x."""
    K = 512
    nb = 2
    ones = np.ones((nb, 8), np.uint8)
    z = np.zeros((nb, 8), np.uint8)
    x = kqgen.normal_f32(41, K)
    for qv in (16, 15):
        W = kqgen.q5k_pack(np.full((nb, 256), qv, np.uint8), ones, z, np.full(nb, 0x3C00, np.uint16),
                           np.zeros(nb, np.uint16))
        y, _ = oracle.gemv("q5_k", W, 1, K, x)
        assert np.isclose(y[0], qv * x.astype(np.float64).sum(), rtol=1e-13, atol=1e-12)

def test_q4k_scale_min_roundtrip_exhaustive():
    # every 6-bit value in every scale and min slot, others varied
    for v in range(64):
        nb = 8
        q = np.zeros((nb, 256), np.uint8)
        sc = np.zeros((nb, 8), np.uint8)
        m = np.zeros((nb, 8), np.uint8)
        for j in range(8):
            sc[j, j] = v
            m[j, j] = 63 - v
            sc[j, (j + 3) % 8] = (v * 7 + j) % 64
            m[j, (j + 5) % 8] = (v * 11 + j) % 64
        d = np.full(nb, 0x3C00, np.uint16)
        dm = np.full(nb, 0x3800, np.uint16)
        W = kqgen.q4k_pack(q, sc, m, d, dm)
        _, sc2, d2 = oracle.unpack("q4_k", W, nb)
        sc2 = sc2.reshape(nb, 16)
        assert np.array_equal(sc2[:, :8], sc) and np.array_equal(sc2[:, 8:], m)
        assert np.all(d2.reshape(nb, 2) == [1.0, 0.5])


def test_q4k_quant_roundtrip_all_positions():
    nb = 16
    q = (np.arange(nb * 256).reshape(nb, 256) * 7 + np.arange(nb)[:, None]) % 16
    q = q.astype(np.uint8)
    z8 = np.zeros((nb, 8), np.uint8)
    W = kqgen.q4k_pack(q, z8, z8, np.zeros(nb, np.uint16), np.zeros(nb, np.uint16))
    q2, _, _ = oracle.unpack("q4_k", W, nb)
    assert np.array_equal(q2.reshape(nb, 256), q)


def test_q6k_roundtrip_exhaustive():
    nb = 64
    q = ((np.arange(256)[None, :] + 17 * np.arange(nb)[:, None]) % 64).astype(np.uint8)
    s = ((np.arange(16)[None, :] * 16 + np.arange(nb)[:, None]) % 256 - 128).astype(np.int8)
    d = (np.arange(nb) * 977 % 0x7C00).astype(np.uint16)
    W = kqgen.q6k_pack(q, s, d)
    q2, s2, d2 = oracle.unpack("q6_k", W, nb)
    assert np.array_equal(q2.reshape(nb, 256), q)
    assert np.array_equal(s2.view(np.int8).reshape(nb, 16), s)
    want_d = d.view(np.float16).astype(np.float32)
    assert np.array_equal(d2.reshape(nb, 2)[:, 0], want_d)
    # every q value in every position across the 64 blocks
    assert all(len(set(q[:, i].tolist())) == 64 for i in range(256))
    assert len(set(s.ravel().tolist())) == 256


# ---------------------------- special cases that reduce to library routines
@pytest.mark.parametrize("N,K", [(5, 256), (7, 768), (3, 2048)])
def test_q4k_unit_scales_is_integer_matvec(N, K):
    """d=1, sc=1, dmin=0, m=0: W is the integer quant matrix; y = Q @ x."""
    nb = N * K // 256
    lg = kqgen.q4k_draw(101 + K, nb)
    ones = np.ones((nb, 8), np.uint8)
    W = kqgen.q4k_pack(lg["q"], ones, np.zeros((nb, 8), np.uint8),
                       np.full(nb, 0x3C00, np.uint16), np.zeros(nb, np.uint16))
    x = kqgen.normal_f32(5, K)
    Q = lg["q"].reshape(N, K).astype(np.float64)
    y, _ = oracle.gemv("q4_k", W, N, K, x)
    assert np.allclose(y, Q @ x.astype(np.float64), rtol=1e-13, atol=1e-12)


def test_q4k_zero_quants_closed_form():
    """q = 0 everywhere: y_r = -sum_b dmin_b * sum_j m_bj * (sum of x over sub-block j)."""
    N, K = 6, 1024
    nb = N * K // 256
    lg = kqgen.q4k_draw(77, nb)
    W = kqgen.q4k_pack(np.zeros_like(lg["q"]), lg["sc"], lg["m"], lg["d"], lg["dmin"])
    x = kqgen.normal_f32(8, K)
    X = x.astype(np.float64).reshape(K // 32, 32).sum(axis=1).reshape(K // 256, 8)
    dmin = lg["dmin"].view(np.float16).astype(np.float64).reshape(N, K // 256)
    m = lg["m"].astype(np.float64).reshape(N, K // 256, 8)
    want = -np.einsum("rb,rbj,bj->r", dmin, m, X)
    y, _ = oracle.gemv("q4_k", W, N, K, x)
    assert np.allclose(y, want, rtol=1e-12, atol=1e-15)


def test_q4k_zero_scales_gives_exact_zero():
    N, K = 4, 512
    nb = N * K // 256
    lg = kqgen.q4k_draw(78, nb)
    z = np.zeros((nb, 8), np.uint8)
    W = kqgen.q4k_pack(lg["q"], z, z, lg["d"], lg["dmin"])
    y, s = oracle.gemv("q4_k", W, N, K, kqgen.normal_f32(9, K))
    assert np.all(y == 0.0) and np.all(s == 0.0)


def test_q4k_one_hot_reads_subblock_scale():
    """d=1, dmin=0, q=1, sc_j = j+1: x = e_i gives y = (i%256)//32 + 1."""
    K = 512
    sc = np.tile(np.arange(1, 9, dtype=np.uint8), (2, 1))
    W = kqgen.q4k_pack(np.ones((2, 256), np.uint8), sc, np.zeros((2, 8), np.uint8),
                       np.full(2, 0x3C00, np.uint16), np.zeros(2, np.uint16))
    for i in range(K):
        x = np.zeros(K, np.float32)
        x[i] = 1.0
        y, _ = oracle.gemv("q4_k", W, 1, K, x)
        assert y[0] == (i % 256) // 32 + 1


@pytest.mark.parametrize("N,K", [(4, 256), (3, 2048)])
def test_q6k_unit_scale_is_centered_integer_matvec(N, K):
    """d=1, s=1: W = Q - 32; y = (Q - 32) @ x."""
    nb = N * K // 256
    lg = kqgen.q6k_draw(202 + K, nb)
    W = kqgen.q6k_pack(lg["q"], np.ones((nb, 16), np.int8), np.full(nb, 0x3C00, np.uint16))
    x = kqgen.normal_f32(6, K)
    Q = lg["q"].reshape(N, K).astype(np.float64) - 32
    y, _ = oracle.gemv("q6_k", W, N, K, x)
    assert np.allclose(y, Q @ x.astype(np.float64), rtol=1e-13, atol=1e-12)


def test_q6k_mid_quants_give_exact_zero_and_zero_quants_closed_form():
    N, K = 3, 768
    nb = N * K // 256
    lg = kqgen.q6k_draw(303, nb)
    x = kqgen.normal_f32(10, K)
    W32 = kqgen.q6k_pack(np.full_like(lg["q"], 32), lg["s"], lg["d"])
    y, _ = oracle.gemv("q6_k", W32, N, K, x)
    assert np.all(y == 0.0)
    W0 = kqgen.q6k_pack(np.zeros_like(lg["q"]), lg["s"], lg["d"])
    y0, _ = oracle.gemv("q6_k", W0, N, K, x)
    X = x.astype(np.float64).reshape(K // 16, 16).sum(axis=1).reshape(K // 256, 16)
    d = lg["d"].view(np.float16).astype(np.float64).reshape(N, K // 256)
    s = lg["s"].astype(np.float64).reshape(N, K // 256, 16)
    want = -32.0 * np.einsum("rb,rbg,bg->r", d, s, X)
    assert np.allclose(y0, want, rtol=1e-12, atol=1e-15)


# -------------------------------------------------------------- invariants
@pytest.mark.parametrize("fmt", ["q4_k", "q5_k", "q6_k", "q2_k", "q3_k", "q8_0"])
def test_linearity_in_x(fmt):
    N, K = 8, 1024
    W = kqgen.matrix(fmt, 11, N, K)
    rng = np.random.default_rng(3)
    x1 = rng.integers(-50, 50, K).astype(np.float32)
    x2 = rng.integers(-50, 50, K).astype(np.float32)
    xc = (2.0 * x1 - 3.0 * x2).astype(np.float32)   # exact in fp32
    y1, s1 = oracle.gemv(fmt, W, N, K, x1)
    y2, s2 = oracle.gemv(fmt, W, N, K, x2)
    yc, _ = oracle.gemv(fmt, W, N, K, xc)
    assert np.all(np.abs(yc - (2 * y1 - 3 * y2)) <= 1e-12 * (2 * s1 + 3 * s2))


@pytest.mark.parametrize("fmt", ["q4_k", "q5_k", "q6_k", "q2_k", "q3_k", "q8_0"])
def test_one_hot_extracts_column_and_ones_give_row_sums(fmt):
    N, K = 4, 512
    W = kqgen.matrix(fmt, 12, N, K)
    Wd = oracle.dequant(fmt, W, N, K)
    for i in (0, 1, 31, 32, 255, 256, 300, 511):
        x = np.zeros(K, np.float32)
        x[i] = 1.0
        y, _ = oracle.gemv(fmt, W, N, K, x)
        assert np.array_equal(y, Wd[:, i])
    y, s = oracle.gemv(fmt, W, N, K, np.ones(K, np.float32))
    assert np.allclose(y, Wd.sum(axis=1), rtol=1e-13, atol=1e-15)
    assert np.allclose(s, np.abs(Wd).sum(axis=1), rtol=1e-13)


@pytest.mark.parametrize("fmt", ["q4_k", "q5_k", "q6_k", "q2_k", "q3_k", "q8_0"])
def test_brute_force_tiny_from_logical_values(fmt):
    """Dense W built from the generator's logical values (never its bytes)
    matches the oracle's byte path."""
    N, K = 8, 512
    nb = N * K // 256
    if fmt in ("q4_k", "q5_k"):
        lg = kqgen.q4k_draw(31, nb) if fmt == "q4_k" else kqgen.q5k_draw(34, nb)
        W = kqgen.q4k_pack(**lg) if fmt == "q4_k" else kqgen.q5k_pack(**lg)
        d = lg["d"].view(np.float16).astype(np.float64)[:, None]
        dm = lg["dmin"].view(np.float16).astype(np.float64)[:, None]
        sc = np.repeat(lg["sc"].astype(np.float64), 32, axis=1)
        m = np.repeat(lg["m"].astype(np.float64), 32, axis=1)
        dense = (d * sc * lg["q"] - dm * m).reshape(N, K)
    elif fmt == "q2_k":
        lg = kqgen.q2k_draw(35, nb)
        W = kqgen.q2k_pack(**lg)
        d = lg["d"].view(np.float16).astype(np.float64)[:, None]
        dm = lg["dmin"].view(np.float16).astype(np.float64)[:, None]
        sc = np.repeat(lg["sc"].astype(np.float64), 16, axis=1)
        m = np.repeat(lg["m"].astype(np.float64), 16, axis=1)
        dense = (d * sc * lg["q"] - dm * m).reshape(N, K)
    elif fmt == "q3_k":
        lg = kqgen.q3k_draw(36, nb)
        W = kqgen.q3k_pack(**lg)
        d = lg["d"].view(np.float16).astype(np.float64)[:, None]
        v = np.repeat(lg["v"].astype(np.float64) - 32, 16, axis=1)
        dense = (d * v * lg["q"].astype(np.float64)).reshape(N, K)
    elif fmt == "q8_0":
        lg = kqgen.q80_draw(37, nb)
        W = kqgen.q80_pack(**lg)
        d = np.repeat(lg["d"].view(np.float16).astype(np.float64), 32, axis=1)
        dense = (d * lg["q"].astype(np.float64)).reshape(N, K)
    else:
        lg = kqgen.q6k_draw(32, nb)
        W = kqgen.q6k_pack(**lg)
        d = lg["d"].view(np.float16).astype(np.float64)[:, None]
        s = np.repeat(lg["s"].astype(np.float64), 16, axis=1)
        dense = (d * s * (lg["q"].astype(np.float64) - 32)).reshape(N, K)
    x = kqgen.normal_f32(33, K)
    y, _ = oracle.gemv(fmt, W, N, K, x)
    ref = dense @ x.astype(np.float64)
    assert np.all(np.abs(y - ref) <= 1e-12 * np.abs(dense) @ np.abs(x.astype(np.float64)))


def test_multi_moe_forms_are_loops_of_gemv():
    K, N, E = 512, 6, 5
    W = kqgen.matrix("q4_k", 40, E * N, K)
    X = np.stack([kqgen.normal_f32(41 + c, K) for c in range(3)])
    ym, _ = oracle.gemv_multi("q4_k", W[: N * 2 * 144], N, K, X)
    for c in range(3):
        assert np.array_equal(ym[c], oracle.gemv("q4_k", W, N, K, X[c])[0])
    ids = np.array([4, 0, 2], np.int32)
    ye, _ = oracle.moe_gemv("q4_k", W, E, N, K, ids, X)
    stride = N * 2 * 144
    for i, e in enumerate(ids):
        assert np.array_equal(ye[i], oracle.gemv("q4_k", W[e * stride:], N, K, X[i])[0])
    with pytest.raises(ValueError):
        oracle.moe_gemv("q4_k", W, E, N, K, np.array([5]), X[:1])


def test_rows_subset_matches_full():
    N, K = 40, 1024
    W = kqgen.matrix("q6_k", 50, N, K)
    x = kqgen.normal_f32(51, K)
    y, s = oracle.gemv("q6_k", W, N, K, x, nthreads=3)
    rows = np.array([39, 0, 17, 17, 5])
    yr, sr = oracle.gemv_rows("q6_k", W, K, rows, x)
    assert np.array_equal(yr, y[rows]) and np.array_equal(sr, s[rows])


# ------------------------------------------------------------- prologues
def test_rmsnorm_hand_example_and_invariants():
    """[1, -2, 3, 4]: mean square 30/4, so the factor is 1/sqrt(7.5)
    = 0.36514837167011077; with gamma = 1 and eps = 0 the output has mean
    square 1, and scaling x by a power of two changes nothing."""
    x = np.array([1, -2, 3, 4], np.float32)
    out = oracle.rmsnorm(x, np.ones(4, np.float32), 0.0)
    assert np.allclose(out, np.array([1, -2, 3, 4]) * 0.36514837167011077, rtol=0, atol=1e-15)
    rng = np.random.default_rng(5)
    x = rng.standard_normal(4096).astype(np.float32)
    assert abs(np.mean(oracle.rmsnorm(x, np.ones_like(x), 0.0) ** 2) - 1.0) < 1e-12
    assert np.array_equal(oracle.rmsnorm(x * np.float32(8), np.ones_like(x), 0.0),
                          oracle.rmsnorm(x, np.ones_like(x), 0.0))
    g = rng.standard_normal(4096).astype(np.float32)
    assert np.allclose(oracle.rmsnorm(x, g, 0.0), oracle.rmsnorm(x, np.ones_like(x), 0.0) * g, rtol=1e-15)
    # eps = mean square halves the squared factor
    ms = float(np.mean(x.astype(np.float64) ** 2))
    r = oracle.rmsnorm(x, np.ones_like(x), ms) / oracle.rmsnorm(x, np.ones_like(x), 0.0)
    assert np.allclose(r, 1 / np.sqrt(2.0), rtol=1e-12)


def test_swiglu_hand_values_and_identities():
    """silu(0) = 0, silu(1) = 1/(1 + e^-1) = 0.7310585786300049; with up = 1
    the output is silu(gate); silu(-g) = silu(g) - g; up = 0 gives 0."""
    K = 6
    gate = np.array([0, 1, -1, 2, -3, 40], np.float32)
    ones = np.ones(K, np.float32)
    s = oracle.swiglu(np.concatenate([gate, ones]))
    assert s[0] == 0.0 and abs(s[1] - 0.7310585786300049) < 1e-15
    assert abs(s[5] - 40.0) < 1e-12                         # silu(g) -> g for large g
    neg = oracle.swiglu(np.concatenate([-gate, ones]))
    assert np.allclose(neg, s - gate.astype(np.float64), rtol=0, atol=1e-14)
    assert np.all(oracle.swiglu(np.concatenate([gate, np.zeros(K, np.float32)])) == 0)
    up = np.array([2, 3, 5, 7, 11, 13], np.float32)
    assert np.allclose(oracle.swiglu(np.concatenate([gate, up])), s * up, rtol=1e-15)


@pytest.mark.parametrize("fmt", ["q4_k", "q6_k", "q5_k", "q2_k", "q3_k", "q8_0"])
def test_gemv_fused_reduces_to_plain_forms(fmt):
    """The fused oracle with no prologue equals the plain GEMV (float inputs
    widen exactly); with a prologue it is the plain product of the
    prologue's output."""
    N, K = 5, 2048
    W = kqgen.matrix(fmt, 11, N, K)
    rng = np.random.default_rng(6)
    X = rng.standard_normal((2, K)).astype(np.float32)
    y0, s0 = oracle.gemv_fused(fmt, W, N, K, X, "none")
    y1, s1 = oracle.gemv_multi(fmt, W, N, K, X)
    assert np.array_equal(y0, y1) and np.array_equal(s0, s1)
    Wd = oracle.dequant(fmt, W, N, K)
    g = rng.standard_normal(K).astype(np.float32)
    yr, _ = oracle.gemv_fused(fmt, W, N, K, X, "rmsnorm", g, 1e-5)
    assert np.allclose(yr[1], Wd @ oracle.rmsnorm(X[1], g, 1e-5), rtol=1e-12, atol=1e-12)
    GU = rng.standard_normal((1, 2 * K)).astype(np.float32)
    ys, _ = oracle.gemv_fused(fmt, W, N, K, GU, "swiglu")
    assert np.allclose(ys[0], Wd @ oracle.swiglu(GU[0]), rtol=1e-12, atol=1e-12)
