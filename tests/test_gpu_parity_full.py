"""Full-size and exact parity of the GEMV kernels against the CPU oracle.

* The launches the benchmark times, at their real sizes and with every
  output checked: the 8B-shaped gate|up (28672 x 4096, Q4_K) and down
  (4096 x 14336, Q6_K), and the 70B-shaped qkv, o, k/v, gate|up and down
  matrices ("Kortex: Streaming 70B Models on Consumer GPUs", the tables:
  Llama-3.1-8B and Llama-3.3-70B Q4_K_M decode), through plain kq_gemv (no
  prologue, the instantiation the chain runs).
* A streamed chain of 70B-shaped layers at the real slot size, equal bit for
  bit to the same matrices resident ("Out-of-core LLM inference engine
  written from scratch in Rust", Results: streamed execution matches fully
  resident execution).
* Every position of two super-blocks of every format, through the GEMV units
  themselves (not the debug unpacker): weights with d = 1 and small integer
  scales, x one-hot with value 1, so each output is a dequantised weight,
  an exactly representable integer, and must equal the oracle's
  dequantised column exactly, for one column and for eight.
* Activations with outliers (a few channels a thousand times larger; groups
  of one large value among 31 small ones), for one column and for eight.

Tolerance: |y - y_ref| <= 1e-3 * sum_i |w_i x_i| + 1e-6 per output.
"""
import numpy as np
import pytest
import torch

import kqgen
import oracle
from kqtest import assert_close, dev, matrix, oracle_gemv, x_vec

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("dequant_quant_gemv_b200.kq")

ONE = 0x3C00  # fp16 1.0


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


# --------------------------------------------- full-size, every output
FULL = [
    ("q4_k", 28672, 4096, "8B gate|up"),
    ("q6_k", 4096, 14336, "8B down"),
    ("q4_k", 6144, 4096, "8B qkv"),
    ("q4_k", 4096, 4096, "8B o"),
    ("q4_k", 10240, 8192, "70B qkv"),
    ("q4_k", 8192, 8192, "70B o"),
    ("q4_k", 1024, 8192, "70B k / v"),
    ("q4_k", 57344, 8192, "70B gate|up"),
    ("q6_k", 8192, 28672, "70B down"),
]


@pytest.mark.parametrize("fmt,N,K,what", FULL)
def test_plain_gemv_full_size_every_output(fmt, N, K, what):
    W = matrix(fmt, 0xF011 + N + K, N, K)
    x = x_vec(0xF012 + N + K, K)
    y = kq.gemv(dev(W), fmt, N, K, dev(x))
    y_ref, s_ref = oracle_gemv(fmt, W, N, K, x)
    assert_close(y, y_ref, s_ref, f"{what} {N}x{K}")
    assert kq.device_fault() == 0


def test_streamed_70b_layers_equal_resident_bitwise():
    """Two 70B-shaped layers (qkv, o, gate|up, down: 541.9 MB each) in pinned
    host memory, streamed through two device slots of the real size, equal
    the same launches on resident copies bit for bit; gate|up of layer 1 is
    also checked against the oracle."""
    layer = [("q4_k", 10240, 8192), ("q4_k", 8192, 8192), ("q4_k", 57344, 8192), ("q6_k", 8192, 28672)]
    n_layers = 2
    mats, hosts, xs, ys = [], [], [], []
    for li in range(n_layers):
        row = []
        for mi, (fmt, N, K) in enumerate(layer):
            h = torch.empty(N * kqgen.row_bytes(fmt, K), dtype=torch.uint8, pin_memory=True)
            kqgen.matrix(fmt, kqgen.tensor_seed(0x70B, li, mi), N, K, out=h.numpy())
            hosts.append(h)
            row.append((h, fmt, N, K))
            xs.append(dev(x_vec(kqgen.tensor_seed(0x70C, li, mi), K)))
            ys.append(torch.full((N,), float("nan"), device="cuda"))
        mats.append(row)
    ch = kq.Chain(mats, n_slots=2)
    assert ch.slot_bytes >= sum(N * kqgen.row_bytes(f, K) for f, N, K in layer)
    ch.run(xs, ys)
    ch.wait(60000)
    ch.close()
    i = 0
    for li in range(n_layers):
        for h, fmt, N, K in mats[li]:
            y_res = kq.gemv(h.cuda(), fmt, N, K, xs[i])
            assert torch.equal(ys[i], y_res), (li, fmt, N, K)
            i += 1
    fmt, N, K = layer[2]
    y_ref, s_ref = oracle_gemv(fmt, hosts[len(layer) + 2].numpy(), N, K, xs[len(layer) + 2].cpu().numpy())
    assert_close(ys[len(layer) + 2], y_ref, s_ref, "streamed 70B gate|up")


def test_stream_chain_entry_points():
    """kq_stream_chain_create / kq_stream_chain / kq_stream_chain_destroy: a
    waited-for pass over three 8B-shaped layers in two slots equals resident
    launches bitwise, and one output matches the oracle."""
    layer = [("q4_k", 6144, 4096), ("q4_k", 4096, 4096), ("q4_k", 28672, 4096), ("q6_k", 4096, 14336)]
    mats, xs, ys = [], [], []
    for li in range(3):
        row = []
        for mi, (fmt, N, K) in enumerate(layer):
            h = torch.empty(N * kqgen.row_bytes(fmt, K), dtype=torch.uint8, pin_memory=True)
            kqgen.matrix(fmt, kqgen.tensor_seed(0x8B, li, mi), N, K, out=h.numpy())
            row.append((h, fmt, N, K))
            xs.append(dev(x_vec(kqgen.tensor_seed(0x8C, li, mi), K)))
            ys.append(torch.full((N,), float("nan"), device="cuda"))
        mats.append(row)
    sc = kq.StreamChain(mats, n_slots=2)
    sc.run_wait(xs, ys, timeout_ms=60000)
    sc.close()
    i = 0
    for li in range(3):
        for h, fmt, N, K in mats[li]:
            assert torch.equal(ys[i], kq.gemv(h.cuda(), fmt, N, K, xs[i])), (li, fmt)
            i += 1
    h, fmt, N, K = mats[2][3]
    y_ref, s_ref = oracle_gemv(fmt, h.numpy(), N, K, xs[11].cpu().numpy())
    assert_close(ys[11], y_ref, s_ref, "stream chain down")


# ------------------------------------------------ exact one-hot sweeps
def _exact_blocks(fmt, nb, key, unit_scales):
    """Blocks with d (and dmin) = 1 and small integer scales, so that every
    dequantised weight is an exactly representable integer."""
    if fmt in ("q4_k", "q5_k"):
        lg = getattr(kqgen, fmt[:2] + "k_draw")(key, nb)
        sc = np.ones_like(lg["sc"]) if unit_scales else lg["sc"]
        m = np.zeros_like(lg["m"]) if unit_scales else lg["m"]
        pack = kqgen.q4k_pack if fmt == "q4_k" else kqgen.q5k_pack
        return pack(lg["q"], sc, m, np.full(nb, ONE, np.uint16), np.full(nb, ONE, np.uint16))
    if fmt == "q2_k":
        lg = kqgen.q2k_draw(key, nb)
        sc = np.ones_like(lg["sc"]) if unit_scales else lg["sc"]
        m = np.zeros_like(lg["m"]) if unit_scales else lg["m"]
        return kqgen.q2k_pack(lg["q"], sc, m, np.full(nb, ONE, np.uint16), np.full(nb, ONE, np.uint16))
    if fmt == "q3_k":
        lg = kqgen.q3k_draw(key, nb)
        v = np.full_like(lg["v"], 33) if unit_scales else lg["v"]
        return kqgen.q3k_pack(lg["q"], v, np.full(nb, ONE, np.uint16))
    if fmt == "q6_k":
        lg = kqgen.q6k_draw(key, nb)
        s = np.ones_like(lg["s"]) if unit_scales else lg["s"]
        return kqgen.q6k_pack(lg["q"], s, np.full(nb, ONE, np.uint16))
    lg = kqgen.q80_draw(key, nb)
    return kqgen.q80_pack(lg["q"], np.full_like(lg["d"], ONE))


# K per format: rows must be 16-byte aligned for the bulk copies
SWEEP_K = {"q4_k": 512, "q5_k": 512, "q8_0": 512, "q2_k": 1024, "q3_k": 2048, "q6_k": 2048}


@pytest.mark.parametrize("fmt", ["q4_k", "q5_k", "q6_k", "q2_k", "q3_k", "q8_0"])
@pytest.mark.parametrize("unit_scales", [True, False])
def test_one_hot_sweep_exact(fmt, unit_scales):
    """All 512 positions of the first two super-blocks (one at an even and one
    at an odd block index, the two alignment classes of the 2-byte aligned
    formats), 64 rows: kq_gemv with x = e_i, and kq_gemv_multi with eight
    one-hot columns, must reproduce column i of the oracle's dequantised
    matrix exactly."""
    N, K = 64, SWEEP_K[fmt]
    nb = N * K // 256
    W = _exact_blocks(fmt, nb, 0x0E + (1 if unit_scales else 2) + 17 * K, unit_scales)
    Wd = oracle.dequant(fmt, W, N, K)
    assert np.all(Wd == np.round(Wd)) and np.abs(Wd).max() < 2 ** 20   # exact integers
    Wt = dev(W)
    cols, cols8 = [], []
    for i in range(512):
        x = torch.zeros(K, device="cuda")
        x[i] = 1.0
        cols.append(kq.gemv(Wt, fmt, N, K, x))
    for i0 in range(0, 512, 8):
        X = torch.zeros((8, K), device="cuda")
        for c in range(8):
            X[c, i0 + c] = 1.0
        cols8.append(kq.gemv_multi(Wt, fmt, N, K, X))
    Y1 = torch.stack(cols, 1).double().cpu().numpy()
    Y8 = torch.cat(cols8, 0).t().double().cpu().numpy()
    want = Wd[:, :512]
    bad1 = np.argwhere(Y1 != want)
    assert bad1.size == 0, f"k=1: {len(bad1)} positions differ, first (row, i) {bad1[:4].tolist()}"
    bad8 = np.argwhere(Y8 != want)
    assert bad8.size == 0, f"k=8: {len(bad8)} positions differ, first (row, i) {bad8[:4].tolist()}"


# ------------------------------------------------------------ outliers
def _outlier_inputs(K, seed, k):
    rng = np.random.default_rng(seed)
    X = np.stack([x_vec(seed + c, K) for c in range(k)]).astype(np.float32)
    for c in range(k):
        # a few channels a thousand times larger than the rest
        idx = rng.choice(K, size=6, replace=False)
        X[c, idx] *= 1000.0
        # groups of 32 holding one large value among 31 small ones
        for g in rng.choice(K // 32, size=8, replace=False):
            X[c, 32 * g:32 * g + 32] *= 1e-2
            X[c, 32 * g + int(rng.integers(32))] = np.float32(rng.choice([-1, 1]) * rng.uniform(50, 2000))
    return X


@pytest.mark.parametrize("fmt,N,K", [("q4_k", 512, 4096), ("q6_k", 256, 14336), ("q5_k", 512, 4096),
                                     ("q2_k", 512, 4096), ("q3_k", 512, 4096), ("q8_0", 512, 4096),
                                     ("q4_k", 300, 8192), ("q6_k", 96, 28672)])
@pytest.mark.parametrize("k", [1, 8])
def test_outlier_activations(fmt, N, K, k):
    W = matrix(fmt, 0x0A7 + N, N, K)
    X = _outlier_inputs(K, 0x0A8 + K + k, k)
    Wt = dev(W)
    Y = kq.gemv_multi(Wt, fmt, N, K, dev(X))
    y_ref, s_ref = oracle.gemv_multi(fmt, W, N, K, X, nthreads=0)
    for c in range(k):
        assert_close(Y[c], y_ref[c], s_ref[c], f"{fmt} k={k} col {c}")
