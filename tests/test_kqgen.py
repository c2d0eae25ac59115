"""The seeded input generator: determinism, the published SplitMix64 stream,
and the value distributions the workloads specify (Q4_K quants uniform
0..15, scales/mins uniform 0..63, d/dmin = |N(0,1)|*1e-3 in fp16, x ~ N(0,1)
fp32; Q6_K quants 0..63, scales -64..63)."""
import numpy as np
import pytest

import kqgen
import oracle


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 1234567: the first outputs of the published
    # generator (state += 0x9E3779B97F4A7C15, then the two xor-shift-multiply
    # rounds), computed here with Python integers.
    def ref(seed, n):
        out, s = [], seed
        for _ in range(n):
            s = (s + 0x9E3779B97F4A7C15) % 2**64
            z = s
            z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) % 2**64
            z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) % 2**64
            out.append(z ^ (z >> 31))
        return out
    assert [kqgen.splitmix64(1234567, i) for i in range(5)] == ref(1234567, 5)
    # known first output for seed 0 of the reference generator
    assert kqgen.splitmix64(0, 0) == 0xE220A8397B1DCDAF


def test_fill_is_thread_count_independent_and_matches_draw_pack():
    nb = 37
    a = kqgen.q4k_fill(99, nb, nthreads=1)
    b = kqgen.q4k_fill(99, nb, nthreads=4)
    assert np.array_equal(a, b)
    assert np.array_equal(a, kqgen.q4k_pack(**kqgen.q4k_draw(99, nb)))
    c = kqgen.q6k_fill(98, nb, nthreads=3)
    assert np.array_equal(c, kqgen.q6k_pack(**kqgen.q6k_draw(98, nb)))
    # offset fill = tail of the full fill
    tail = kqgen.q4k_fill(99, 10, b0=nb - 10, nthreads=2)
    assert np.array_equal(tail, a[(nb - 10) * 144:])


@pytest.mark.parametrize("fmt", ["q5_k", "q2_k", "q3_k", "q8_0"])
def test_fill_matches_draw_pack_other_formats(fmt):
    nb = 29
    draw = {"q5_k": kqgen.q5k_draw, "q2_k": kqgen.q2k_draw, "q3_k": kqgen.q3k_draw, "q8_0": kqgen.q80_draw}[fmt]
    pack = {"q5_k": kqgen.q5k_pack, "q2_k": kqgen.q2k_pack, "q3_k": kqgen.q3k_pack, "q8_0": kqgen.q80_pack}[fmt]
    a = kqgen.fill(fmt, 77, nb, nthreads=1)
    assert np.array_equal(a, kqgen.fill(fmt, 77, nb, nthreads=5))
    assert np.array_equal(a, pack(**draw(77, nb)))
    assert a.size == nb * kqgen.block_bytes(fmt)


def test_other_format_distributions():
    """The fill draws every value of each field's range, uniformly."""
    lg = kqgen.q5k_draw(9, 2000)
    c = np.bincount(lg["q"].ravel(), minlength=32)
    assert c.size == 32 and np.all(np.abs(c / c.mean() - 1) < 0.05)
    lg = kqgen.q2k_draw(10, 2000)
    for f, n in (("q", 4), ("sc", 16), ("m", 16)):
        c = np.bincount(lg[f].ravel(), minlength=n)
        assert c.size == n and np.all(np.abs(c / c.mean() - 1) < 0.1), f
    lg = kqgen.q3k_draw(11, 2000)
    c = np.bincount(lg["q"].astype(int).ravel() + 4, minlength=8)
    assert c.size == 8 and np.all(np.abs(c / c.mean() - 1) < 0.05)
    c = np.bincount(lg["v"].ravel(), minlength=64)
    assert c.size == 64 and np.all(np.abs(c / c.mean() - 1) < 0.2)
    lg = kqgen.q80_draw(12, 2000)
    c = np.bincount(lg["q"].astype(int).ravel() + 128, minlength=256)
    assert c.size == 256 and np.all(np.abs(c / c.mean() - 1) < 0.1)
    d = lg["d"].view(np.float16).astype(np.float64)
    assert np.all(d >= 0) and abs(d.mean() / 1e-3 - np.sqrt(2 / np.pi)) < 0.03


def test_q4k_distributions():
    lg = kqgen.q4k_draw(5, 4000)
    counts = np.bincount(lg["q"].ravel(), minlength=16)
    assert counts.size == 16 and np.all(np.abs(counts / counts.mean() - 1) < 0.02)
    for f in ("sc", "m"):
        c = np.bincount(lg[f].ravel(), minlength=64)
        assert c.size == 64 and np.all(np.abs(c / c.mean() - 1) < 0.2)
    d = lg["d"].view(np.float16).astype(np.float64)
    assert np.all(d >= 0)
    # E|N(0,1)| = sqrt(2/pi)
    assert abs(d.mean() / 1e-3 - np.sqrt(2 / np.pi)) < 0.03


def test_q6k_distributions():
    lg = kqgen.q6k_draw(6, 3000)
    c = np.bincount(lg["q"].ravel(), minlength=64)
    assert c.size == 64 and np.all(np.abs(c / c.mean() - 1) < 0.05)
    s = lg["s"].astype(int).ravel()
    assert s.min() == -64 and s.max() == 63
    assert abs(np.mean(s) + 0.5) < 0.5


def test_normal_and_ids():
    x = kqgen.normal_f32(3, 200001)
    assert x.dtype == np.float32
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    assert np.array_equal(x, kqgen.normal_f32(3, 200001, nthreads=5))
    ids = kqgen.topk_ids(1234, 128, 8)
    assert len(set(ids.tolist())) == 8 and ids.min() >= 0 and ids.max() < 128
    # uniformity of the first pick over many seeds
    first = np.array([kqgen.topk_ids(s, 16, 4)[0] for s in range(8000)])
    c = np.bincount(first, minlength=16)
    assert np.all(np.abs(c / c.mean() - 1) < 0.15)


def test_generated_d_decodes_exactly():
    lg = kqgen.q4k_draw(8, 100)
    W = kqgen.q4k_pack(**lg)
    _, _, d = oracle.unpack("q4_k", W, 100)
    assert np.array_equal(d.reshape(100, 2)[:, 0], lg["d"].view(np.float16).astype(np.float32))
