"""The GGUF reader (kq_gguf_*): tensor table, sizes and bytes of files
written by a writer of the public GGUF layout (tests/gguf_writer.py), the
ggml-type to libkq-format map, and malformed files rejected.  Host code
only, so these run without a GPU; one GPU test runs a GEMV on a weight read
from a file.  No real model file is in this environment, so interop with a
file written by another program stays unpinned."""
import numpy as np
import pytest

import gguf_writer as gw
import kqgen

kq = pytest.importorskip("dequant_quant_gemv_b200.kq")


def _tensors():
    q4 = kqgen.matrix("q4_k", 2001, 8, 512)
    q6 = kqgen.matrix("q6_k", 2002, 4, 2048)
    q8 = kqgen.matrix("q8_0", 2003, 3, 256)
    f32 = kqgen.normal_f32(2004, 512)
    q40 = np.arange(18 * 4, dtype=np.uint8)              # Q4_0 (type 2): listed, not sized
    return [("blk.0.ffn_up.weight", 12, [512, 8], q4.tobytes()),
            ("blk.0.ffn_down.weight", 14, [2048, 4], q6.tobytes()),
            ("blk.0.attn_q.weight", 8, [256, 3], q8.tobytes()),
            ("output_norm.weight", 0, [512], f32.tobytes()),
            ("legacy.weight", 2, [128], q40.tobytes())]


META = [("general.architecture", gw.STRING, "llama"),
        ("general.name", gw.STRING, "synthetic"),
        ("llama.block_count", gw.U32, 1),
        ("llama.rope.freq_base", gw.F32, 500000.0),
        ("general.flag", gw.BOOL, True),
        ("tokenizer.ggml.tokens", gw.ARRAY, (gw.STRING, ["<s>", "</s>", "a", "bc"])),
        ("tokenizer.ggml.scores", gw.ARRAY, (gw.F32, [0.0, -1.0, -2.5, 3.0])),
        ("nested", gw.ARRAY, (gw.ARRAY, [(gw.U16, [1, 2]), (gw.U16, [3])])),
        ("general.size", gw.U64, 123456789)]


@pytest.mark.parametrize("alignment", [32, 64, 256])
@pytest.mark.parametrize("version", [2, 3])
def test_table_sizes_and_bytes(tmp_path, alignment, version):
    ts = _tensors()
    p = str(tmp_path / "m.gguf")
    gw.write(p, ts, META, alignment=alignment, version=version)
    g = kq.GGUF(p)
    assert len(g) == len(ts)
    sizes = {12: 144 * 2 * 8, 14: 210 * 8 * 4, 8: 34 * 8 * 3, 0: 4 * 512, 2: 0}
    fmts = {12: kq.Q4_K, 14: kq.Q6_K, 8: kq.Q8_0, 0: 0, 2: 0}
    for i, (name, gt, dims, data) in enumerate(ts):
        inf = g.info(i)
        assert inf["name"] == name and inf["type"] == gt and inf["dims"] == dims
        assert inf["nbytes"] == sizes[gt] and inf["fmt"] == fmts[gt]
        assert inf["offset"] % alignment == 0
        assert g.find(name) == i
        if gt != 2:
            assert g.read(name).tobytes() == data
    assert g.find("missing") == -1
    with pytest.raises(kq.KQError) as e:                 # a type the reader does not size
        g.read("legacy.weight")
    assert e.value.status == 2
    g.close()


def test_format_map():
    want = {12: kq.Q4_K, 13: kq.Q5_K, 14: kq.Q6_K, 10: kq.Q2_K, 11: kq.Q3_K, 8: kq.Q8_0, 0: 0, 1: 0, 2: 0, 99: 0}
    for t, f in want.items():
        assert kq.gguf_format(t) == f


@pytest.mark.parametrize("case", ["magic", "version1", "truncated_table", "data_past_end", "misaligned",
                                  "bad_dims", "missing"])
def test_malformed_files_are_rejected(tmp_path, case):
    ts = _tensors()[:2]
    p = str(tmp_path / "bad.gguf")
    if case == "magic":
        gw.write(p, ts, META, magic=b"GGUG")
    elif case == "version1":
        gw.write(p, ts, META, version=1)
    elif case == "truncated_table":
        gw.write(p, [], META)
        with open(p, "r+b") as f:                        # claim one more tensor than the table holds
            f.seek(8)
            f.write((1).to_bytes(8, "little"))
    elif case == "data_past_end":
        gw.write(p, ts, META, truncate=100)
    elif case == "misaligned":
        gw.write(p, ts, META, offsets=[0, 144 * 16 + 8])
    elif case == "bad_dims":
        gw.write(p, [("w", 12, [0, 8], b"")], META)
    else:
        p = str(tmp_path / "none.gguf")
    with pytest.raises(kq.KQError) as e:
        kq.GGUF(p)
    assert e.value.status == 1


@pytest.mark.gpu
def test_gemv_on_a_weight_read_from_the_file(tmp_path):
    import torch

    import oracle
    from kqtest import assert_close, dev, x_vec
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    N, K = 300, 4096
    W = kqgen.matrix("q4_k", 2010, N, K)
    p = str(tmp_path / "w.gguf")
    gw.write(p, [("blk.0.attn_k.weight", 12, [K, N], W.tobytes())], META)
    g = kq.GGUF(p)
    inf = g.info(0)
    Kf, Nf = inf["dims"]
    Wr = g.read(0)
    x = x_vec(2011, Kf)
    y = kq.gemv(dev(Wr), inf["fmt"], Nf, Kf, dev(x))
    y_ref, s_ref = oracle.gemv("q4_k", W, N, K, x, nthreads=0)
    assert_close(y, y_ref, s_ref, "gemv on a GGUF weight")
