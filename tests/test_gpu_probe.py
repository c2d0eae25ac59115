"""kq_read_probe, the read-only bandwidth probe the benchmark divides by:
both modes read every byte of the buffer exactly once (the XOR of what they
read equals the XOR of the buffer's words, computed here on the host)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("dequant_quant_gemv_b200.kq")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


@pytest.mark.parametrize("nbytes", [16, 48 * 1024 * 148 + 16 * 7, 300 << 20])
@pytest.mark.parametrize("mode", [0, 1])
def test_probe_reads_every_word_once(nbytes, mode):
    rng = np.random.default_rng(nbytes + mode)
    host = rng.integers(0, 2 ** 32, nbytes // 4, dtype=np.uint32)
    want = int(np.bitwise_xor.reduce(host)) if host.size else 0
    buf = torch.from_numpy(host.view(np.uint8)).cuda()
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    kq.read_probe(buf, mode, out)
    torch.cuda.synchronize()
    assert int(out.cpu().numpy().view(np.uint32)[0]) == want
    assert kq.device_fault() == 0
