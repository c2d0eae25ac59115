"""kq_chain_plan on the CPU: how many leading layers stay resident next to
the streaming ring within a device-memory budget ("Kortex: Streaming 70B
Models on Consumer GPUs", Key components: the layers that fit stay in
VRAM, the rest stream).  Host arithmetic only; the layer size is the sum of
each matrix's bytes rounded up to 256, as the chain lays a layer out."""
import pytest

kq = pytest.importorskip("dequant_quant_gemv_b200.kq")

# a 70B-shaped layer: qkv, o, gate|up (Q4_K), down (Q6_K)
L70 = [(None, "q4_k", 10240, 8192), (None, "q4_k", 8192, 8192), (None, "q4_k", 57344, 8192),
       (None, "q6_k", 8192, 28672)]


def layer_bytes(layer):
    blk = {"q4_k": 144, "q5_k": 176, "q6_k": 210}
    return sum(-(-N * (K // 256) * blk[f] // 256) * 256 for (_, f, N, K) in layer)


def test_plan_keeps_what_fits_beside_the_ring():
    lb = layer_bytes(L70)
    assert lb == 541_851_648
    for budget_gb in (3, 8, 20, 40):
        budget = budget_gb * 10**9
        r, s = kq.chain_plan([L70] * 80, budget, max_slots=4)
        assert s == 4
        assert r == (budget - 4 * lb) // lb
        assert (r + s) * lb <= budget < (r + s + 1) * lb


def test_plan_everything_resident_and_small_budgets():
    lb = layer_bytes(L70)
    assert kq.chain_plan([L70] * 80, 80 * lb, max_slots=4) == (80, 0)
    assert kq.chain_plan([L70] * 80, 180 * 10**9, max_slots=4) == (80, 0)
    # fewer slots when the budget holds fewer than max_slots layers
    assert kq.chain_plan([L70] * 80, 2 * lb + 5, max_slots=4) == (0, 2)
    assert kq.chain_plan([L70] * 80, lb, max_slots=4) == (0, 1)
    # never more resident layers than leave the ring its slots
    assert kq.chain_plan([L70] * 6, 5 * lb, max_slots=4) == (1, 4)
    with pytest.raises(kq.KQError):
        kq.chain_plan([L70] * 80, lb - 1, max_slots=4)   # not even one layer
    with pytest.raises(kq.KQError):
        kq.chain_plan([L70] * 80, 20 * 10**9, max_slots=0)
    with pytest.raises(kq.KQError):
        kq.chain_plan([[(None, "q4_k", 16, 300)]] * 4, 10**9)  # K not a multiple of 256
