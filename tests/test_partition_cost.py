"""Pope et al. partitioning cost model, pinned by the numbers the CS349E lecture 4
script (`03_pope_partitioning.py`) prints for PaLM 540B on TPU v4.

Each expected value below is quoted from that page's observations or tables
(demo 1, demo 3 = the paper's Table 1, demo 4); the tolerances are the page's
own rounding (one printed digit), or ~1 % where the page compares to Table 1.
"""
import pytest

from tensor_llama_transformer_b200 import partition_cost as pc

M, CHIP = pc.PALM_540B, pc.TPU_V4


def test_demo1_1d_comm_independent_of_chips():
    """Demo 1, B = 512: the 1D FFN traffic over 118 layers is 16.5 ms at n = 64 and
    does not change with n."""
    t = pc.ffn_comm_1d(512, M.E, CHIP.link_bw) * M.layers
    assert t == pytest.approx(16.5e-3, abs=0.05e-3)


@pytest.mark.parametrize("n,ms", [(64, 8.3), (256, 4.1)])
def test_demo1_2d_comm(n, ms):
    """Demo 1: 2D is 8.3 ms at n = 64 and 4.1 ms at n = 256, i.e. 1/2 and 1/4 of the 1D
    16.5 ms (the page's 8.3 is half of its rounded 16.5; the unrounded half is 8.249)."""
    t = pc.ffn_comm_2d(512, M.E, M.F, n, CHIP.link_bw) * M.layers
    assert t == pytest.approx(ms * 1e-3, abs=0.06e-3)
    t1 = pc.ffn_comm_1d(512, M.E, CHIP.link_bw) * M.layers
    assert t == pytest.approx(t1 * 4 / n ** 0.5, rel=1e-12)


def test_demo1_crossover_at_16_chips():
    """Demo 1: 1D and 2D are equal at sqrt(n) = 4 (F = 4E), and 2D is cheaper above 16 chips."""
    t1 = pc.ffn_comm_1d(512, M.E, CHIP.link_bw)
    assert pc.ffn_comm_2d(512, M.E, M.F, 16, CHIP.link_bw) == pytest.approx(t1, rel=1e-12)
    assert pc.ffn_comm_2d(512, M.E, M.F, 8, CHIP.link_bw) > t1
    assert pc.ffn_comm_2d(512, M.E, M.F, 32, CHIP.link_bw) < t1
    assert M.F == 4 * M.E


def test_demo1_weight_read_and_compute():
    """Demo 1 at n = 64: reading the FFN weights takes 8.4 ms per chip, compute 18.7 ms."""
    assert pc.ffn_weight_read(M.E, M.F, M.layers, 64, CHIP.mem_bw) == pytest.approx(8.4e-3, abs=0.05e-3)
    assert pc.ffn_compute(512, M.E, M.F, M.layers, 64, CHIP.peak_flops) == pytest.approx(18.7e-3,
                                                                                         abs=0.05e-3)


@pytest.mark.parametrize("layout,b128,b512", [
    ("mha", 1320, 330),              # multi-head attention
    ("mqa_heads", 660, 165),         # multi-query, split by heads: KV copied to every chip
    ("mqa_batch", 43000, 10700),     # multi-query, split by batch (Pope)
])
def test_demo3_table1_max_context(layout, b128, b512):
    """Demo 3 = the paper's Table 1 (64 TPU v4, 30 % of HBM for the KV cache):
    longest context at batch 128 / 512, within the ~1 % the page reports."""
    assert pc.max_context(M, CHIP, 64, 128, layout) == pytest.approx(b128, rel=0.015)
    assert pc.max_context(M, CHIP, 64, 512, layout) == pytest.approx(b512, rel=0.015)


def test_demo4_decode_bound():
    """Demo 4 (64 chips, context 2048, B = 64): reading 540B int8 parameters takes
    ~7 ms per chip; the measured steps (28.5 ms int8, 36.9 ms bf16) are 2.4-3.4 times
    the lower bound; the int8 serving cost is about 28 chip-ms per token."""
    b8 = pc.decode_bound(M, CHIP, 64, 64, 2048, weight_bytes=1)
    b16 = pc.decode_bound(M, CHIP, 64, 64, 2048, weight_bytes=2)
    assert b8.weights == pytest.approx(7.0e-3, abs=0.05e-3)
    assert b16.weights == pytest.approx(2 * b8.weights, rel=1e-12)
    r8, r16 = 28.5e-3 / b8.bound, 36.9e-3 / b16.bound
    assert 2.35 <= min(r8, r16) and max(r8, r16) <= 3.45
    assert r8 == pytest.approx(3.4, abs=0.05) and r16 == pytest.approx(2.4, abs=0.05)
    assert pc.cost_chip_ms_per_token(64, 28.5e-3, 64) == pytest.approx(28.5, abs=0.05)


def test_weights_dominate_small_batch_decode():
    """Demo 4's reading: at small batch the weight read is the largest term of the bound."""
    b = pc.decode_bound(M, CHIP, 64, 64, 2048, weight_bytes=2)
    assert b.weights > max(b.kv, b.compute, b.comm)


# Demo 2 (the paper's Figure 3 setting): one FFN layer, E 16384, F 65536, 64 chips.
E2, F2 = 16384, 65536


def test_demo2_crossover_at_f_over_4():
    """Weight-stationary and weight-gathered traffic are equal at BL = F / 4 = 16,384
    tokens; fewer tokens favour moving activations, more favour moving weights."""
    bl = F2 // 4
    t_g, N = pc.ffn_comm_gathered(bl, E2, F2, 64, CHIP.link_bw)
    assert t_g == pytest.approx(pc.ffn_comm_2d(bl, E2, F2, 64, CHIP.link_bw), rel=1e-12)
    assert N == pytest.approx(4.0)  # sqrt(BL n / F)
    assert pc.ffn_layout(2048, E2, F2, 64, CHIP.link_bw) == "stationary"
    assert pc.ffn_layout(65536, E2, F2, 64, CHIP.link_bw) == "gathered"


def test_demo2_traffic_scaling():
    """Stationary traffic grows as BL, gathered as sqrt(BL)."""
    a = pc.ffn_comm_gathered(65536, E2, F2, 64, CHIP.link_bw)[0]
    b = pc.ffn_comm_gathered(262144, E2, F2, 64, CHIP.link_bw)[0]
    assert b / a == pytest.approx(2.0, rel=1e-12)
    assert pc.ffn_comm_2d(262144, E2, F2, 64, CHIP.link_bw) / pc.ffn_comm_2d(
        65536, E2, F2, 64, CHIP.link_bw) == pytest.approx(4.0, rel=1e-12)


def test_demo2_compute_share_last_row():
    """Demo 2's last row (1,048,576 tokens): compute is 94 % of compute + the cheaper
    communication (the page's printed observation)."""
    bl = 1048576
    comp = pc.ffn_compute(bl, E2, F2, 1, 64, CHIP.peak_flops)
    comm = min(pc.ffn_comm_gathered(bl, E2, F2, 64, CHIP.link_bw)[0],
               pc.ffn_comm_2d(bl, E2, F2, 64, CHIP.link_bw))
    assert round(comp / (comp + comm) * 100) == 94


def test_2d_traffic_general_f():
    """4 BL sqrt(E F / n): the paper's 8 BL E / sqrt(n) at F = 4 E (the printed values
    above pin that case); for F = E it is half of that, and at any F the optimum
    weight-gathered traffic (4 E sqrt(BL F / n)) meets it at BL = E."""
    bw = CHIP.link_bw
    E, n, bl = 8192, 64, 1024
    assert pc.ffn_comm_2d(bl, E, 4 * E, n, bw) == pytest.approx(8.0 * bl * E * 2 / (8 * bw),
                                                                rel=1e-12)
    assert pc.ffn_comm_2d(bl, E, E, n, bw) == pytest.approx(
        0.5 * pc.ffn_comm_2d(bl, E, 4 * E, n, bw), rel=1e-12)
    for F in (E, 2 * E, 4 * E, 7 * E):
        t_g, _ = pc.ffn_comm_gathered(E, E, F, n, bw)
        assert t_g == pytest.approx(pc.ffn_comm_2d(E, E, F, n, bw), rel=1e-12)
