"""Host logic of bench.py's roofline accounting: the per-kernel modular
multiply counts add up to the whole key switch's count at every level and
basis of the workloads, and the operation variants scale from it as stated."""
import pytest

import bench
from key_switching_b200 import synth


@pytest.mark.parametrize("logN,L,alpha", [(12, 4, 2), (16, 24, 4), (17, 40, 5)])
def test_stage_counts_sum_to_key_switch(logN, L, alpha):
    for l in sorted({L, L - 1, alpha + 1, alpha, 1}):
        total = bench.workload_counts(logN, L, alpha, l)["modmuls"]
        assert sum(bench.stage_modmuls(logN, L, alpha, l).values()) == total, l


def test_key_switch_counts_n16():
    w = bench.workload_counts(16, 24, 4, 24)
    assert w["modmuls"] == 195_035_136
    assert w["chacha_blocks"] == 6 * 28 * (1 << 16) // 8       # beta x (l + alpha) limbs, 8 coefficients per block
    assert w["bytes"] == (2 * 24 + 6 * 28 + 2 * 24) * (1 << 16) * 4   # c0, c1 in; key b; c0', c1' out
    stored = bench.workload_counts(16, 24, 4, 24, regen=False)
    assert stored["bytes"] - w["bytes"] == 6 * 28 * (1 << 16) * 4 and stored["chacha_blocks"] == 0


def test_operation_variants():
    ks = bench.workload_counts(16, 24, 4, 24)
    rot = bench.op_counts(synth.WORKLOADS["rotate_n16"], 24)
    assert rot == ks                                              # the automorphism is a permutation
    rel = bench.op_counts(synth.WORKLOADS["relin_mul_n16"], 24)
    assert rel["modmuls"] - ks["modmuls"] == 4 * 24 * (1 << 16)   # four slot products per coefficient
    h = bench.op_counts(synth.WORKLOADS["hoisted8_n16"], 24)
    st = bench.stage_modmuls(16, 24, 4, 24)
    up = st["intt_row_c1"] + st["modup_col"]
    assert h["modmuls"] == up + 8 * (ks["modmuls"] - up)           # one ModUp, eight finishes
    assert h["chacha_blocks"] == 8 * ks["chacha_blocks"]
