"""The tensor-core rates behind the composite roofline: back-to-back
block-scaled FP4 MMAs (kind::mxf4nvf4, M128 N256 K64) and BF16 MMAs
(kind::f16, M128 N256 K16) on every SM with every operand resident, through
fp4attn_probe_mma_rate.  The FP4 score product runs at four times the BF16
rate per clock (the nominal dense ratio the roofline takes), and the BF16
product at its 8192 FLOP per clock per SM."""
import pytest

from gpu_helpers import fa

pytestmark = pytest.mark.gpu


def test_fp4_block_scaled_mma_runs_at_four_times_bf16_per_clock():
    f4 = fa().fp4attn_probe_mma_rate(0, reps=20000)
    b16 = fa().fp4attn_probe_mma_rate(1, reps=5000)
    print("fp4", f4, "bf16", b16)
    assert 0.9 * 8192 < b16["flop_per_clk_sm"] <= 8192 * 1.01
    assert f4["flop_per_clk_sm"] / b16["flop_per_clk_sm"] > 3.6


def test_mma_rate_probe_rejects_bad_arguments():
    with pytest.raises(RuntimeError):
        fa().fp4attn_probe_mma_rate(2, reps=10)
    with pytest.raises(RuntimeError):
        fa().fp4attn_probe_mma_rate(0, reps=0)
