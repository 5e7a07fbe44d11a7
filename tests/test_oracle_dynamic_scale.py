"""Pins for the oracle's dynamic per-tensor scale (CPU only).

FastVideo "Pika H3 Flex in FastVideo": section "NVFP4 QAD" sets static
activation scales and names scaling to the largest value as the plain
alternative; section "FP4 attention" quantises Q and K with E2M1 values and
one E4M3 scale per 16 channels under a per-tensor global scale.  The dynamic
scale maps the largest magnitude of the transformed tensor to the top of the
two-level range: g = fl32(amax / (6 * 448)), at least 2^-64.

The pins do not reuse the oracle's transform: the amax is recomputed in fp64
from scipy's Hadamard matrix and numpy's mean, and the remaining checks are
closed forms and exact invariants of the definition.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from nvfp4_precision_b200 import synth

G_MIN = np.float32(2.0 ** -64)


def bits_of(x):
    return synth.bf16_bits(torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16))


def values_of(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _data(seed=5, N=200, H=3):
    w = synth.custom("dyn", 1, H, N, seed=seed, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w, ("q", "k"))
    return synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"])


def _fp64_amax(bits, smooth):
    x = values_of(bits)  # [B,H,N,128]
    if smooth:
        x = x - x.mean(axis=2, keepdims=True)
    Hm = scipy.linalg.hadamard(128).astype(np.float64) / np.sqrt(128.0)
    return np.abs(x @ Hm).max()


@pytest.mark.parametrize("flags", [0, oracle.NO_SMOOTH_K])
def test_dynamic_g_is_the_transformed_amax_over_2688(flags):
    qb, kb = _data()
    gq, gk, st = oracle.dynamic_gscale(qb, kb, flags)
    assert st == oracle.OK
    aq = _fp64_amax(qb, smooth=False)
    ak = _fp64_amax(kb, smooth=not (flags & oracle.NO_SMOOTH_K))
    # fp32 transform vs fp64: a few units in the last place of the largest output
    assert abs(float(gq) - aq / 2688.0) <= 1e-5 * aq / 2688.0
    assert abs(float(gk) - ak / 2688.0) <= 1e-5 * ak / 2688.0


def test_dynamic_g_without_transforms_is_exact_closed_form():
    qb, kb = _data(seed=6)
    gq, gk, st = oracle.dynamic_gscale(qb, kb, oracle.NO_SMOOTH_K | oracle.NO_HADAMARD)
    assert st == oracle.OK
    assert gq == np.float32(np.abs(values_of(qb)).max()) / np.float32(2688.0)
    assert gk == np.float32(np.abs(values_of(kb)).max()) / np.float32(2688.0)


def test_dynamic_g_puts_the_tensor_amax_at_the_top_of_the_range():
    qb, kb = _data(seed=7)
    out = oracle.quantize_qk(qb, kb, dynamic=True)
    assert out["status"] == oracle.OK
    for t, bits, smooth in (("q", qb, False), ("k", kb, True)):
        g = out["g" + t]
        # the block holding the amax gets the largest UE4M3 scale, 448 (0x7E)
        assert out[t + "_scales"].max() == 0x7E
        deq = oracle.dequant(out[t + "_codes"], out[t + "_scales"], float(g))
        top = np.abs(deq).max()
        assert top == np.float32(np.float32(g * np.float32(448.0)) * np.float32(6.0))
        assert abs(top - _fp64_amax(bits, smooth)) <= 1e-5 * top


@pytest.mark.parametrize("e", [5, -7])
def test_dynamic_quantisation_is_invariant_to_power_of_two_scaling(e):
    """Scaling the inputs by 2^e scales every fp32 step exactly (mean, butterflies,
    amax, g), so the codes and scale bytes are unchanged and g scales by 2^e."""
    qb, kb = _data(seed=8)
    qs = bits_of(values_of(qb) * 2.0 ** e)
    ks = bits_of(values_of(kb) * 2.0 ** e)
    a = oracle.quantize_qk(qb, kb, dynamic=True)
    b = oracle.quantize_qk(qs, ks, dynamic=True)
    for key in ("q_codes", "q_scales", "k_codes", "k_scales"):
        assert np.array_equal(a[key], b[key]), key
    assert b["gq"] == np.float32(a["gq"] * 2.0 ** e) and b["gk"] == np.float32(a["gk"] * 2.0 ** e)
    if e < 0:
        # with the unit scale the small inputs fall into E4M3's subnormal range
        c = oracle.quantize_qk(qs, ks)
        assert not np.array_equal(c["q_codes"], a["q_codes"])


def test_dynamic_scale_removes_the_unit_scale_saturation():
    """With g = 1 a block amax above 6 * 448 saturates the scale at 448 and the
    codes at 6, so the dequantised maximum is 2688; the dynamic scale keeps it."""
    x = np.zeros((1, 1, 4, 128), np.float32)
    x[0, 0, :, 0] = [9984.0, -3.0, 1.0, 0.5]  # 9984 is exact in bf16
    xb = bits_of(x)
    f = oracle.NO_SMOOTH_K | oracle.NO_HADAMARD
    unit = oracle.quantize_qk(xb, xb, flags=f)
    assert np.abs(oracle.dequant(unit["q_codes"], unit["q_scales"])).max() == 2688.0
    dyn = oracle.quantize_qk(xb, xb, flags=f, dynamic=True)
    assert dyn["gq"] == np.float32(9984.0) / np.float32(2688.0)
    top = np.abs(oracle.dequant(dyn["q_codes"], dyn["q_scales"], float(dyn["gq"]))).max()
    assert abs(top - 9984.0) <= 1e-3


def test_dynamic_scale_of_zero_and_tiny_tensors():
    z = np.zeros((1, 2, 5, 128), np.float32)
    zb = bits_of(z)
    out = oracle.quantize_qk(zb, zb, dynamic=True)
    assert out["status"] == oracle.OK
    assert out["gq"] == G_MIN and out["gk"] == G_MIN
    assert not out["q_codes"].any() and not out["q_scales"].any() and not out["k_codes"].any()
    t = z.copy()
    t[0, 1, 2, 7] = 2.0 ** -80  # amax / 2688 < 2^-64: g is raised to 2^-64
    tb = bits_of(t)
    gq, gk, st = oracle.dynamic_gscale(tb, tb, oracle.NO_SMOOTH_K)
    assert st == oracle.OK and gq == G_MIN and gk == G_MIN
    out = oracle.quantize_qk(tb, tb, flags=oracle.NO_SMOOTH_K, dynamic=True)
    # scale 2^-80 / 6 / 2^-64 is below E4M3's smallest subnormal: the block is
    # zero (codes keep the sign of their input, so only the magnitude bits are 0)
    assert not out["q_scales"].any() and not (out["q_codes"] & 0x77).any()


def test_dynamic_scale_reports_nonfinite_input():
    q = np.zeros((1, 1, 3, 128), np.float32)
    q[0, 0, 2, 9] = np.inf
    _, _, st = oracle.dynamic_gscale(bits_of(q), bits_of(np.zeros_like(q)))
    assert st == oracle.ERR_RANGE
