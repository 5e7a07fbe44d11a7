"""Pins for the oracle's smooth-K and Hadamard steps (CPU only).

FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention": subtracting the
per-head mean key is exact for softmax (q.(k_j - kbar) = q.k_j - q.kbar, a shift
shared by every key), and applying the same orthonormal Hadamard matrix to Q and
K leaves every q.k unchanged.  These tests check the oracle's implementation of
both against scipy's Hadamard matrix, exact integer arithmetic and the two
invariances stated on the page.
"""
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from nvfp4_precision_b200 import synth


def bf16_bits_of(x: np.ndarray) -> np.ndarray:
    return synth.bf16_bits(torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16))


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def test_hadamard_scale_constant():
    c = oracle.hadamard_scale()
    assert np.float32(c).view(np.uint32) == 0x3DB504F3
    assert c == np.float32(1.0 / np.sqrt(128.0))


def test_fwht_equals_sylvester_matrix_on_integers():
    H = scipy.linalg.hadamard(128).astype(np.int64)
    rng = np.random.default_rng(0)
    x = rng.integers(-1000, 1000, size=(16, 128))
    got = oracle.fwht128(x.astype(np.float32))
    want = x @ H.T  # Sylvester H is symmetric; every partial sum is an exact fp32 integer
    assert np.array_equal(got.astype(np.int64), want)


def test_fwht_applied_twice_is_128_times_identity():
    rng = np.random.default_rng(1)
    x = rng.integers(-50, 50, size=(8, 128)).astype(np.float32)
    assert np.array_equal(oracle.fwht128(oracle.fwht128(x)), 128 * x)


def test_transform_matches_fp64_orthonormal_hadamard_within_fp32_bound():
    Hn = scipy.linalg.hadamard(128) / np.sqrt(128.0)
    assert np.allclose(Hn @ Hn.T, np.eye(128), atol=1e-14)
    rng = np.random.default_rng(2)
    xb = bf16_bits_of(rng.standard_normal((64, 128)) * 3)
    y = oracle.transform_rows(xb)
    x = bits_to_f32(xb).astype(np.float64)
    exact = x @ Hn.T
    # 7 butterfly stages and one scaling, each a relative 2^-24 rounding
    bound = 9 * 2.0 ** -24 * np.abs(x).sum(axis=1, keepdims=True) / np.sqrt(128.0)
    assert np.all(np.abs(y - exact) <= bound)


def test_no_hadamard_flag_is_identity_and_mean_is_subtracted():
    rng = np.random.default_rng(3)
    xb = bf16_bits_of(rng.standard_normal((4, 128)))
    mean = rng.standard_normal(128).astype(np.float32)
    y = oracle.transform_rows(xb, mean=mean, flags=oracle.NO_HADAMARD)
    assert np.array_equal(y, bits_to_f32(xb) - mean)


def exact_ksum(kf32: np.ndarray) -> np.ndarray:
    """sum_n round_half_even(k * 2^24) with Python integers (brute force)."""
    BH, N, D = kf32.shape
    out = np.zeros((BH, D), dtype=object)
    for bh in range(BH):
        for c in range(D):
            out[bh, c] = sum(round(Fraction(float(v)) * (1 << 24)) for v in kf32[bh, :, c])
    return out


def test_ksum_is_exact_fixed_point_sum():
    rng = np.random.default_rng(4)
    k = rng.standard_normal((2, 37, 128)) * 3
    # values below the 2^-24 resolution, including exact ties at 0.5 and 1.5 units
    k[0, :6, 0] = [2.0 ** -25, 3 * 2.0 ** -25, -(2.0 ** -25), 2.0 ** -30, 5 * 2.0 ** -26, 1000.5]
    kb = bf16_bits_of(k)
    S, st = oracle.ksum(kb)
    assert st == oracle.OK
    want = exact_ksum(bits_to_f32(kb))
    assert np.array_equal(S.astype(object), want)


def test_ksum_order_independent_and_mean_of_constant():
    rng = np.random.default_rng(5)
    kb = bf16_bits_of(rng.standard_normal((1, 300, 128)) * 7)
    S1, _ = oracle.ksum(kb)
    S2, _ = oracle.ksum(np.ascontiguousarray(kb[:, rng.permutation(300)]))
    assert np.array_equal(S1, S2)
    const = bf16_bits_of(np.full((1, 77, 128), -1.75))
    S, _ = oracle.ksum(const)
    assert np.all(oracle.kmean(S, 77) == np.float32(-1.75))


def test_kmean_is_correctly_rounded_within_half_ulp():
    rng = np.random.default_rng(6)
    kb = bf16_bits_of(rng.standard_normal((3, 1000, 128)) * 5 + 2)
    S, _ = oracle.ksum(kb)
    m = oracle.kmean(S, 1000)
    for bh in range(3):
        for c in range(0, 128, 7):
            exact = Fraction(int(S[bh, c]), 1000 * (1 << 24))
            got = Fraction(float(m[bh, c]))
            ulp = Fraction(float(np.spacing(np.float32(m[bh, c]))))
            assert abs(got - exact) <= ulp / 2 * (1 + Fraction(1, 1 << 20))


def test_ksum_range_errors():
    k = np.zeros((1, 4, 128), np.float32)
    k[0, 1, 5] = 2.0 ** 20
    S, st = oracle.ksum(bf16_bits_of(k))
    assert st == oracle.ERR_RANGE
    k[0, 1, 5] = np.inf
    S, st = oracle.ksum(bf16_bits_of(k))
    assert st == oracle.ERR_RANGE
    k[0, 1, 5] = 2.0 ** 19
    S, st = oracle.ksum(bf16_bits_of(k))
    assert st == oracle.OK and S[0, 5] == 2 ** 43


def softmax(x):
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return e / e.sum(axis=-1, keepdims=True)


def test_page_invariances_before_quantisation():
    """(qH).(kH) = q.k and softmax(q.(k - kbar)) = softmax(q.k), on the
    oracle's own fp32 transform of offset keys (the page's exactness claims)."""
    w = synth.custom("inv", 1, 1, 256, seed=11, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w, ("q", "k"))
    qb = synth.bf16_bits(d["q"])[0, 0]
    kb = synth.bf16_bits(d["k"])[0, 0]
    S, _ = oracle.ksum(kb[None])
    mean = oracle.kmean(S, 256)[0]
    yq = oracle.transform_rows(qb).astype(np.float64)
    yk = oracle.transform_rows(kb, mean=mean).astype(np.float64)
    q = bits_to_f32(qb).astype(np.float64)
    k = bits_to_f32(kb).astype(np.float64)
    ksm = bits_to_f32(kb).astype(np.float64) - mean.astype(np.float64)
    scale = 1 / np.sqrt(128)
    # Hadamard: logits of the smoothed keys unchanged by the rotation
    lhs = yq @ yk.T
    rhs = q @ ksm.T
    tol = 1e-5 * np.abs(q).sum(1)[:, None] * np.abs(ksm).sum(1)[None, :] / 128
    assert np.all(np.abs(lhs - rhs) <= tol + 1e-4)
    # Smoothing: softmax rows unchanged by the shared shift q.kbar
    p_orig = softmax(q @ k.T * scale)
    p_smooth = softmax(lhs * scale)
    assert np.max(np.abs(p_orig - p_smooth)) < 1e-4
    # in exact arithmetic the same identities hold to fp64 rounding
    Hn = scipy.linalg.hadamard(128) / np.sqrt(128.0)
    assert np.allclose((q @ Hn) @ (ksm @ Hn).T, q @ ksm.T, rtol=0, atol=1e-9)
    assert np.allclose(softmax(q @ ksm.T * scale), p_orig, rtol=0, atol=1e-12)
