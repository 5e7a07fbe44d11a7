"""Pins for the oracle's NVFP4 pack and dequantisation (CPU only).

FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention": Q and K are
quantised with E2M1 values and one E4M3 scale per 16 channels under a unit
global scale.  The yuxiaoba.github.io review's block-scale figure caption: a
block of sixteen values shares one scale and a small value rounds to zero.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

E2M1_GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def bf16_bits_of(x):
    return synth.bf16_bits(torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16))


def unpack_codes(codes):
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,))


def test_page_block_example(golden_dir):
    ex = json.load(open(os.path.join(golden_dir, "page_block_example.json")))
    row = np.zeros((1, 1, 1, 128), np.float32)
    row[0, 0, 0, :16] = ex["block"]
    qb = bf16_bits_of(row)
    out = oracle.quantize_qk(qb, qb, flags=oracle.NO_SMOOTH_K | oracle.NO_HADAMARD)
    assert out["status"] == oracle.OK
    assert out["q_scales"][0, 0, 0, 0] == ex["expected_scale_byte"]
    assert oracle.ue4m3_decode(np.array([ex["expected_scale_byte"]], np.uint8))[0] == ex["expected_scale_value"]
    codes = unpack_codes(out["q_codes"][0, 0, 0])[:16]
    assert codes.tolist() == ex["expected_codes"]
    assert out["q_codes"][0, 0, 0, :2].tolist() == ex["expected_packed_bytes_first_two"]
    deq = oracle.dequant(out["q_codes"], out["q_scales"])[0, 0, 0, :16]
    assert deq.tolist() == ex["expected_dequant"]
    # the small value is lost, the others survive exactly
    assert deq[1] == 0.0 and ex["block"][1] != 0.0
    # all-zero blocks give a zero scale and zero codes
    assert np.all(out["q_scales"][0, 0, 0, 1:] == 0) and np.all(out["q_codes"][0, 0, 0, 8:] == 0)


def test_grid_values_round_trip_exactly():
    """Rows already on a s*E2M1 grid with amax = 6s come back unchanged."""
    rng = np.random.default_rng(0)
    scales = np.array([0.25, 0.5, 1.0, 1.125, 2.0, 0.0625, 3.5, 40.0])
    rows = []
    for s in scales:
        for _ in range(3):
            blk = rng.choice(E2M1_GRID, 16) * rng.choice([-1, 1], 16) * s
            blk[rng.integers(16)] = 6 * s
            rows.append(blk)
    y = np.concatenate(rows).reshape(-1, 128).astype(np.float32)
    codes, sc = oracle.quantize_rows(y)
    assert np.array_equal(oracle.dequant(codes, sc), y)


def test_error_bound_and_sign_symmetry():
    rng = np.random.default_rng(1)
    y = (rng.standard_t(3, size=(512, 128)) * np.exp2(rng.integers(-8, 8, (512, 1)))).astype(np.float32)
    codes, sc = oracle.quantize_rows(y)
    yh = oracle.dequant(codes, sc).astype(np.float64)
    sd = oracle.ue4m3_decode(sc).astype(np.float64)          # [512, 8]
    a = np.abs(y.reshape(512, 8, 16)).max(-1).astype(np.float64)
    err = np.abs(y.reshape(512, 8, 16) - yh.reshape(512, 8, 16)).max(-1)
    # half the widest E2M1 gap (4 -> 6) times the scale, or the saturation excess
    bound = np.maximum(sd * 1.0, a - 6 * sd)
    assert np.all(err <= bound + 1e-30)
    # scale is amax/6 to within UE4M3 rounding (relative 2^-4), in the normal, unsaturated range
    normal = (a / 6 >= 2.0 ** -6) & (a / 6 <= 448.0)
    rel = np.abs(sd[normal] - a[normal] / 6) / (a[normal] / 6)
    assert rel.max() <= 2.0 ** -4
    # rounding is odd-symmetric
    c2, s2 = oracle.quantize_rows(-y)
    assert np.array_equal(s2, sc)
    assert np.array_equal(oracle.dequant(c2, s2), -oracle.dequant(codes, sc))


def test_tiny_and_huge_blocks():
    y = np.zeros((2, 128), np.float32)
    y[0, :16] = 6 * 2.0 ** -11          # a/6 = 2^-11 rounds to scale 0: whole block is zero
    y[0, 16:32] = np.linspace(-1, 1, 16) * 1e6   # a/6 > 448: scale saturates, codes saturate
    codes, sc = oracle.quantize_rows(y)
    assert sc[0, 0] == 0 and np.all(unpack_codes(codes)[0, :16] == 0)
    assert sc[0, 1] == 0x7E
    u = unpack_codes(codes)[0, 16:32]
    assert (u[0] & 7) == 7 and (u[-1] & 7) == 7


def test_global_scale_divides_block_scale():
    rng = np.random.default_rng(2)
    y = rng.standard_normal((64, 128)).astype(np.float32) * 8
    g = np.float32(2.0)  # power of two: exact rescaling of every step
    c1, s1 = oracle.quantize_rows(y, 1.0)
    c2, s2 = oracle.quantize_rows(y, float(g))
    assert np.array_equal(oracle.dequant(c2, s2, float(g)), oracle.dequant(c1, s1, 1.0))


def test_monotone_within_block():
    y = np.linspace(-6.5, 6.5, 128, dtype=np.float32).reshape(1, 128)
    # one block with a fixed amax of 6 so all share scale 1.0
    y = np.tile(np.linspace(-6, 6, 16, dtype=np.float32), 8).reshape(1, 128)
    codes, sc = oracle.quantize_rows(y)
    d = oracle.dequant(codes, sc)[0]
    for b in range(8):
        assert np.all(np.diff(d[16 * b:16 * b + 16]) >= 0)


def test_quantize_qk_flags_and_layout():
    w = synth.custom("q", 1, 2, 48, seed=3, k_offset_std=2.0)
    d = synth.generate(w, ("q", "k"))
    qb, kb = synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"])
    full = oracle.quantize_qk(qb, kb)
    assert full["status"] == oracle.OK
    # Q path = transform then pack, row by row
    yq = oracle.transform_rows(qb.reshape(-1, 128))
    c, s = oracle.quantize_rows(yq)
    assert np.array_equal(full["q_codes"].reshape(-1, 64), c)
    assert np.array_equal(full["q_scales"].reshape(-1, 8), s)
    # K path uses the per-head mean
    S, _ = oracle.ksum(kb.reshape(2, 48, 128))
    m = oracle.kmean(S, 48)
    assert np.array_equal(full["k_mean"].reshape(2, 128), m)
    yk = np.concatenate([oracle.transform_rows(kb[0, h], mean=m[h]) for h in range(2)])
    c, s = oracle.quantize_rows(yk)
    assert np.array_equal(full["k_codes"].reshape(-1, 64), c)
    # NO_SMOOTH_K: the mean is not subtracted and reported as zero
    ns = oracle.quantize_qk(qb, kb, flags=oracle.NO_SMOOTH_K)
    assert np.all(ns["k_mean"] == 0)
    c, s = oracle.quantize_rows(oracle.transform_rows(kb.reshape(-1, 128)))
    assert np.array_equal(ns["k_codes"].reshape(-1, 64), c)


def test_quantize_qk_flags_nonfinite_q():
    q = np.zeros((1, 1, 2, 128), np.float32)
    q[0, 0, 1, 3] = np.nan
    out = oracle.quantize_qk(bf16_bits_of(q), bf16_bits_of(np.zeros_like(q)))
    assert out["status"] == oracle.ERR_RANGE
