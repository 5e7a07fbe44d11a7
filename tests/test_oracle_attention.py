"""Pins for the oracle's fp64 attention (CPU only).

The oracle computes softmax(Q K^T * scale) V over the dequantised Q and K and
bf16 V (FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention": QK in
FP4, P and V in BF16; attention is dense and non-causal).  It is checked
against PyTorch's fp64 scaled_dot_product_attention, closed forms and
invariants, and the page's qualitative claim that smoothing K plus the
Hadamard rotation lowers FP4 attention error on data with outlier channels.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from nvfp4_precision_b200 import synth


def bits_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def rand_head(N, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    q = (rng.standard_normal((N, 128)) * scale).astype(np.float32)
    k = (rng.standard_normal((N, 128)) * scale).astype(np.float32)
    v = synth.bf16_bits(torch.from_numpy(rng.standard_normal((N, 128)).astype(np.float32)).to(torch.bfloat16))
    return q, k, v


@pytest.mark.parametrize("N", [1, 2, 3, 17, 64, 200])
@pytest.mark.parametrize("scale", [None, 0.05])
def test_matches_torch_sdpa_fp64(N, scale):
    q, k, v = rand_head(N, N, 2.0)
    O, lse = oracle.attention_head(q, k, v, scale=scale)
    s = 1 / np.sqrt(128) if scale is None else scale
    qt = torch.from_numpy(q.astype(np.float64))[None, None]
    kt = torch.from_numpy(k.astype(np.float64))[None, None]
    vt = torch.from_numpy(bits_to_f32(v).astype(np.float64))[None, None]
    want = F.scaled_dot_product_attention(qt, kt, vt, scale=s)[0, 0].numpy()
    assert np.max(np.abs(O - want)) < 1e-12
    logits = (q.astype(np.float64) @ k.astype(np.float64).T) * s
    assert np.allclose(lse, torch.logsumexp(torch.from_numpy(logits), -1).numpy(), atol=1e-12, rtol=0)


def test_row_subset_matches_full():
    q, k, v = rand_head(50, 1)
    O, lse = oracle.attention_head(q, k, v)
    rows = np.array([0, 7, 49, 13])
    O2, lse2 = oracle.attention_head(q, k, v, rows=rows)
    assert np.array_equal(O2, O[rows]) and np.array_equal(lse2, lse[rows])


def test_key_permutation_invariance_and_normalisation():
    q, k, v = rand_head(80, 2, 3.0)
    O, lse = oracle.attention_head(q, k, v)
    perm = np.random.default_rng(0).permutation(80)
    O2, lse2 = oracle.attention_head(q, np.ascontiguousarray(k[perm]), np.ascontiguousarray(v[perm]))
    assert np.max(np.abs(O - O2)) < 1e-12 and np.max(np.abs(lse - lse2)) < 1e-12
    logits = (q.astype(np.float64) @ k.astype(np.float64).T) / np.sqrt(128)
    assert np.allclose(np.exp(logits - lse[:, None]).sum(1), 1.0, atol=1e-12)


def test_single_key_and_dominant_key():
    q, k, v = rand_head(1, 3)
    O, lse = oracle.attention_head(q, k, v)
    assert np.array_equal(O[0], bits_to_f32(v[0]).astype(np.float64))
    q, k, v = rand_head(10, 4)
    k[6] = q[0] * 100  # logit of key 6 exceeds the others by far more than 800
    O, _ = oracle.attention_head(q, k, v, rows=np.array([0]))
    assert np.array_equal(O[0], bits_to_f32(v[6]).astype(np.float64))


def test_smooth_and_hadamard_lower_fp4_error_on_outlier_data():
    """Qualitative ordering of the page's per-layer error table: plain FP4 >
    FP4 with smooth K + Hadamard (not the page's values, which need real data)."""
    w = synth.custom("ord", 1, 2, 512, seed=5, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w)
    qb, kb, vb = (synth.bf16_bits(d[t]) for t in "qkv")
    errs = {}
    for name, flags in [("plain", oracle.NO_SMOOTH_K | oracle.NO_HADAMARD), ("smooth+H", 0)]:
        qq = oracle.quantize_qk(qb, kb, flags=flags)
        O, _ = oracle.attention(qq["q_codes"], qq["q_scales"], qq["k_codes"], qq["k_scales"], vb)
        errs[name] = O
    # exact unquantised attention on the original bf16 values
    ref = np.empty_like(errs["plain"])
    for h in range(2):
        ref[0, h], _ = oracle.attention_head(bits_to_f32(qb[0, h]), bits_to_f32(kb[0, h]), vb[0, h])
    e_plain = np.abs(errs["plain"] - ref).mean()
    e_fix = np.abs(errs["smooth+H"] - ref).mean()
    assert e_fix < e_plain, (e_fix, e_plain)
