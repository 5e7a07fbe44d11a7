"""The page's toy heads on the GPU product path (FastVideo "Pika H3 Flex in
FastVideo", section "FP4 attention": 64 channels in four 16-value blocks,
32 keys, Gaussian values, a per-channel key bias and two scaled-up channels,
NVFP4 Q and K at unit global scale, P and V in BF16).

fp4attn_quantize_qk and fp4attn_forward take heads of 64 channels: the
prologue's codes, scales and key means must equal the oracle's width-general
restatement bit for bit (every flag combination), attention must stay within
the attention tolerance of the oracle's fp64 attention over the same
dequantised Q and K, and the toy study -- the error of O against fp64
attention of the unquantised inputs, per transform -- must show on the GPU
what it shows on the oracle.  Run with -s to see the table."""
import numpy as np
import pytest
import torch

import oracle
import oracle.toy as toy
from nvfp4_precision_b200 import synth

from gpu_helpers import assert_attention_close, fa

pytestmark = pytest.mark.gpu

FLAGS = {"plain": 3, "smooth K": 2, "Hadamard": 1, "both": 0}  # NO_SMOOTH_K = 1, NO_HADAMARD = 2


def _gpu_quantize(q, k, flags):
    out = fa().fp4attn_quantize_qk(q[None].cuda(), k[None].cuda(), flags=flags)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    return out


def _check_codes(out, ref, what):
    for key in ("q_codes", "q_scales", "k_codes", "k_scales", "k_mean"):
        got = out[key][0].cpu().numpy()
        if not np.array_equal(got, ref[key]):
            bad = np.argwhere(got != ref[key])
            raise AssertionError(f"{what}: {key} differs at {bad.shape[0]} places, first {bad[:3].tolist()}")


@pytest.mark.parametrize("flags", [0, 1, 2, 3])
def test_toy_prologue_bit_exact(flags):
    t = synth.toy_heads(256, seed=7)
    out = _gpu_quantize(t["q"], t["k"], flags)
    ref = toy.quantize(synth.bf16_bits(t["q"]), synth.bf16_bits(t["k"]), flags)
    if flags & 1:
        ref["k_mean"] = np.zeros_like(ref["k_mean"])
    _check_codes(out, ref, f"toy heads, flags {flags}")


@pytest.mark.parametrize("H,N", [(3, 1000), (2, 1), (1, 257)])
def test_narrow_prologue_bit_exact_longer_heads(H, N):
    """Heads of 64 channels beyond the toy's 32 keys: several key-sum CTAs per
    head, ragged tails, a single row."""
    t = synth.toy_heads(H, seed=11 + N, N=N)
    out = _gpu_quantize(t["q"], t["k"], 0)
    ref = toy.quantize(synth.bf16_bits(t["q"]), synth.bf16_bits(t["k"]), 0)
    _check_codes(out, ref, f"H{H} N{N}")


def _attention(out, v, want_lse=True):
    o, lse = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"],
                                  v[None].cuda().contiguous(), workspace=out["workspace"], want_lse=want_lse)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    return o[0].float().cpu().numpy(), (lse[0].cpu().numpy() if lse is not None else None)


@pytest.mark.parametrize("H,N", [(256, 32), (2, 700)])
def test_narrow_attention_within_tolerance(H, N):
    t = synth.toy_heads(H, seed=21, N=N)
    out = _gpu_quantize(t["q"], t["k"], 0)
    og, lg = _attention(out, t["v"])
    qh, kh = toy.prologue(synth.bf16_bits(t["q"]), synth.bf16_bits(t["k"]), 0)
    vb = synth.bf16_bits(t["v"])
    pad = lambda x: np.ascontiguousarray(np.pad(x, ((0, 0), (0, 64))))  # zero channels add nothing
    res = [oracle.attention_head(pad(qh[h]), pad(kh[h]), pad(vb[h]), 0.125) for h in range(H)]
    O = np.stack([r[0][:, :64] for r in res])
    L = np.stack([r[1] for r in res])
    assert_attention_close(og, O, f"d=64 H{H} N{N}")
    assert np.max(np.abs(lg - L)) < 1e-3 * max(1.0, np.abs(L).max())


def _lower(e, better, worse="plain"):
    d = e[worse] - e[better]
    return d.mean() > 4 * d.std(ddof=1) / np.sqrt(d.size)


@pytest.mark.parametrize("kw,better", [(dict(), "both"), (dict(n_scaled=0), "smooth K"),
                                       (dict(k_bias_std=0.0, scale_factor=10.0), "Hadamard")])
def test_toy_study_on_the_gpu(kw, better):
    """Per-head relative error of O against fp64 attention of the unquantised
    bf16 inputs, for each transform, with the GPU's codes and attention: the
    same conclusions as the oracle's study (the page's: both transforms beat
    plain FP4; each transform removes the error it targets)."""
    t = synth.toy_heads(256, seed=7 if not kw else 8, **kw)
    qb, kb, vb = (synth.bf16_bits(t[n]) for n in "qkv")
    ref = toy.attention(toy._bits_to_f32(qb), toy._bits_to_f32(kb), vb, bf16_p=False)
    e = {}
    for name, flags in FLAGS.items():
        og, _ = _attention(_gpu_quantize(t["q"], t["k"], flags), t["v"], want_lse=False)
        e[name] = np.linalg.norm(og - ref, axis=(1, 2)) / np.linalg.norm(ref, axis=(1, 2))
    oracle_e = toy.errors(qb, kb, vb)
    print(kw or "page's toy", {k: (round(float(e[k].mean()), 4), round(float(oracle_e[k].mean()), 4)) for k in e})
    assert _lower(e, better)
    for k in e:  # the GPU's bf16 O against the oracle's fp64 O: the same study within bf16 rounding
        assert abs(e[k].mean() - oracle_e[k].mean()) < 5e-3, k
