"""GPU parity of the general forms of the path: Q, K, V and O in any strides
(the [B,N,H,128] layout a QKV projection writes, padded rows), and the dynamic
per-tensor global scale g = fl32(amax / (6*448)) of the transformed Q and K
(FastVideo "Pika H3 Flex in FastVideo", sections "NVFP4 QAD" and "FP4
attention").  Codes, scales and g are compared bit for bit with the oracle on
the contiguous copies; O with the attention tolerance (max |dO| <= 2e-2,
mean |dO| <= 2e-3)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import assert_attention_close, fa

pytestmark = pytest.mark.gpu

CODE_KEYS = ("q_codes", "q_scales", "k_codes", "k_scales", "k_mean")


def _bnhd(t: torch.Tensor) -> torch.Tensor:
    """A [B,H,N,128] view of a new contiguous [B,N,H,128] copy of t on the GPU."""
    return t.transpose(1, 2).contiguous().cuda().transpose(1, 2)


def _padded(t: torch.Tensor, pad: int = 8) -> torch.Tensor:
    """A [B,H,N,128] view whose rows are 128 + pad elements apart."""
    B, H, N, D = t.shape
    buf = torch.full((B, H, N, D + pad), float("nan"), dtype=t.dtype, device="cuda")
    buf[..., :D] = t.cuda()
    return buf[..., :D]


def _assert_codes_equal(out, ref, what):
    for key in CODE_KEYS:
        got = out[key].cpu().numpy()
        if not np.array_equal(got, ref[key]):
            bad = np.argwhere(got != ref[key])
            raise AssertionError(f"{what}: {key} differs at {bad.shape[0]} places, first {bad[:3].tolist()}")


def _data(B, H, N, seed, **kw):
    return synth.generate(synth.custom(f"gen{seed}", B, H, N, seed=seed, **kw))


@pytest.mark.parametrize("layout", ["bnhd", "padded"])
@pytest.mark.parametrize("B,H,N", [(2, 3, 300), (1, 4, 1000), (1, 1, 1)])
def test_strided_prologue_bit_exact(layout, B, H, N):
    d = _data(B, H, N, seed=300 + N, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    view = _bnhd if layout == "bnhd" else _padded
    q, k = view(d["q"]), view(d["k"])
    if H > 1 and N > 1:
        assert not q.is_contiguous()
    out = fa().fp4attn_quantize_qk(q, k)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    ref = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]))
    _assert_codes_equal(out, ref, f"{layout} B{B} H{H} N{N}")


@pytest.mark.parametrize("B,H,N", [(2, 3, 300), (1, 2, 1000)])
def test_strided_forward_writes_bnhd_output(B, H, N):
    """V read and O written in [B,N,H,128] with one spare head slot per row that
    must stay untouched."""
    d = _data(B, H, N, seed=400 + N, k_offset_std=2.0)
    out = fa().fp4attn_quantize_qk(d["q"].cuda(), d["k"].cuda())
    v = _bnhd(d["v"])
    buf = torch.full((B, N, H + 1, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    o_view = buf[:, :, :H].transpose(1, 2)
    o, lse = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v,
                                  o=o_view, want_lse=True, workspace=out["workspace"])
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    assert o.data_ptr() == buf.data_ptr()
    assert torch.all(buf[:, :, H] == 7.0), "the spare head slot was written"
    ref = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]))
    O, L = oracle.attention(ref["q_codes"], ref["q_scales"], ref["k_codes"], ref["k_scales"], synth.bf16_bits(d["v"]))
    assert_attention_close(o.float().cpu().numpy(), O, f"strided forward B{B} H{H} N{N}")
    assert np.max(np.abs(lse.cpu().numpy() - L)) < 1e-3 * max(1.0, np.abs(L).max())


def test_strided_forward_matches_contiguous_bit_for_bit():
    """The layout changes only the addresses: the same inputs in [B,N,H,128]
    and [B,H,N,128] give the same O bits."""
    d = _data(1, 3, 777, seed=33, k_offset_std=2.0)
    out = fa().fp4attn_quantize_qk(d["q"].cuda(), d["k"].cuda())
    args = (out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"])
    o1, _ = fa().fp4attn_forward(*args, d["v"].cuda(), workspace=out["workspace"])
    o2, _ = fa().fp4attn_forward(*args, _padded(d["v"], 24), workspace=out["workspace"])
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("N", [129, 1000])
def test_bf16qk_strided(N):
    d = _data(2, 2, N, seed=500 + N, k_offset_std=2.0)
    B, H = 2, 2
    q, k, v = _bnhd(d["q"]), _padded(d["k"]), _bnhd(d["v"])
    buf = torch.full((B, N, H, 136), 3.0, dtype=torch.bfloat16, device="cuda")
    o_view = buf[..., :128].transpose(1, 2)
    o, _ = fa().fp4attn_forward_bf16qk(q, k, v, o=o_view)
    assert torch.all(buf[..., 128:] == 3.0), "the row padding was written"
    qf, kf, vb = d["q"].float().numpy(), d["k"].float().numpy(), synth.bf16_bits(d["v"])
    og = o.float().cpu().numpy()
    for b in range(B):
        for h in range(H):
            O, _ = oracle.attention_head(qf[b, h], kf[b, h], vb[b, h])
            assert_attention_close(og[b, h][None, None], O[None, None], f"bf16qk strided N{N} b{b} h{h}")


# ---------------------------------------------------------------- dynamic g --

@pytest.mark.parametrize("flags", [0, 1, 2, 3])
def test_dynamic_gscale_bit_exact(flags):
    d = _data(2, 3, 700, seed=600 + flags, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    qb, kb = synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"])
    ref = oracle.quantize_qk(qb, kb, flags=flags, dynamic=True)
    assert ref["status"] == oracle.OK
    out = fa().fp4attn_quantize_qk(_bnhd(d["q"]), d["k"].cuda(), flags=flags, dynamic_gscale=True)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    gq, gk = out["q_gscale"].item(), out["k_gscale"].item()
    assert np.float32(gq) == ref["gq"] and np.float32(gk) == ref["gk"], (gq, gk, ref["gq"], ref["gk"])
    _assert_codes_equal(out, ref, f"dynamic flags {flags}")
    o, _ = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], d["v"].cuda(),
                                out["q_gscale"], out["k_gscale"], workspace=out["workspace"])
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    O, _ = oracle.attention(ref["q_codes"], ref["q_scales"], ref["k_codes"], ref["k_scales"], synth.bf16_bits(d["v"]),
                            float(ref["gq"]), float(ref["gk"]))
    assert_attention_close(o.float().cpu().numpy(), O, f"dynamic attention flags {flags}")


def test_dynamic_gscale_beyond_the_unit_scale_range():
    """Keys with magnitudes in the thousands: the unit scale saturates, the
    dynamic one matches the oracle bit for bit."""
    d = _data(1, 2, 500, seed=71, k_offset_std=2.0)
    d["k"] = (d["k"].float() * 2048.0).to(torch.bfloat16)
    qb, kb = synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"])
    ref = oracle.quantize_qk(qb, kb, flags=oracle.NO_SMOOTH_K, dynamic=True)
    assert ref["gk"] > 1.0
    out = fa().fp4attn_quantize_qk(d["q"].cuda(), d["k"].cuda(), flags=oracle.NO_SMOOTH_K, dynamic_gscale=True)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    assert np.float32(out["k_gscale"].item()) == ref["gk"]
    _assert_codes_equal(out, ref, "dynamic large keys")


def test_dynamic_gscale_zero_and_empty_tensors():
    g_min = np.float32(2.0 ** -64)
    z = torch.zeros((1, 2, 130, 128), dtype=torch.bfloat16, device="cuda")
    out = fa().fp4attn_quantize_qk(z, z, dynamic_gscale=True)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    assert np.float32(out["q_gscale"].item()) == g_min and np.float32(out["k_gscale"].item()) == g_min
    assert not out["q_scales"].any() and not out["k_scales"].any()
    assert not (out["q_codes"] & 0x77).any() and not (out["k_codes"] & 0x77).any()
    e = torch.zeros((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    gq = torch.full((1,), 5.0, device="cuda")
    gk = torch.full((1,), 5.0, device="cuda")
    fa().fp4attn_quantize_qk(e, e, gq, gk, dynamic_gscale=True)
    assert np.float32(gq.item()) == g_min and np.float32(gk.item()) == g_min


def test_dynamic_gscale_full_size_sampled_heads():
    """The 15-second clip (B1 H48 N109568) in [B,N,H,128]: g of each tensor
    (over all 48 heads) bit for bit, and the codes of heads 0 and 47."""
    w = synth.WORKLOADS["clip15s"]
    d = synth.generate(w, ("q", "k"))
    qb, kb = synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"])
    gq, gk, st = oracle.dynamic_gscale(qb, kb)
    assert st == oracle.OK
    out = fa().fp4attn_quantize_qk(_bnhd(d["q"]), _bnhd(d["k"]), dynamic_gscale=True)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    assert np.float32(out["q_gscale"].item()) == gq and np.float32(out["k_gscale"].item()) == gk
    for h in (0, 47):
        ref = oracle.quantize_qk(qb[:, h:h + 1], kb[:, h:h + 1], float(gq), float(gk))
        for key in CODE_KEYS:
            got = out[key][:, h:h + 1].cpu().numpy()
            assert np.array_equal(got, ref[key]), f"head {h}: {key}"
