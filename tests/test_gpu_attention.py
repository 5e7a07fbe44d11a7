"""GPU parity of the FP4 attention kernel and its tcgen05 building blocks.

Attention is compared element by element with the oracle's fp64 attention over
the same dequantised Q and K: max |dO| <= 2e-2 and mean |dO| <= 2e-3 (bf16 O).
The block-scaled QK^T tile is compared with fp64 dot products of the oracle's
dequantised values (exact products, fp32 accumulation: relative 1e-5)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import (assert_attention_close, fa, gpu_attention_from_codes, gpu_prologue,
                         oracle_attention, oracle_prologue)

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_not_hung():
    assert fa().fp4attn_probe_wait_timeout(2_000_000) == fa().ERR_TIMEOUT  # 2 ms limit


def _codes_for(name, B, H, N, seed, **kw):
    d = synth.generate(synth.custom(name, B, H, N, seed=seed, **kw), ("q", "k", "v"))
    return d, oracle_prologue(d)


def test_qk_tile_block_scaled_mma():
    d, o = _codes_for("qk", 1, 1, 256, 21, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    qh = oracle.dequant(o["q_codes"][0, 0], o["q_scales"][0, 0]).astype(np.float64)
    kh = oracle.dequant(o["k_codes"][0, 0], o["k_scales"][0, 0]).astype(np.float64)
    for qi, ki in [(0, 0), (128, 0), (0, 128)]:
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        s = fa().fp4attn_probe_qk_tile(t(o["q_codes"][0, 0, qi:qi + 128]), t(o["q_scales"][0, 0, qi:qi + 128]),
                                       t(o["k_codes"][0, 0, ki:ki + 128]), t(o["k_scales"][0, 0, ki:ki + 128]))
        want = qh[qi:qi + 128] @ kh[ki:ki + 128].T
        got = s.cpu().numpy().astype(np.float64)
        err = np.abs(got - want) / (np.abs(qh[qi:qi + 128]) @ np.abs(kh[ki:ki + 128]).T + 1e-30)
        assert err.max() < 1e-5, f"tile ({qi},{ki}): max rel err {err.max():.3e}"


def test_pv_tile_bf16_mma_from_tmem():
    g = torch.Generator().manual_seed(5)
    p = torch.rand((128, 128), generator=g).to(torch.bfloat16)
    v = torch.randn((128, 128), generator=g).to(torch.bfloat16)
    o = fa().fp4attn_probe_pv_tile(p.cuda(), v.cuda()).cpu().double()
    want = p.double() @ v.double()
    assert (o - want).abs().max().item() < 1e-3


def _attention_case(name, B, H, N, seed, rows=None, gq=None, gk=None, scale=0.0, **kw):
    d, o = _codes_for(name, B, H, N, seed, **kw)
    og, lse_g, st = gpu_attention_from_codes(o, d["v"], gq=gq, gk=gk, softmax_scale=scale)
    assert st == 0, f"{name}: device status {st}"
    O, L = oracle_attention(o, d["v"], rows=rows, gq=1.0 if gq is None else gq, gk=1.0 if gk is None else gk,
                            scale=None if scale == 0.0 else scale)
    if rows is not None:
        og = og[:, :, rows]
        lse_g = lse_g[:, :, rows]
    assert_attention_close(og, O, name)
    assert np.max(np.abs(lse_g - L)) < 1e-3 * max(1.0, np.abs(L).max()), f"{name}: lse"


def test_attention_tiny_full():
    d = synth.generate(synth.WORKLOADS["tiny"])
    o = oracle_prologue(d)
    og, lse_g, st = gpu_attention_from_codes(o, d["v"])
    assert st == 0
    O, L = oracle_attention(o, d["v"])
    assert_attention_close(og, O, "tiny")
    assert np.max(np.abs(lse_g - L)) < 1e-3 * max(1.0, np.abs(L).max())


@pytest.mark.parametrize("N", [1, 77, 128, 129, 300, 1000])
def test_attention_ragged_lengths(N):
    _attention_case(f"ragged{N}", 1, 2, N, 40 + N, k_offset_std=2.0)


def test_attention_global_and_softmax_scales():
    _attention_case("scales", 1, 2, 640, 7, gq=0.5, gk=3.0, scale=0.05, k_offset_std=2.0,
                    n_outliers=2, outlier_factor=20.0)


def test_attention_mid_every_row():
    """Every query row of every head of the mid workload (B1 H8 N8192, two
    outlier channels) against the oracle's fp64 attention of all rows."""
    w = synth.WORKLOADS["mid"]
    d = synth.generate(w)
    o = oracle_prologue(d)
    og, lse_g, st = gpu_attention_from_codes(o, d["v"])
    assert st == 0
    v_bits = synth.bf16_bits(d["v"])
    for h in range(w.H):
        qh = oracle.dequant(o["q_codes"][0, h], o["q_scales"][0, h])
        kh = oracle.dequant(o["k_codes"][0, h], o["k_scales"][0, h])
        O, L = oracle.attention_all_rows(qh, kh, v_bits[0, h])
        assert_attention_close(og[0, h][None, None], O[None, None], f"mid head {h}")
        assert np.max(np.abs(lse_g[0, h] - L)) < 1e-3 * max(1.0, np.abs(L).max()), f"mid head {h}: lse"


def test_end_to_end_prologue_then_attention_tiny():
    """The product path: GPU prologue output feeds GPU attention."""
    d = synth.generate(synth.WORKLOADS["tiny"])
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    out = fa().fp4attn_quantize_qk(q, k)
    o, _ = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v,
                                workspace=out["workspace"])
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    ref = oracle_prologue(d)
    O, _ = oracle_attention(ref, d["v"])
    assert_attention_close(o.float().cpu().numpy(), O, "tiny end to end")
