"""GPU parity on the method's degenerate cases (FastVideo "Pika H3 Flex in
FastVideo", section "FP4 attention"):

* every key of a head identical: smoothing K leaves zeros, every score is 0
  and each output row is the mean of V (uniform attention);
* Q = 0: again uniform attention, whatever K is;
* V constant: O is that constant for any scores;
* empty shapes through the strided, dynamic-scale and backward entry points.

Each case is also compared with the oracle where it applies."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import assert_attention_close, fa

pytestmark = pytest.mark.gpu


def _run(q, k, v, **kw):
    out = fa().fp4attn_quantize_qk(q.cuda(), k.cuda(), **kw)
    o, lse = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v.cuda(),
                                  out.get("q_gscale"), out.get("k_gscale"), want_lse=True, workspace=out["workspace"])
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    return out, o.float().cpu().numpy(), lse.cpu().numpy()


def _vbar(v):
    return v.double().mean(dim=2, keepdim=True).numpy()


def test_identical_keys_give_uniform_attention():
    d = synth.generate(synth.custom("same_k", 1, 2, 700, seed=3))
    k = d["k"][:, :, :1].expand(-1, -1, 700, -1).contiguous()
    out, o, lse = _run(d["q"], k, d["v"])
    assert not out["k_codes"].any() or not (out["k_codes"] & 0x77).any()  # smoothed keys are all zero
    vbar = np.broadcast_to(_vbar(d["v"]), o.shape)
    assert_attention_close(o, vbar, "identical keys")
    assert np.allclose(lse, np.log(700.0), atol=1e-4)


@pytest.mark.parametrize("dynamic", [False, True])
def test_zero_queries_give_uniform_attention(dynamic):
    d = synth.generate(synth.custom("zero_q", 1, 2, 513, seed=4, k_offset_std=2.0, n_outliers=2,
                                    outlier_factor=20.0))
    q = torch.zeros_like(d["q"])
    out, o, lse = _run(q, d["k"], d["v"], dynamic_gscale=dynamic)
    assert_attention_close(o, np.broadcast_to(_vbar(d["v"]), o.shape), "zero queries")
    assert np.allclose(lse, np.log(513.0), atol=1e-4)


def test_constant_values_give_constant_output():
    d = synth.generate(synth.custom("const_v", 1, 2, 300, seed=5, k_offset_std=2.0, n_outliers=2,
                                    outlier_factor=20.0))
    v = torch.full_like(d["v"], 0.75)
    out, o, _ = _run(d["q"], d["k"], v)
    # O = 0.75 * sum(bf16(p)) / sum(p): within 2^-9 relative of 0.75 before the
    # final bf16 rounding, so at most one bf16 step (2^-8 at 0.75) away
    assert np.abs(o - 0.75).max() <= 2.0 ** -8
    ref = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]))
    O, _ = oracle.attention(ref["q_codes"], ref["q_scales"], ref["k_codes"], ref["k_scales"], synth.bf16_bits(v))
    assert_attention_close(o, O, "constant V")


def test_empty_shapes_through_the_general_entry_points():
    dev = "cuda"
    for B, H, N in ((1, 2, 0), (0, 2, 64), (1, 0, 64)):
        q = torch.zeros((B, N, H, 128), dtype=torch.bfloat16, device=dev).transpose(1, 2)
        out = fa().fp4attn_quantize_qk(q, q, dynamic_gscale=True)
        assert fa().fp4attn_read_status(out["workspace"]) == 0
        assert float(out["q_gscale"].item()) == 2.0 ** -64
        o, _ = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], q,
                                    workspace=out["workspace"])
        assert o.shape == (B, H, N, 128)
        ob, _ = fa().fp4attn_forward_bf16qk(q, q, q)
        assert ob.shape == (B, H, N, 128)
        z = torch.zeros((B, H, N, 128), dtype=torch.bfloat16, device=dev)
        lse = torch.zeros((B, H, N), dtype=torch.float32, device=dev)
        dq, dk, dv, ws = fa().fp4attn_backward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"],
                                               z, z, z, lse)
        assert fa().fp4attn_read_status(ws) == 0 and dq.shape == z.shape
        assert fa().fp4attn_dequant_bf16(out["q_codes"], out["q_scales"]).shape == (B, H, N, 128)
