"""GPU parity of the BF16-QK attention (fp4attn_forward_bf16qk), the BF16
counterpart of the FP4 kernel: compared with the oracle's fp64 attention of
the same bf16 Q, K and V (no smoothing, rotation or quantisation on either
side), with the FP4 kernel's tolerance (max |dO| <= 2e-2, mean |dO| <= 2e-3;
the GPU rounds S to fp32, P to bf16 and O to bf16)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import assert_attention_close, fa

pytestmark = pytest.mark.gpu


def _oracle(d, rows=None, scale=None, heads=None):
    B, H, N, _ = d["q"].shape
    heads = range(H) if heads is None else heads
    q = d["q"].float().numpy()
    k = d["k"].float().numpy()
    vb = synth.bf16_bits(d["v"])
    R = N if rows is None else len(rows)
    O = np.empty((B, len(heads), R, 128))
    L = np.empty((B, len(heads), R))
    for b in range(B):
        for j, h in enumerate(heads):
            O[b, j], L[b, j] = oracle.attention_head(q[b, h], k[b, h], vb[b, h], scale, rows)
    return O, L


def _gpu(d, scale=0.0):
    q, k, v = (d[t].cuda() for t in "qkv")
    B, H, N, _ = v.shape
    ws = fa().new_workspace(B, H, N)
    ws.zero_()
    o, lse = fa().fp4attn_forward_bf16qk(q, k, v, softmax_scale=scale, want_lse=True, workspace=ws)
    assert fa().fp4attn_read_status(ws) == 0
    return o, lse


def _check(name, d, rows=None, scale=0.0):
    o, lse = _gpu(d, scale)
    O, L = _oracle(d, rows, None if scale == 0.0 else scale)
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    if rows is not None:
        og, lg = og[:, :, rows], lg[:, :, rows]
    assert_attention_close(og, O, name)
    assert np.max(np.abs(lg - L)) < 1e-3 * max(1.0, np.abs(L).max()), f"{name}: lse"


def test_bf16qk_tiny_full():
    _check("bf16qk tiny", synth.generate(synth.WORKLOADS["tiny"]))


@pytest.mark.parametrize("N", [1, 77, 128, 129, 300, 1000])
def test_bf16qk_ragged_lengths(N):
    d = synth.generate(synth.custom(f"bf16qk_ragged{N}", 1, 2, N, seed=60 + N, k_offset_std=2.0))
    _check(f"bf16qk ragged {N}", d)


def test_bf16qk_softmax_scale_with_outliers():
    d = synth.generate(synth.custom("bf16qk_scale", 1, 2, 640, seed=9, k_offset_std=2.0, n_outliers=2,
                                    outlier_factor=20.0))
    _check("bf16qk scale", d, scale=0.05)


def test_bf16qk_mid_sampled():
    w = synth.WORKLOADS["mid"]
    _check("bf16qk mid", synth.generate(w), rows=synth.sample_rows(w.N, 256, seed=w.seed))


def test_bf16qk_full_size_sampled():
    """15-second clip (B1 H48 N109568): all heads on the GPU, heads 0 and 47 on
    64 sampled rows against the oracle."""
    w = synth.WORKLOADS["clip15s"]
    d = synth.generate(w)
    o, lse = _gpu(d)
    rows = synth.sample_rows(w.N, 64, seed=w.seed)
    rows_t = torch.from_numpy(rows).cuda()
    for h in (0, 47):
        one = synth.generate(w, ("q", "k", "v"), heads=[h])
        O, L = _oracle(one, rows)
        og = o[0, h].index_select(0, rows_t).float().cpu().numpy()[None, None]
        assert_attention_close(og, O, f"bf16qk clip15s head {h}")
        lg = lse[0, h].index_select(0, rows_t).cpu().numpy()
        assert np.max(np.abs(lg - L[0, 0])) < 1e-3 * max(1.0, np.abs(L).max()), f"head {h}: lse"
