"""Parity at the full sizes of the 5-second and 15-second clip workloads
(B=1, H=48, N=36864 / 109568, d=128), through the same calls and launch
configuration that bench.py times: fp4attn_quantize_qk on all heads, then
fp4attn_forward on all heads.  The same step with Q, K, V and O in the
projection layout [B,N,H,128] must give the same bits.

The oracle cannot afford a whole attention at these sizes, so three heads are
checked: their NVFP4 codes and scales bit for bit against the oracle's
prologue of that head, and 64 sampled query rows per head (row 0, row N-1,
audio-tail rows where the workload has a tail, the rest uniform) against the
oracle's fp64 attention of those rows over all N keys, with the same
tolerance as the smaller cases (max |dO| <= 2e-2, mean |dO| <= 2e-3)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import assert_attention_close, fa

pytestmark = pytest.mark.gpu

HEADS = (0, 23, 47)
ROWS_PER_HEAD = 64


@pytest.mark.parametrize("name", ["clip5s", "clip15s"])
def test_full_size_product_path_sampled(name):
    w = synth.WORKLOADS[name]
    d = synth.generate(w)
    dev = torch.device("cuda")
    q, k, v = d["q"].to(dev), d["k"].to(dev), d["v"].to(dev)
    out = fa().fp4attn_quantize_qk(q, k)
    o_gpu, lse_gpu = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v,
                                          workspace=out["workspace"], want_lse=True)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    # the same step with Q, K, V and O in [B,N,H,128] (strided views): the same bits
    qt, kt, vt = (x.transpose(1, 2).contiguous().transpose(1, 2) for x in (q, k, v))
    del q, k
    out_t = fa().fp4attn_quantize_qk(qt, kt)
    ot = torch.empty((w.B, w.N, w.H, 128), dtype=torch.bfloat16, device=dev).transpose(1, 2)
    fa().fp4attn_forward(out_t["q_codes"], out_t["q_scales"], out_t["k_codes"], out_t["k_scales"], vt, o=ot,
                         workspace=out_t["workspace"])
    assert fa().fp4attn_read_status(out_t["workspace"]) == 0
    for key in ("q_codes", "q_scales", "k_codes", "k_scales"):
        assert torch.equal(out_t[key], out[key]), f"{name} [B,N,H,128]: {key}"
    assert torch.equal(ot, o_gpu), f"{name} [B,N,H,128]: O"
    del qt, kt, vt, ot, out_t
    rows = synth.sample_rows(w.N, ROWS_PER_HEAD, seed=w.seed, tail_rows=w.tail_rows,
                             n_tail=4 if w.tail_rows else 0)
    rows_t = torch.from_numpy(rows).to(dev)
    for h in HEADS:
        one = synth.generate(w, ("q", "k", "v"), heads=[h])
        ref = oracle.quantize_qk(synth.bf16_bits(one["q"]), synth.bf16_bits(one["k"]))
        assert ref["status"] == 0
        for key in ("q_codes", "q_scales", "k_codes", "k_scales"):
            got = out[key][0, h].cpu().numpy()
            assert np.array_equal(got, ref[key][0, 0]), f"{name} head {h}: {key} differs from the oracle"
        O, L = oracle.attention(ref["q_codes"], ref["q_scales"], ref["k_codes"], ref["k_scales"],
                                synth.bf16_bits(one["v"]), rows=rows)
        og = o_gpu[0, h].index_select(0, rows_t).float().cpu().numpy()[None, None]
        assert_attention_close(og, O, f"{name} head {h}")
        lg = lse_gpu[0, h].index_select(0, rows_t).cpu().numpy()
        assert np.max(np.abs(lg - L[0, 0])) < 1e-3 * max(1.0, np.abs(L).max()), f"{name} head {h}: lse"
