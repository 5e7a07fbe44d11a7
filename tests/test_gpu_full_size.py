"""Parity at the full sizes of the 5-second and 15-second clip workloads
(B=1, H=48, N=36864 / 109568, d=128), through the same calls and launch
configuration that bench.py times: fp4attn_quantize_qk on all heads, then
fp4attn_forward on all heads.  The same step with Q, K, V and O in the
projection layout [B,N,H,128] must give the same bits.

Every head is checked.  The NVFP4 codes, scales and key means of all 48 heads
are compared bit for bit with the oracle's prologue of the whole tensor.  The
oracle cannot afford a whole attention at these sizes, so each head gets its
own seeded sample of query rows (row 0, row N-1, four audio-tail rows where
the workload has a tail, the rest uniform), each against the oracle's fp64
attention of that row over all N keys, with the same tolerance as the smaller
cases (max |dO| <= 2e-2, mean |dO| <= 2e-3) and the log-sum-exp to 1e-3
relative."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import assert_attention_close, fa

pytestmark = pytest.mark.gpu

ROWS_PER_HEAD = 48


@pytest.mark.parametrize("name", ["clip5s", "clip15s"])
def test_full_size_product_path_every_head(name):
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
    del q, k, v
    out_t = fa().fp4attn_quantize_qk(qt, kt)
    ot = torch.empty((w.B, w.N, w.H, 128), dtype=torch.bfloat16, device=dev).transpose(1, 2)
    fa().fp4attn_forward(out_t["q_codes"], out_t["q_scales"], out_t["k_codes"], out_t["k_scales"], vt, o=ot,
                         workspace=out_t["workspace"])
    assert fa().fp4attn_read_status(out_t["workspace"]) == 0
    for key in ("q_codes", "q_scales", "k_codes", "k_scales"):
        assert torch.equal(out_t[key], out[key]), f"{name} [B,N,H,128]: {key}"
    assert torch.equal(ot, o_gpu), f"{name} [B,N,H,128]: O"
    del qt, kt, vt, ot, out_t

    # the oracle's prologue of the whole tensor: every head's codes bit for bit
    q_bits, k_bits, v_bits = (synth.bf16_bits(d[t]) for t in ("q", "k", "v"))
    del d
    ref = oracle.quantize_qk(q_bits, k_bits)
    del q_bits, k_bits
    assert ref["status"] == 0
    for key in ("q_codes", "q_scales", "k_codes", "k_scales", "k_mean"):
        got = out[key].cpu().numpy()
        if not np.array_equal(got, ref[key]):
            bad = np.argwhere(got != ref[key])
            raise AssertionError(f"{name}: {key} differs from the oracle at {bad.shape[0]} places, "
                                 f"first {bad[:3].tolist()}")

    # every head's attention on its own row sample
    worst = (0.0, 0.0)
    for h in range(w.H):
        rows = synth.sample_rows(w.N, ROWS_PER_HEAD, seed=w.seed * 1000 + h, tail_rows=w.tail_rows,
                                 n_tail=4 if w.tail_rows else 0)
        rows_t = torch.from_numpy(rows).to(dev)
        O, L = oracle.attention(ref["q_codes"][:, h:h + 1], ref["q_scales"][:, h:h + 1],
                                ref["k_codes"][:, h:h + 1], ref["k_scales"][:, h:h + 1],
                                v_bits[:, h:h + 1], rows=rows)
        og = o_gpu[0, h].index_select(0, rows_t).float().cpu().numpy()[None, None]
        mx, mean = assert_attention_close(og, O, f"{name} head {h}")
        worst = (max(worst[0], mx), max(worst[1], mean))
        lg = lse_gpu[0, h].index_select(0, rows_t).cpu().numpy()
        assert np.max(np.abs(lg - L[0, 0])) < 1e-3 * max(1.0, np.abs(L).max()), f"{name} head {h}: lse"
    print(f"{name}: {w.H} heads x {ROWS_PER_HEAD} rows, worst max|dO|={worst[0]:.3e} mean|dO|={worst[1]:.3e}")
