"""GPU parity at the largest supported sequence, N = 2^18 (the limit that keeps
the fixed-point key sum exact: |k| < 2^20 and N <= 2^18 give |sum| < 2^62).

* The prologue on two heads of 262144 rows, bit for bit against the oracle,
  including keys close to the range limit (a few channels near +-2^19), where
  the key sums reach 2^61.
* The attention on the same length, sampled rows against the oracle's fp64
  attention over all 262144 keys (max |dO| <= 2e-2, mean |dO| <= 2e-3)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import assert_attention_close, fa

pytestmark = pytest.mark.gpu

N_MAX = 262144
KEYS = ("q_codes", "q_scales", "k_codes", "k_scales", "k_mean")


def test_prologue_at_max_length_with_keys_near_the_range_limit():
    w = synth.custom("maxlen_pro", 1, 2, N_MAX, seed=77, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w, ("q", "k"))
    k = d["k"].clone()
    # channel 5 of head 0 at +(2^19 - 2^11) in every row (bf16-exact): its key
    # sum is 2^18 * (2^19 - 2^11) * 2^24, just under 2^61; channel 9 alternates sign
    k[0, 0, :, 5] = float(2 ** 19 - 2 ** 11)
    k[0, 0, ::2, 9] = -float(2 ** 19)
    k[0, 0, 1::2, 9] = float(2 ** 18)
    qb, kb = synth.bf16_bits(d["q"]), synth.bf16_bits(k)
    ref = oracle.quantize_qk(qb, kb)
    assert ref["status"] == oracle.OK
    out = fa().fp4attn_quantize_qk(d["q"].cuda(), k.cuda())
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    for key in KEYS:
        got = out[key].cpu().numpy()
        assert np.array_equal(got, ref[key]), f"{key} differs from the oracle"
    assert ref["k_mean"][0, 0, 5] == np.float32(2 ** 19 - 2 ** 11)
    assert ref["k_mean"][0, 0, 9] == np.float32((-(2 ** 19) + 2 ** 18) / 2)


def test_attention_at_max_length_sampled():
    w = synth.custom("maxlen_att", 1, 2, N_MAX, seed=78, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w)
    out = fa().fp4attn_quantize_qk(d["q"].cuda(), d["k"].cuda())
    o, lse = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], d["v"].cuda(),
                                  want_lse=True, workspace=out["workspace"])
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    rows = synth.sample_rows(N_MAX, 48, seed=w.seed)
    rows_t = torch.from_numpy(rows).cuda()
    vb = synth.bf16_bits(d["v"])
    ref = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]))
    for h in range(2):
        qh = oracle.dequant(ref["q_codes"][0, h], ref["q_scales"][0, h])
        kh = oracle.dequant(ref["k_codes"][0, h], ref["k_scales"][0, h])
        O, L = oracle.attention_head(qh, kh, vb[0, h], None, rows)
        og = o[0, h].index_select(0, rows_t).float().cpu().numpy()
        assert_attention_close(og[None, None], O[None, None], f"N=2^18 head {h}")
        lg = lse[0, h].index_select(0, rows_t).cpu().numpy()
        assert np.max(np.abs(lg - L)) < 1e-3 * max(1.0, np.abs(L).max())
