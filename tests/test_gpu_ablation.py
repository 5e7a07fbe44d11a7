"""Ablation of the two transforms (FastVideo "Pika H3 Flex in FastVideo",
section "FP4 attention": smoothing K and rotating Q and K by a Hadamard
matrix lower the error of FP4 attention; the page's per-layer errors fall from
plain FP4 to FP4 with both transforms).

For each synthetic distribution the GPU runs the product path with each
combination of transforms (the prologue's NO_SMOOTH_K / NO_HADAMARD flags) and
with BF16 Q and K; the error of O is measured against the oracle's fp64
attention of the unquantised bf16 Q, K and V on sampled rows (relative
Frobenius norm, averaged over heads).  The test checks the page's
qualitative claim -- on biased or outlier-heavy keys both transforms together
beat plain FP4 -- and that each transform removes the error it targets
(smoothing for a per-channel key bias, the rotation for outlier channels).
Run with -s to see the table."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import fa

pytestmark = pytest.mark.gpu

CASES = (
    ("N(0,1)", dict(seed=100)),
    ("key bias std 2", dict(seed=101, k_offset_std=2.0)),
    ("2 channels x20", dict(seed=102, n_outliers=2, outlier_factor=20.0)),
    ("bias + 2 channels x20", dict(seed=103, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)),
)
LABELS = ("plain", "smooth K", "Hadamard", "both")
FLAGS = {"plain": 3, "smooth K": 2, "Hadamard": 1, "both": 0}  # NO_SMOOTH_K = 1, NO_HADAMARD = 2


def _errors(w, rows):
    d = synth.generate(w)
    q, k, v = (d[t].cuda() for t in "qkv")
    qf, kf, vb = d["q"].float().numpy(), d["k"].float().numpy(), synth.bf16_bits(d["v"])
    exact = [oracle.attention_head(qf[0, h], kf[0, h], vb[0, h], None, rows)[0] for h in range(w.H)]

    def rel(o):
        og = o.float().cpu().numpy()
        return float(np.mean([np.linalg.norm(og[0, h, rows] - exact[h]) / np.linalg.norm(exact[h])
                              for h in range(w.H)]))

    err = {}
    for label in LABELS:
        out = fa().fp4attn_quantize_qk(q, k, flags=FLAGS[label])
        o, _ = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v,
                                    workspace=out["workspace"])
        assert fa().fp4attn_read_status(out["workspace"]) == 0
        err[label] = rel(o)
    o, _ = fa().fp4attn_forward_bf16qk(q, k, v)
    err["BF16 QK"] = rel(o)
    return err


def test_transforms_lower_fp4_attention_error():
    table = {}
    for name, kw in CASES:
        w = synth.custom("ablation", 1, 4, 4096, **kw)
        table[name] = _errors(w, synth.sample_rows(w.N, 256, seed=w.seed))
    cols = LABELS + ("BF16 QK",)
    print("\n| keys | " + " | ".join(cols) + " |\n|---|" + "---|" * len(cols))
    for name, err in table.items():
        print(f"| {name} | " + " | ".join(f"{err[c]:.4f}" for c in cols) + " |")
    # BF16 QK is far more accurate than any FP4 variant
    for err in table.values():
        assert err["BF16 QK"] < 0.2 * min(err[label] for label in LABELS)
    # the page's claim: both transforms beat plain FP4 on biased / outlier keys
    for name in ("key bias std 2", "2 channels x20", "bias + 2 channels x20"):
        assert table[name]["both"] < 0.8 * table[name]["plain"], name
    # each transform removes the error it targets
    assert table["key bias std 2"]["smooth K"] < 0.8 * table["key bias std 2"]["plain"]
    assert table["2 channels x20"]["Hadamard"] < 0.9 * table["2 channels x20"]["plain"]
    # on unstructured keys the transforms change nothing material
    e = table["N(0,1)"]
    assert max(e[label] for label in LABELS) < 1.1 * min(e[label] for label in LABELS)
