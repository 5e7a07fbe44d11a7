"""Shared helpers of the GPU parity tests: run the oracle and the CUDA path on
the same seeded inputs.  Oracle inputs and expected values never come from the
CUDA path; the CUDA path may be fed the oracle's codes to test attention on
its own."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from nvfp4_precision_b200 import synth

# Attention tolerance (absolute, on O), against the oracle's fp64 attention over
# the same dequantised Q and K.
MAX_ABS_TOL = 2e-2
MEAN_ABS_TOL = 2e-3


def fa():
    from nvfp4_precision_b200 import fp4attn
    return fp4attn


def oracle_prologue(d: dict, flags: int = 0, gq: float = 1.0, gk: float = 1.0) -> dict:
    return oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]), gq, gk, flags)


def gpu_prologue(d: dict, flags: int = 0, gq=None, gk=None) -> dict:
    q = d["q"].cuda()
    k = d["k"].cuda()
    gqt = None if gq is None else torch.tensor([gq], dtype=torch.float32, device="cuda")
    gkt = None if gk is None else torch.tensor([gk], dtype=torch.float32, device="cuda")
    out = fa().fp4attn_quantize_qk(q, k, gqt, gkt, flags=flags)
    status = fa().fp4attn_read_status(out["workspace"])
    res = {key: out[key].cpu().numpy() for key in ("q_codes", "q_scales", "k_codes", "k_scales", "k_mean")}
    res["status"] = status
    return res


def gpu_attention_from_codes(codes: dict, v: torch.Tensor, gq=None, gk=None, softmax_scale=0.0, want_lse=True):
    dev = "cuda"
    t = {key: torch.from_numpy(np.ascontiguousarray(codes[key])).to(dev)
         for key in ("q_codes", "q_scales", "k_codes", "k_scales")}
    gqt = None if gq is None else torch.tensor([gq], dtype=torch.float32, device=dev)
    gkt = None if gk is None else torch.tensor([gk], dtype=torch.float32, device=dev)
    B, H, N, _ = v.shape
    ws = fa().new_workspace(B, H, N)
    ws.zero_()
    o, lse = fa().fp4attn_forward(t["q_codes"], t["q_scales"], t["k_codes"], t["k_scales"], v.to(dev).contiguous(),
                                  gqt, gkt, softmax_scale=softmax_scale, want_lse=want_lse, workspace=ws)
    status = fa().fp4attn_read_status(ws)
    return o.float().cpu().numpy(), (lse.cpu().numpy() if lse is not None else None), status


def oracle_attention(codes: dict, v: torch.Tensor, rows=None, gq=1.0, gk=1.0, scale=None):
    return oracle.attention(codes["q_codes"], codes["q_scales"], codes["k_codes"], codes["k_scales"],
                            synth.bf16_bits(v), gq, gk, scale, rows)


def assert_attention_close(o_gpu: np.ndarray, o_ref: np.ndarray, what: str):
    diff = np.abs(o_gpu.astype(np.float64) - o_ref)
    mx, mean = float(diff.max()), float(diff.mean())
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, f"{what}: max|dO|={mx:.3e} mean|dO|={mean:.3e}"
    return mx, mean
