"""Parity of the training-time backward at the full size of the 15-second clip
workload (B=1, H=48, N=109568, d=128), through the call and launch
configuration that bench.py times: fp4attn_backward over all 48 heads.

Head 0 gets the oracle's inputs, as in the kernel-parity tests of the smaller
cases: its NVFP4 codes (checked bit for bit against the GPU prologue first),
the oracle's exact forward output rounded to bf16 and its lse.  The other 47
heads run on the GPU forward's O and lse.  The oracle then computes 64 sampled
query rows (dq) and 64 sampled key rows (dk, dv, including the first and last
keys of key tiles) of head 0 over all N keys and queries, and the GPU must
match them with the kernel-parity bound (max |d| <= 2e-2 max |ref|,
||d||_F <= 1e-2 ||ref||_F over the sampled rows).

Two properties that hold at any size are checked on every head:
* the centring: each column of dk sums to zero, up to the bf16 rounding of dk
  (at most 2^-9 of each element) and fp32 sums: |sum_j dk_jc| <= 2^-8 sum_j |dk_jc|;
* the rows of P sum to one, so each column of dv sums to that of dO, up to the
  bf16 rounding of P (2^-9) and of dv: |sum_j dv_jc - sum_i dO_ic| <=
  2^-8 (sum_i |dO_ic| + sum_j |dv_jc|)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import fa

pytestmark = pytest.mark.gpu

TIGHT = (2e-2, 1e-2)


def _assert_close(g, r, what):
    assert np.isfinite(g).all(), f"{what}: non-finite"
    d = np.abs(g.astype(np.float64) - r)
    mx, ref = float(d.max()), float(np.abs(r).max())
    fro = float(np.linalg.norm(d) / np.linalg.norm(r))
    print(f"{what}: max|d| {mx:.3e} (ref max {ref:.3e}), fro rel {fro:.3e}")
    assert mx <= TIGHT[0] * ref and fro <= TIGHT[1], f"{what}: max|d|={mx:.3e} ref={ref:.3e} fro={fro:.3e}"


def test_full_size_backward_sampled():
    w = synth.WORKLOADS["clip15s"]
    N = w.N
    d = synth.generate(w)
    dev = torch.device("cuda")
    v = d["v"].to(dev)
    out = fa().fp4attn_quantize_qk(d["q"].to(dev), d["k"].to(dev))
    o, lse = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v,
                                  workspace=out["workspace"], want_lse=True)
    assert fa().fp4attn_read_status(out["workspace"]) == 0

    # head 0: the oracle's codes, exact forward (O rounded to bf16) and lse
    ref = oracle.quantize_qk(synth.bf16_bits(d["q"][:, :1]), synth.bf16_bits(d["k"][:, :1]))
    assert ref["status"] == 0
    for key in ("q_codes", "q_scales", "k_codes", "k_scales"):
        assert np.array_equal(out[key][0, 0].cpu().numpy(), ref[key][0, 0]), f"head 0: {key}"
        out[key][0, 0] = torch.from_numpy(ref[key][0, 0]).to(dev)
    qh = oracle.dequant(ref["q_codes"][0, 0], ref["q_scales"][0, 0])
    kh = oracle.dequant(ref["k_codes"][0, 0], ref["k_scales"][0, 0])
    vb = synth.bf16_bits(d["v"][0, 0])
    O_exact, L = oracle.attention_all_rows(qh, kh, vb)
    o_bf = torch.from_numpy(O_exact.astype(np.float32)).to(torch.bfloat16)
    o[0, 0] = o_bf.to(dev)
    lse[0, 0] = torch.from_numpy(L.astype(np.float32)).to(dev)

    gen = torch.Generator(device=dev).manual_seed(17)
    dO = torch.randn((1, w.H, N, 128), generator=gen, device=dev).to(torch.bfloat16)
    dO0 = torch.randn((N, 128), generator=torch.Generator().manual_seed(18)).to(torch.bfloat16)
    dO[0, 0] = dO0.to(dev)

    dq, dk, dv, ws = fa().fp4attn_backward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v, o,
                                           dO, lse)
    assert fa().fp4attn_read_status(ws) == 0

    I = synth.sample_rows(N, 64, seed=w.seed + 11)
    J = np.union1d(synth.sample_rows(N, 60, seed=w.seed + 12), [127, 128, N - 129, N - 128])
    rq, rk, rv = oracle.attention_backward_rows(qh, kh, vb, dO0.double().numpy(), o_bf.double().numpy(), O_exact,
                                                L, I, J)
    It, Jt = torch.from_numpy(I).to(dev), torch.from_numpy(J).to(dev)
    _assert_close(dq[0, 0].index_select(0, It).float().cpu().numpy(), rq, "clip15s head 0 dq")
    _assert_close(dk[0, 0].index_select(0, Jt).float().cpu().numpy(), rk, "clip15s head 0 dk")
    _assert_close(dv[0, 0].index_select(0, Jt).float().cpu().numpy(), rv, "clip15s head 0 dv")

    # properties on every head
    dk64, dv64, do64 = dk.double(), dv.double(), dO.double()
    col = dk64.sum(dim=2).abs()
    assert bool((col <= 2.0 ** -8 * dk64.abs().sum(dim=2)).all()), "dk columns do not sum to zero"
    gap = (dv64.sum(dim=2) - do64.sum(dim=2)).abs()
    assert bool((gap <= 2.0 ** -8 * (do64.abs().sum(dim=2) + dv64.abs().sum(dim=2))).all()), \
        "dv column sums differ from those of dO"
