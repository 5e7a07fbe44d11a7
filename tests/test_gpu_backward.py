"""GPU parity of the training-time FP4 attention (FastVideo "Pika H3 Flex in
FastVideo", section "NVFP4 QAD": 4-bit math on from the first step; the summary
list: the training-time FP4 attention matches the inference kernel): the bf16
dequantisation bit-exact, and the straight-through backward against the
oracle's fp64 gradients on the same NVFP4 codes.

The backward takes D_i = sum_c dO_ic O_ic from the forward output it is given
(as FlashAttention does).  Two kinds of test:

* kernel parity: both sides get the same inputs -- the oracle's dequantised
  Q^ and K^, its O rounded to bf16 and its lse -- so they take D from the same
  O.  The GPU then differs only by rounding P and dS to bf16 (unit roundoff
  2^-9) before the BF16 tensor-core products (fp32 accumulation) and by the
  bf16 outputs: a few 2^-9 relative on terms whose sum cancels (rows of dS sum
  to zero), bounded as max |d| <= 2e-2 max |ref| and ||d||_F <= 1e-2 ||ref||_F
  per gradient tensor and head;
* end to end: the GPU forward's bf16 O and lse feed the GPU backward, the
  oracle uses the exact definition.  The bf16 rounding of O (2^-9 relative)
  moves D by about 2^-9 ||dO_i|| ||O_i||, large against dP - D, which enters dS
  multiplied by P; a numpy emulation of exactly these roundings is 1.4-1.9%
  (norm-wise, dq) from the exact gradients on these inputs, so the bound for
  dq and dk is max |d| <= 6e-2 max |ref|, ||d||_F <= 4e-2 ||ref||_F (dv keeps
  the tight bound: it does not involve D).

Where a gradient vanishes exactly (one key: P = 1 and dS = 0) the reference
magnitude is floored at 1e-3 of the value gradient's, never degenerate."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import fa

pytestmark = pytest.mark.gpu

TIGHT = (2e-2, 1e-2)   # (max, Frobenius), relative
E2E_DQK = (6e-2, 4e-2)


def _dout(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def _gpu_step(d, dO, flags=0, scale=0.0):
    q, k, v = (d[t].cuda() for t in "qkv")
    out = fa().fp4attn_quantize_qk(q, k, flags=flags)
    o, lse = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v,
                                  softmax_scale=scale, want_lse=True, workspace=out["workspace"])
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    dq, dk, dv, ws = fa().fp4attn_backward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v, o,
                                           dO.cuda(), lse, scale, flags)
    assert fa().fp4attn_read_status(ws) == 0
    return dq.float().cpu().numpy(), dk.float().cpu().numpy(), dv.float().cpu().numpy()


def _assert_close(g, r, what, floor=0.0, tol=TIGHT):
    assert np.isfinite(g).all(), f"{what}: non-finite"
    d = np.abs(g.astype(np.float64) - r)
    mx, ref = float(d.max()), max(float(np.abs(r).max()), floor)
    fro = float(np.linalg.norm(d) / max(np.linalg.norm(r), floor * np.sqrt(r.size), 1e-300))
    print(f"{what}: max|d| {mx:.3e} (ref max {ref:.3e}), fro rel {fro:.3e}")
    assert mx <= tol[0] * ref + 1e-30 and fro <= tol[1], f"{what}: max|d|={mx:.3e} ref={ref:.3e} fro={fro:.3e}"


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)


def _kernel_parity(d, dO, flags=0, scale=None):
    """Same inputs on both sides: the oracle's codes, its O (rounded to bf16)
    and lse."""
    B, H, N, _ = d["q"].shape
    vb = synth.bf16_bits(d["v"])
    codes = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]), flags=flags)
    qh = oracle.dequant(codes["q_codes"], codes["q_scales"])
    kh = oracle.dequant(codes["k_codes"], codes["k_scales"])
    O = np.empty((B, H, N, 128))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            O[b, h], L[b, h] = oracle.attention_head(qh[b, h], kh[b, h], vb[b, h], scale)
    o_bf = _bf16(O)
    t = lambda key: torch.from_numpy(np.ascontiguousarray(codes[key])).cuda()
    dq, dk, dv, ws = fa().fp4attn_backward(t("q_codes"), t("q_scales"), t("k_codes"), t("k_scales"), d["v"].cuda(),
                                           o_bf.cuda(), dO.cuda(), torch.from_numpy(L.astype(np.float32)).cuda(),
                                           0.0 if scale is None else scale, flags)
    assert fa().fp4attn_read_status(ws) == 0
    ref = oracle.attention_backward(codes["q_codes"], codes["q_scales"], codes["k_codes"], codes["k_scales"], vb,
                                    dO.double().numpy(), scale=scale, flags=flags, O=o_bf.double().numpy())
    return (dq.float().cpu().numpy(), dk.float().cpu().numpy(), dv.float().cpu().numpy()), ref


def test_dequant_bf16_bit_exact():
    d = synth.generate(synth.custom("dqb", 1, 3, 777, seed=41, k_offset_std=2.0, n_outliers=2,
                                    outlier_factor=20.0), ("q", "k"))
    ref = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]))
    codes = torch.from_numpy(ref["k_codes"]).cuda()
    scales = torch.from_numpy(ref["k_scales"]).cuda()
    got = fa().fp4attn_dequant_bf16(codes, scales).float().cpu().numpy()
    want = oracle.dequant(ref["k_codes"], ref["k_scales"])  # exact in bf16 for g = 1
    assert np.array_equal(got, want)
    g = torch.tensor([0.37], dtype=torch.float32, device="cuda")
    got = fa().fp4attn_dequant_bf16(codes, scales, g).cpu()
    want = torch.from_numpy(oracle.dequant(ref["k_codes"], ref["k_scales"], 0.37)).to(torch.bfloat16)
    assert torch.equal(got, want)


@pytest.mark.parametrize("flags", [0, 3])
@pytest.mark.parametrize("N", [1, 64, 200, 1000])
def test_backward_parity(N, flags):
    w = synth.custom(f"bwd{N}", 1, 2, N, seed=700 + N, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w)
    dO = _dout((1, 2, N, 128), seed=N)
    (dq, dk, dv), (rq, rk, rv) = _kernel_parity(d, dO, flags)
    for h in range(2):
        floor = 1e-3 * float(np.abs(rv[0, h]).max())
        _assert_close(dq[0, h], rq[0, h], f"N{N} flags{flags} h{h} dq", floor)
        _assert_close(dk[0, h], rk[0, h], f"N{N} flags{flags} h{h} dk", floor)
        _assert_close(dv[0, h], rv[0, h], f"N{N} flags{flags} h{h} dv")
    if not flags & oracle.NO_SMOOTH_K:
        # the centring: every column of dk sums to zero (up to the bf16 rounding of dk)
        assert np.abs(dk.astype(np.float64).sum(axis=2)).max() <= 2e-3 * np.abs(dk).max() * np.sqrt(N)


@pytest.mark.parametrize("N,flags", [(64, 0), (1000, 0), (1000, 3)])
def test_backward_dv_within_an_elementwise_bound(N, flags):
    """dV element by element, with both sides given the same inputs: the
    GPU's P differs from the exact softmax by its bf16 rounding (2^-9
    relative) plus the exp2 approximation, the fp32 scores and the fp32 lse
    (together under 5e-4 relative); dV = P^T dO then accumulates in fp32 and
    is rounded to bf16.  So |dV_gpu - dV| <= 2.5e-3 (P^T |dO|) + 2^-9 |dV| to
    first order, elementwise; the test allows twice that, with P^T |dO| taken
    from the exact softmax of the same dequantised Q and K."""
    w = synth.custom(f"bwd{N}", 1, 2, N, seed=700 + N, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w)
    dO = _dout((1, 2, N, 128), seed=N)
    (_, _, dv), (_, _, rv) = _kernel_parity(d, dO, flags)
    codes = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]), flags=flags)
    qh = oracle.dequant(codes["q_codes"], codes["q_scales"]).astype(np.float64)
    kh = oracle.dequant(codes["k_codes"], codes["k_scales"]).astype(np.float64)
    for h in range(2):
        S = qh[0, h] @ kh[0, h].T / np.sqrt(128.0)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        A = P.T @ np.abs(dO[0, h].double().numpy())
        err = np.abs(dv[0, h].astype(np.float64) - rv[0, h])
        bound = 5e-3 * A + 2.0 ** -8 * np.abs(rv[0, h]) + 1e-30
        print(f"N{N} flags{flags} h{h}: worst |d|/bound {float((err / bound).max()):.3f}")
        assert (err <= bound).all(), f"N{N} flags{flags} h{h}: {int((err > bound).sum())} elements over the bound"


def test_backward_softmax_scale():
    w = synth.custom("bwd_scale", 1, 1, 300, seed=77, k_offset_std=2.0)
    d = synth.generate(w)
    dO = _dout((1, 1, 300, 128), seed=5)
    (dq, dk, dv), (rq, rk, rv) = _kernel_parity(d, dO, 0, scale=0.05)
    for g, r, name in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        _assert_close(g[0, 0], r[0, 0], f"scale 0.05 {name}")


def test_autograd_function_matches_the_c_calls_and_is_deterministic():
    w = synth.custom("bwd_ag", 1, 2, 333, seed=88, k_offset_std=2.0)
    d = synth.generate(w)
    dO = _dout((1, 2, 333, 128), seed=9)
    q, k, v = (d[t].cuda().requires_grad_(True) for t in "qkv")
    o = fa().fp4_attention(q, k, v)
    o.backward(dO.cuda())
    dq, dk, dv = _gpu_step(d, dO)
    assert np.array_equal(q.grad.float().cpu().numpy(), dq)
    assert np.array_equal(k.grad.float().cpu().numpy(), dk)
    assert np.array_equal(v.grad.float().cpu().numpy(), dv)


@pytest.mark.parametrize("N", [200, 1000])
def test_end_to_end_forward_and_backward(N):
    """GPU forward (bf16 O, lse) into the GPU backward, against the exact
    definition."""
    w = synth.custom(f"e2e{N}", 1, 2, N, seed=900 + N, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w)
    dO = _dout((1, 2, N, 128), seed=3 * N)
    dq, dk, dv = _gpu_step(d, dO)
    codes = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]))
    rq, rk, rv = oracle.attention_backward(codes["q_codes"], codes["q_scales"], codes["k_codes"], codes["k_scales"],
                                           synth.bf16_bits(d["v"]), dO.double().numpy())
    for h in range(2):
        _assert_close(dq[0, h], rq[0, h], f"e2e N{N} h{h} dq", tol=E2E_DQK)
        _assert_close(dk[0, h], rk[0, h], f"e2e N{N} h{h} dk", tol=E2E_DQK)
        _assert_close(dv[0, h], rv[0, h], f"e2e N{N} h{h} dv")


def test_backward_mid_workload_two_heads():
    """The mid workload (B1 H8 N8192, outlier channels, key bias): the whole
    forward and backward on the GPU, heads 0 and 7 against the exact
    definition (end-to-end bounds)."""
    w = synth.WORKLOADS["mid"]
    d = synth.generate(w)
    dO = _dout(w.shape, seed=123)
    dq, dk, dv = _gpu_step(d, dO)
    for h in (0, 7):
        one = synth.generate(w, ("q", "k", "v"), heads=[h])
        codes = oracle.quantize_qk(synth.bf16_bits(one["q"]), synth.bf16_bits(one["k"]))
        rq, rk, rv = oracle.attention_backward(codes["q_codes"], codes["q_scales"], codes["k_codes"],
                                               codes["k_scales"], synth.bf16_bits(one["v"]),
                                               dO[:, h:h + 1].double().numpy())
        _assert_close(dq[0, h], rq[0, 0], f"mid h{h} dq", tol=E2E_DQK)
        _assert_close(dk[0, h], rk[0, 0], f"mid h{h} dk", tol=E2E_DQK)
        _assert_close(dv[0, h], rv[0, 0], f"mid h{h} dv")


@pytest.mark.parametrize("name,kw", [("N(0,1)", dict(seed=51)),
                                     ("bias + outliers", dict(seed=52, k_offset_std=2.0, n_outliers=2,
                                                              outlier_factor=20.0))])
def test_fake_quant_forward_matches_the_fp4_kernel_within_1pct_of_quantisation_error(name, kw):
    """The page's summary claim, checked between this library's kernels: the
    fake-quantised forward (the BF16 kernel on the dequantised Q^ and K^, as a
    training framework would run it) differs from the FP4 kernel by under 1% of
    the FP4 kernel's own quantisation error (its distance to the BF16 kernel on
    the unquantised Q and K)."""
    w = synth.custom("fakeq", 1, 4, 4096, **kw)
    d = synth.generate(w)
    q, k, v = (d[t].cuda() for t in "qkv")
    out = fa().fp4attn_quantize_qk(q, k)  # smoothing shifts each score row: softmax ignores it
    o4, _ = fa().fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v,
                                 workspace=out["workspace"])
    qh = fa().fp4attn_dequant_bf16(out["q_codes"], out["q_scales"])
    kh = fa().fp4attn_dequant_bf16(out["k_codes"], out["k_scales"])
    of, _ = fa().fp4attn_forward_bf16qk(qh, kh, v)
    ob, _ = fa().fp4attn_forward_bf16qk(q, k, v)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    quant_err = torch.linalg.vector_norm((o4.float() - ob.float()))
    fake_gap = torch.linalg.vector_norm((of.float() - o4.float()))
    print(f"{name}: |fake - fp4| / |fp4 - bf16| = {float(fake_gap / quant_err):.4f}")
    assert fake_gap <= 0.01 * quant_err


def test_autograd_with_dynamic_scales_and_flags():
    """fp4_attention with the dynamic per-tensor scales and each transform off:
    gradients against the oracle's (same g, end-to-end bounds).  The backward
    works on the unit-scale Q~, K~ and takes g as scalars: rounding g * Q~ to
    bf16 instead would move the scores of these outlier-heavy keys (lse up to
    about 360) by tenths of a unit and the gradients by over 10%."""
    w = synth.custom("bwd_dyn", 1, 2, 400, seed=91, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w)
    dO = _dout((1, 2, 400, 128), seed=11)
    for flags in (0, 3):
        q, k, v = (d[t].cuda().requires_grad_(True) for t in "qkv")
        o = fa().fp4_attention(q, k, v, flags=flags, dynamic_gscale=True)
        o.backward(dO.cuda())
        ref = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]), flags=flags, dynamic=True)
        rq, rk, rv = oracle.attention_backward(ref["q_codes"], ref["q_scales"], ref["k_codes"], ref["k_scales"],
                                               synth.bf16_bits(d["v"]), dO.double().numpy(), float(ref["gq"]),
                                               float(ref["gk"]), flags=flags)
        for h in range(2):
            _assert_close(q.grad[0, h].float().cpu().numpy(), rq[0, h], f"dyn flags{flags} h{h} dq", tol=E2E_DQK)
            _assert_close(k.grad[0, h].float().cpu().numpy(), rk[0, h], f"dyn flags{flags} h{h} dk", tol=E2E_DQK)
            _assert_close(v.grad[0, h].float().cpu().numpy(), rv[0, h], f"dyn flags{flags} h{h} dv")


def test_backward_kernel_parity_with_global_scales():
    """Static global scales gQ = 0.37, gK = 1.9 (the scales enter the backward
    as scalars); same inputs on both sides (the oracle's codes, its O rounded
    to bf16 and its lse), tight bounds."""
    gq, gk = 0.37, 1.9
    w = synth.custom("bwd_g", 1, 2, 333, seed=93, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w)
    dO = _dout((1, 2, 333, 128), seed=13)
    vb = synth.bf16_bits(d["v"])
    codes = oracle.quantize_qk(synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]), gq, gk)
    O = np.empty((1, 2, 333, 128))
    L = np.empty((1, 2, 333))
    for h in range(2):
        O[0, h], L[0, h] = oracle.attention_head(oracle.dequant(codes["q_codes"][0, h], codes["q_scales"][0, h], gq),
                                                 oracle.dequant(codes["k_codes"][0, h], codes["k_scales"][0, h], gk),
                                                 vb[0, h])
    o_bf = _bf16(O)
    t = lambda key: torch.from_numpy(np.ascontiguousarray(codes[key])).cuda()
    g = lambda x: torch.tensor([x], dtype=torch.float32, device="cuda")
    dq, dk, dv, ws = fa().fp4attn_backward(t("q_codes"), t("q_scales"), t("k_codes"), t("k_scales"), d["v"].cuda(),
                                           o_bf.cuda(), dO.cuda(), torch.from_numpy(L.astype(np.float32)).cuda(),
                                           q_gscale=g(gq), k_gscale=g(gk))
    assert fa().fp4attn_read_status(ws) == 0
    rq, rk, rv = oracle.attention_backward(codes["q_codes"], codes["q_scales"], codes["k_codes"], codes["k_scales"],
                                           vb, dO.double().numpy(), gq, gk, O=o_bf.double().numpy())
    for h in range(2):
        _assert_close(dq[0, h].float().cpu().numpy(), rq[0, h], f"g h{h} dq")
        _assert_close(dk[0, h].float().cpu().numpy(), rk[0, h], f"g h{h} dk")
        _assert_close(dv[0, h].float().cpu().numpy(), rv[0, h], f"g h{h} dv")


def test_autograd_in_the_projection_layout_matches_contiguous_bit_for_bit():
    """Q, K, V as [B,H,N,128] views of [B,N,H,128] tensors (no copies): the
    forward output and the three gradients equal the contiguous run's bits."""
    w = synth.custom("bwd_bnhd", 1, 3, 500, seed=95, k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)
    d = synth.generate(w)
    dO = _dout((1, 3, 500, 128), seed=15).cuda()
    runs = []
    for layout in ("bhnd", "bnhd"):
        if layout == "bhnd":
            leaves = [d[t].cuda().requires_grad_(True) for t in "qkv"]
            views = leaves
        else:
            leaves = [d[t].transpose(1, 2).contiguous().cuda().requires_grad_(True) for t in "qkv"]
            views = [x.transpose(1, 2) for x in leaves]
        o = fa().fp4_attention(*views)
        o.backward(dO)
        grads = [x.grad if layout == "bhnd" else x.grad.transpose(1, 2) for x in leaves]
        runs.append([o.detach()] + grads)
    for a, b in zip(*runs):
        assert torch.equal(a.contiguous(), b.contiguous())
    assert runs[1][0].stride() == runs[1][0].transpose(1, 2).contiguous().transpose(1, 2).stride()
