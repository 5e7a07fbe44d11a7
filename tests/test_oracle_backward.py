"""Pins for the oracle's training-time backward (CPU only).

FastVideo "Pika H3 Flex in FastVideo": section "NVFP4 QAD" distils the 4-bit
student with 4-bit math on from the first step, and the summary list states
that the training-time FP4 attention matches the inference kernel.  Reading:
fake quantisation with a straight-through estimator -- attention gradients at
the dequantised Q and K, passed unchanged through the quantiser, with the
exact transforms (rotation, key centring) differentiated.

Independent checks: torch's fp64 autograd of softmax attention, central finite
differences of a numpy fp64 forward, closed-form invariants (key-gradient
column sums vanish, value-gradient column sums equal those of dO), and the
straight-through composition against autograd through an fp64 transform built
from scipy's Hadamard matrix.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from nvfp4_precision_b200 import synth


def _head(N, seed, k_bias=0.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((N, 128)).astype(np.float32)
    k = (rng.standard_normal((N, 128)) + k_bias * rng.standard_normal(128)).astype(np.float32)
    v = torch.from_numpy(rng.standard_normal((N, 128)).astype(np.float32)).to(torch.bfloat16)
    dO = rng.standard_normal((N, 128))
    return q, k, synth.bf16_bits(v), v.double().numpy(), dO


def _torch_grads(q, k, v, dO, scale):
    Q = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    K = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    V = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    O = torch.softmax(scale * Q @ K.T, dim=-1) @ V
    O.backward(torch.tensor(dO))
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


@pytest.mark.parametrize("N,scale", [(1, None), (7, None), (130, None), (300, 0.05)])
def test_backward_matches_torch_fp64_autograd(N, scale):
    q, k, vb, v, dO = _head(N, seed=N)
    s = 1.0 / np.sqrt(128.0) if scale is None else scale
    got = oracle.attention_backward_head(q, k, vb, dO, scale)
    want = _torch_grads(q, k, v, dO, s)
    for g, w, name in zip(got, want, ("dq", "dk", "dv")):
        assert np.allclose(g, w, rtol=1e-10, atol=1e-12 * max(1.0, np.abs(w).max())), name


def test_backward_matches_finite_differences():
    N = 6
    q, k, vb, v, dO = _head(N, seed=11, k_bias=1.0)
    s = 1.0 / np.sqrt(128.0)

    def loss(qq, kk, vv):
        S = s * qq @ kk.T
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        return float(np.sum((P @ vv) * dO))

    dq, dk, dv = oracle.attention_backward_head(q, k, vb, dO)
    q64, k64 = q.astype(np.float64), k.astype(np.float64)
    h = 1e-6
    rng = np.random.default_rng(0)
    for _ in range(6):
        i, c = int(rng.integers(N)), int(rng.integers(128))
        for x, g, which in ((q64, dq, 0), (k64, dk, 1), (v, dv, 2)):
            xp, xm = x.copy(), x.copy()
            xp[i, c] += h
            xm[i, c] -= h
            args_p = [q64, k64, v]
            args_m = [q64, k64, v]
            args_p[which], args_m[which] = xp, xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[i, c]) <= 1e-6 * max(1.0, abs(fd)), (which, i, c, fd, g[i, c])


def test_backward_invariants():
    q, k, vb, v, dO = _head(257, seed=5, k_bias=2.0)
    dq, dk, dv = oracle.attention_backward_head(q, k, vb, dO)
    # a shift shared by every key leaves softmax unchanged: the key gradients sum to 0
    assert np.abs(dk.sum(axis=0)).max() <= 1e-10 * np.abs(dk).sum(axis=0).max()
    # every row of P sums to 1: the value gradients sum to the output gradients
    assert np.allclose(dv.sum(axis=0), dO.sum(axis=0), rtol=1e-10, atol=1e-10)


def test_ste_grads_orthonormal_rotation_and_flags():
    rng = np.random.default_rng(3)
    dqh, dkh = rng.standard_normal((40, 128)), rng.standard_normal((40, 128))
    dq, dk = oracle.ste_grads(dqh, dkh, 0)
    Hm = scipy.linalg.hadamard(128) / np.sqrt(128.0)
    assert np.allclose(dq, dqh @ Hm, rtol=1e-12, atol=1e-12)
    assert np.allclose(dk, (dkh - dkh.mean(axis=0)) @ Hm, rtol=1e-12, atol=1e-12)
    assert np.allclose(np.linalg.norm(dq), np.linalg.norm(dqh))
    dq, dk = oracle.ste_grads(dqh, dkh, oracle.NO_HADAMARD)
    assert np.array_equal(dq, dqh) and np.allclose(dk, dkh - dkh.mean(axis=0))
    dq, dk = oracle.ste_grads(dqh, dkh, oracle.NO_SMOOTH_K | oracle.NO_HADAMARD)
    assert np.array_equal(dq, dqh) and np.array_equal(dk, dkh)


@pytest.mark.parametrize("flags", [0, oracle.NO_SMOOTH_K, oracle.NO_HADAMARD])
def test_straight_through_composition_equals_autograd_of_the_exact_transform(flags):
    """Without quantisation the straight-through gradient is the exact one:
    autograd of attention(c H q, c H (k - mean k), v) in fp64."""
    N = 33
    q, k, vb, v, dO = _head(N, seed=21, k_bias=1.5)
    Hm = torch.tensor(scipy.linalg.hadamard(128) / np.sqrt(128.0))
    if flags & oracle.NO_HADAMARD:
        Hm = torch.eye(128, dtype=torch.float64)
    Q = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    K = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    Kc = K if flags & oracle.NO_SMOOTH_K else K - K.mean(dim=0, keepdim=True)
    Qt, Kt = Q @ Hm, Kc @ Hm
    s = 1.0 / np.sqrt(128.0)
    O = torch.softmax(s * Qt @ Kt.T, dim=-1) @ torch.tensor(v)
    O.backward(torch.tensor(dO))
    # the oracle takes the transformed rows as its (fp32) dequantised operands;
    # use rows exactly representable in fp32 so both sides see the same values
    qt = Qt.detach().numpy().astype(np.float32)
    kt = Kt.detach().numpy().astype(np.float32)
    Q2 = torch.tensor(qt.astype(np.float64))
    K2 = torch.tensor(kt.astype(np.float64))
    dqh, dkh, _ = oracle.attention_backward_head(qt, kt, vb, dO)
    dq, dk = oracle.ste_grads(dqh, dkh, flags)
    # reference: the same composition evaluated by autograd at the fp32-rounded rows
    Qr = Q2.clone().requires_grad_(True)
    Kr = K2.clone().requires_grad_(True)
    Or = torch.softmax(s * Qr @ Kr.T, dim=-1) @ torch.tensor(v)
    Or.backward(torch.tensor(dO))
    gq = Qr.grad @ Hm.T
    gk = Kr.grad @ Hm.T
    if not flags & oracle.NO_SMOOTH_K:
        gk = gk - gk.mean(dim=0, keepdim=True)
    assert np.allclose(dq, gq.numpy(), rtol=1e-9, atol=1e-11)
    assert np.allclose(dk, gk.numpy(), rtol=1e-9, atol=1e-11)
    # and at the exact (unrounded) transform the gradients agree to fp32 rounding
    assert np.allclose(dq, Q.grad.numpy(), rtol=1e-4, atol=1e-5)
    assert np.allclose(dk, K.grad.numpy(), rtol=1e-4, atol=1e-5)


def test_attention_backward_over_quantised_heads():
    w = synth.custom("bwd", 1, 2, 96, seed=9, k_offset_std=2.0)
    d = synth.generate(w)
    qb, kb, vb = synth.bf16_bits(d["q"]), synth.bf16_bits(d["k"]), synth.bf16_bits(d["v"])
    codes = oracle.quantize_qk(qb, kb)
    dO = np.random.default_rng(1).standard_normal((1, 2, 96, 128))
    dq, dk, dv = oracle.attention_backward(codes["q_codes"], codes["q_scales"], codes["k_codes"],
                                           codes["k_scales"], vb, dO)
    for h in range(2):
        qh = oracle.dequant(codes["q_codes"][0, h], codes["q_scales"][0, h])
        kh = oracle.dequant(codes["k_codes"][0, h], codes["k_scales"][0, h])
        a, b, c = oracle.attention_backward_head(qh, kh, vb[0, h], dO[0, h])
        e, f = oracle.ste_grads(a, b, 0)
        assert np.array_equal(dq[0, h], e) and np.array_equal(dk[0, h], f) and np.array_equal(dv[0, h], c)
    # the straight-through key gradient has zero column sums (the centring)
    assert np.abs(dk.sum(axis=2)).max() <= 1e-9 * np.abs(dk).max() * 96


def test_backward_with_given_output_equals_definition_at_the_exact_output():
    """D taken from a supplied forward output equals the definition when that
    output is the exact O, and moves with it otherwise (the contract of a
    backward that receives the stored forward output)."""
    q, k, vb, v, dO = _head(90, seed=31, k_bias=1.0)
    O, _ = oracle.attention_head(q, k, vb)
    a = oracle.attention_backward_head(q, k, vb, dO)
    b = oracle.attention_backward_head(q, k, vb, dO, O=O)
    for x, y in zip(a, b):
        assert np.allclose(x, y, rtol=1e-11, atol=1e-13 * np.abs(x).max())
    c = oracle.attention_backward_head(q, k, vb, dO, O=O + 0.01)
    assert not np.allclose(c[0], a[0], rtol=1e-6) and np.array_equal(c[2], a[2])


def test_attention_all_rows_equals_the_c_definition():
    """The chunked fp64 forward (torch CPU ops) against the scalar C loop, with
    a chunk size that leaves a ragged last chunk."""
    q, k, vb, v, _ = _head(301, seed=41, k_bias=2.0)
    O1, L1 = oracle.attention_head(q, k, vb)
    O2, L2 = oracle.attention_all_rows(q, k, vb, chunk=64)
    assert np.allclose(O2, O1, rtol=1e-12, atol=1e-14) and np.allclose(L2, L1, rtol=1e-13, atol=1e-13)
    O3, L3 = oracle.attention_all_rows(q, k, vb, scale=0.05, chunk=1000)
    O4, L4 = oracle.attention_head(q, k, vb, scale=0.05)
    assert np.allclose(O3, O4, rtol=1e-12, atol=1e-14) and np.allclose(L3, L4, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("flags", [0, oracle.NO_SMOOTH_K, oracle.NO_HADAMARD, oracle.NO_SMOOTH_K | oracle.NO_HADAMARD])
def test_sampled_backward_rows_equal_the_whole_head(flags):
    """The sampled-row backward (the key mean through the row sums of dS) against
    the whole-head C definition plus ste_grads, with D taken from a perturbed
    forward output so that the rows of dS do not sum to zero."""
    N = 257
    q, k, vb, v, dO = _head(N, seed=43, k_bias=1.5)
    O_exact, lse = oracle.attention_all_rows(q, k, vb)
    O = O_exact + 0.01 * np.random.default_rng(2).standard_normal(O_exact.shape)
    dqh, dkh, dv = oracle.attention_backward_head(q, k, vb, dO, O=O)
    dq, dk = oracle.ste_grads(dqh, dkh, flags)
    I = np.array([0, 5, 128, 256])
    J = np.array([1, 17, 200, 256, 3])
    a, b, c = oracle.attention_backward_rows(q, k, vb, dO, O, O_exact, lse, I, J, flags=flags)
    for got, want in ((a, dq[I]), (b, dk[J]), (c, dv[J])):
        assert np.allclose(got, want, rtol=1e-10, atol=1e-12 * np.abs(want).max())
    # the centring term is not zero here, so dropping it would be caught
    if not flags & oracle.NO_SMOOTH_K:
        _, dk_raw = oracle.ste_grads(dqh, dkh, flags | oracle.NO_SMOOTH_K)
        assert not np.allclose(b, dk_raw[J], rtol=1e-6, atol=0)
