"""The page's toy heads at their own width -- TEST INFRASTRUCTURE ONLY, like
the rest of this package.

FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention": the toy heads
have 64 channels (four 16-value blocks) and 32 keys, Gaussian values, a
per-channel key bias and two scaled-up channels; they are quantised like the
FP4 attention kernel (E2M1 values, one E4M3 scale per 16 channels, unit
global scale) with P and V in BF16, and the page compares plain FP4 against FP4
with both transforms (smooth K, the same orthonormal Hadamard on Q and K).

The CUDA library is d = 128 only; this module restates the prologue for any
power-of-two width in numpy, with the same pinned steps as the C oracle:
  * key mean: the exact fixed-point sum of round_half_even(k * 2^24) per
    channel, then (float)(sum / (N 2^24)) -- channels are independent, so it
    is the C key sum of the head zero-padded to 128 channels;
  * Hadamard: the Sylvester-order butterflies in fp32, strides ascending, then
    x fp32(1/sqrt(d)) (1/8 exactly for d = 64);
  * NVFP4 pack: blocks of 16 are independent, so a row of d <= 128 is packed
    as the first d/16 blocks of the C pack of the zero-padded 128-wide row.
Attention is fp64 over the dequantised Q and K, with the exponentials of each
row (row max subtracted) rounded to bf16 for P.V and the row sum taken over
those rounded values, as in the kernel (P and V stay in BF16)."""
from __future__ import annotations

import numpy as np

from . import NO_HADAMARD, NO_SMOOTH_K, dequant, kmean, ksum, quantize_rows


def _bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalised fp32 Walsh-Hadamard transform of each row (width a power of
    two): for h = 1, 2, 4, ...: (x_i, x_{i+h}) <- (x_i + x_{i+h}, x_i - x_{i+h})
    for every i with (i & h) == 0, each an fp32 round-to-nearest operation."""
    y = np.array(x, dtype=np.float32, copy=True)
    d = y.shape[-1]
    assert d & (d - 1) == 0
    h = 1
    while h < d:
        v = y.reshape(y.shape[:-1] + (d // (2 * h), 2, h))
        a, b = v[..., 0, :].copy(), v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        h *= 2
    return y


def _pad128(x: np.ndarray) -> np.ndarray:
    out = np.zeros(x.shape[:-1] + (128,), dtype=x.dtype)
    out[..., : x.shape[-1]] = x
    return out


def quantize(q_bits: np.ndarray, k_bits: np.ndarray, flags: int = 0) -> dict:
    """Smooth K, rotate and NVFP4-pack one set of heads of width d (multiple
    of 16, at most 128, a power of two when rotating) at unit global scale.
    q_bits, k_bits: uint16 bf16 bits [H, N, d].  Returns dict(q_codes,
    k_codes [H, N, d/2] uint8 (element 2i in the low nibble of byte i),
    q_scales, k_scales [H, N, d/16] uint8 (UE4M3), k_mean [H, d] float32)."""
    H, N, d = q_bits.shape
    assert d % 16 == 0 and d <= 128
    q = _bits_to_f32(q_bits)
    k = _bits_to_f32(k_bits)
    mean = np.zeros((H, d), np.float32)
    if not flags & NO_SMOOTH_K:
        S, st = ksum(_pad128(np.ascontiguousarray(k_bits, dtype=np.uint16)))
        assert st == 0
        mean = kmean(S, N)[:, :d]
        k = k - mean[:, None, :]
    if not flags & NO_HADAMARD:
        c = np.float32(1.0 / np.sqrt(float(d)))
        q = fwht(q) * c
        k = fwht(k) * c
    out = dict(k_mean=mean)
    for name, y in (("q", q), ("k", k)):
        codes, scales = quantize_rows(_pad128(y.reshape(-1, d)))
        out[name + "_codes"] = codes[:, : d // 2].reshape(H, N, d // 2)
        out[name + "_scales"] = scales[:, : d // 16].reshape(H, N, d // 16)
    return out


def prologue(q_bits: np.ndarray, k_bits: np.ndarray, flags: int = 0):
    """quantize() followed by dequantisation: returns (qhat, khat) float32
    [H, N, d] (unit global scale: exact values of scale x E2M1)."""
    c = quantize(q_bits, k_bits, flags)
    d = q_bits.shape[-1]
    out = []
    for t in ("q", "k"):
        codes = np.zeros(c[t + "_codes"].shape[:-1] + (64,), np.uint8)
        scales = np.zeros(c[t + "_scales"].shape[:-1] + (8,), np.uint8)
        codes[..., : d // 2] = c[t + "_codes"]
        scales[..., : d // 16] = c[t + "_scales"]
        out.append(dequant(codes, scales)[..., :d])
    return out[0], out[1]


def attention(qhat: np.ndarray, khat: np.ndarray, v_bits: np.ndarray, bf16_p: bool = True) -> np.ndarray:
    """fp64 softmax(Q K^T / sqrt(d)) V of each head [H, N, d]; with bf16_p the
    row's exponentials are rounded to bf16 before P.V and the row sum is taken
    over the rounded values."""
    q = np.asarray(qhat, dtype=np.float64)
    k = np.asarray(khat, dtype=np.float64)
    v = _bits_to_f32(v_bits).astype(np.float64)
    s = q @ np.swapaxes(k, -1, -2) / np.sqrt(float(q.shape[-1]))
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    if bf16_p:
        p = _round_bf16(p)
    return (p @ v) / p.sum(axis=-1, keepdims=True)


def _round_bf16(x: np.ndarray) -> np.ndarray:
    """The kernel's p is an fp32 value rounded to bf16 (nearest even): round
    the fp64 value to fp32, then its bit pattern to the upper 16 bits (finite,
    non-negative inputs)."""
    f = np.asarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def errors(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray) -> dict:
    """Relative Frobenius error of each head's O, per variant, against fp64
    attention of the unquantised bf16 Q and K (P unrounded).  Variants: plain
    FP4, + smooth K, + Hadamard, + both."""
    ref = attention(_bits_to_f32(q_bits), _bits_to_f32(k_bits), v_bits, bf16_p=False)
    out = {}
    for name, flags in (("plain", NO_SMOOTH_K | NO_HADAMARD), ("smooth K", NO_HADAMARD),
                        ("Hadamard", NO_SMOOTH_K), ("both", 0)):
        qh, kh = prologue(q_bits, k_bits, flags)
        o = attention(qh, kh, v_bits)
        out[name] = np.linalg.norm(o - ref, axis=(1, 2)) / np.linalg.norm(ref, axis=(1, 2))
    return out
