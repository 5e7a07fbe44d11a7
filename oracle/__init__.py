"""CPU oracle for the FP4 dense-attention path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never imports it, and this package imports nothing from the product.

It wraps the plain C implementation in ``oracle.c`` (codecs, exact fixed-point
key mean, pinned-order Hadamard, NVFP4 pack, dequantisation and fp64
attention) with numpy-friendly functions.  Two helpers for the longest
sequences (every query row of a head's fp64 attention; sampled rows of the
training-time gradients) use torch's fp64 CPU matrix products instead of the
scalar C loops.  Every function is pinned by the CPU tests against something
other than itself.

Method source: FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention"
(smooth K, the same orthonormal Hadamard on Q and K, NVFP4 Q/K with E2M1 values
and one E4M3 scale per 16 channels under a unit global scale, P and V in BF16).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

NO_SMOOTH_K = 1
NO_HADAMARD = 2
OK = 0
ERR_RANGE = 4

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_decode.restype = ctypes.c_float
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_ue4m3_encode.restype = ctypes.c_uint8
        L.oracle_ue4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_ue4m3_decode.restype = ctypes.c_float
        L.oracle_ue4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_encode_array.argtypes = [P, i64, P]
        L.oracle_ue4m3_encode_array.argtypes = [P, i64, P]
        L.oracle_ksum.restype = ctypes.c_int
        L.oracle_ksum.argtypes = [P, i64, i64, P]
        L.oracle_kmean.argtypes = [P, i64, i64, P]
        L.oracle_fwht128.argtypes = [P]
        L.oracle_hadamard_scale.restype = ctypes.c_float
        L.oracle_transform_rows.argtypes = [P, i64, P, ctypes.c_uint32, P]
        L.oracle_quantize_rows.argtypes = [P, i64, ctypes.c_float, P, P]
        L.oracle_quantize_qk.restype = ctypes.c_int
        L.oracle_quantize_qk.argtypes = [P, P, i64, i64, i64, ctypes.c_float, ctypes.c_float,
                                         ctypes.c_uint32, P, P, P, P, P]
        L.oracle_dynamic_gscale.restype = ctypes.c_int
        L.oracle_dynamic_gscale.argtypes = [P, P, i64, i64, i64, ctypes.c_uint32, P, P]
        L.oracle_dequant.argtypes = [P, P, ctypes.c_float, i64, P]
        L.oracle_attention_head.argtypes = [P, P, P, i64, ctypes.c_double, P, i64, P, P]
        L.oracle_attention_backward_head.argtypes = [P, P, P, P, P, i64, ctypes.c_double, P, P, P]
        L.oracle_ste_grads.argtypes = [P, P, i64, ctypes.c_uint32, P, P]
        L.oracle_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().oracle_num_threads()


# -- codecs -----------------------------------------------------------------

def e2m1_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_e2m1_encode_array(_p(x), x.size, _p(out))
    return out


def e2m1_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    f = lib().oracle_e2m1_decode
    return np.array([f(int(c)) for c in codes.ravel()], dtype=np.float32).reshape(codes.shape)


def ue4m3_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_ue4m3_encode_array(_p(x), x.size, _p(out))
    return out


def ue4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    f = lib().oracle_ue4m3_decode
    return np.array([f(int(c)) for c in codes.ravel()], dtype=np.float32).reshape(codes.shape)


# -- smooth K / Hadamard ------------------------------------------------------

def ksum(k_bits: np.ndarray):
    """k_bits: uint16 bf16 bits [BH, N, 128] -> (int64 sums [BH,128], status)."""
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    BH, N = k_bits.shape[0], k_bits.shape[1]
    S = np.zeros((BH, 128), dtype=np.int64)
    st = lib().oracle_ksum(_p(k_bits), BH, N, _p(S))
    return S, st


def kmean(S: np.ndarray, N: int) -> np.ndarray:
    S = np.ascontiguousarray(S, dtype=np.int64)
    m = np.empty(S.shape, dtype=np.float32)
    lib().oracle_kmean(_p(S), S.shape[0], N, _p(m))
    return m


def fwht128(x) -> np.ndarray:
    """Unnormalised pinned-order fp32 FWHT of each row of 128."""
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    flat = x.reshape(-1, 128)
    for r in range(flat.shape[0]):
        lib().oracle_fwht128(_p(flat[r]))
    return x


def hadamard_scale() -> np.float32:
    return np.float32(lib().oracle_hadamard_scale())


def transform_rows(rows_bits: np.ndarray, mean=None, flags: int = 0) -> np.ndarray:
    """Pre-quantisation transform of bf16 rows [R,128]: (row - mean) then H."""
    rows_bits = np.ascontiguousarray(rows_bits, dtype=np.uint16).reshape(-1, 128)
    y = np.empty(rows_bits.shape, dtype=np.float32)
    mp = None
    if mean is not None:
        mean = np.ascontiguousarray(mean, dtype=np.float32)
        mp = _p(mean)
    lib().oracle_transform_rows(_p(rows_bits), rows_bits.shape[0], mp, flags, _p(y))
    return y


# -- NVFP4 pack ---------------------------------------------------------------

def quantize_rows(y: np.ndarray, g: float = 1.0):
    y = np.ascontiguousarray(y, dtype=np.float32).reshape(-1, 128)
    codes = np.empty((y.shape[0], 64), dtype=np.uint8)
    scales = np.empty((y.shape[0], 8), dtype=np.uint8)
    lib().oracle_quantize_rows(_p(y), y.shape[0], g, _p(codes), _p(scales))
    return codes, scales


def dynamic_gscale(q_bits: np.ndarray, k_bits: np.ndarray, flags: int = 0):
    """Per-tensor scales from the transformed tensors' largest magnitudes:
    g = fl32(amax / (6 * 448)), at least 2^-64.  Returns (gq, gk, status) with
    gq, gk as np.float32."""
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    B, H, N, D = q_bits.shape
    assert D == 128 and k_bits.shape == q_bits.shape
    g = np.zeros(2, np.float32)
    st = lib().oracle_dynamic_gscale(_p(q_bits), _p(k_bits), B, H, N, flags, _p(g[:1]), _p(g[1:]))
    return g[0], g[1], st


def quantize_qk(q_bits: np.ndarray, k_bits: np.ndarray, gq: float = 1.0, gk: float = 1.0, flags: int = 0,
                dynamic: bool = False):
    """Whole prologue on uint16 bf16 bits [B,H,N,128].  dynamic=True replaces
    gq and gk by dynamic_gscale(q_bits, k_bits, flags).

    Returns dict(q_codes [B,H,N,64], q_scales [B,H,N,8], k_codes, k_scales,
    k_mean [B,H,128] float32, gq, gk (float32), status)."""
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    B, H, N, D = q_bits.shape
    assert D == 128 and k_bits.shape == q_bits.shape
    dst = OK
    if dynamic:
        gq, gk, dst = dynamic_gscale(q_bits, k_bits, flags)
    out = dict(
        q_codes=np.empty((B, H, N, 64), np.uint8), q_scales=np.empty((B, H, N, 8), np.uint8),
        k_codes=np.empty((B, H, N, 64), np.uint8), k_scales=np.empty((B, H, N, 8), np.uint8),
        k_mean=np.empty((B, H, 128), np.float32))
    st = lib().oracle_quantize_qk(_p(q_bits), _p(k_bits), B, H, N, gq, gk, flags,
                                  _p(out["q_codes"]), _p(out["q_scales"]),
                                  _p(out["k_codes"]), _p(out["k_scales"]), _p(out["k_mean"]))
    out["status"] = st if st != OK else dst
    out["gq"], out["gk"] = np.float32(gq), np.float32(gk)
    return out


def dequant(codes: np.ndarray, scales: np.ndarray, g: float = 1.0) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows = codes.size // 64
    assert scales.size == rows * 8
    out = np.empty(codes.shape[:-1] + (128,), dtype=np.float32)
    lib().oracle_dequant(_p(codes), _p(scales), g, rows, _p(out))
    return out


# -- attention ------------------------------------------------------------------

def attention_head(qhat: np.ndarray, khat: np.ndarray, v_bits: np.ndarray, scale=None, rows=None):
    """fp64 attention of one head.  qhat, khat: float32 [N,128] (dequantised);
    v_bits: uint16 bf16 bits [N,128].  rows: optional int64 query-row subset.
    Returns (O float64 [R,128], lse float64 [R])."""
    qhat = np.ascontiguousarray(qhat, dtype=np.float32)
    khat = np.ascontiguousarray(khat, dtype=np.float32)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    N = khat.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(128.0)
    if rows is None:
        R = qhat.shape[0]
        rp = None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R = rows.size
        rp = _p(rows)
    O = np.empty((R, 128), np.float64)
    lse = np.empty((R,), np.float64)
    lib().oracle_attention_head(_p(qhat), _p(khat), _p(v_bits), N, float(scale), rp, R, _p(O), _p(lse))
    return O, lse


def attention(q_codes, q_scales, k_codes, k_scales, v_bits, gq=1.0, gk=1.0, scale=None, rows=None):
    """fp64 attention over all heads of [B,H,N,...] quantised Q/K and bf16 V.
    rows: optional per-head query-row subset (same rows in every head).
    Returns (O [B,H,R,128] float64, lse [B,H,R] float64)."""
    B, H, N = q_codes.shape[:3]
    R = N if rows is None else len(rows)
    O = np.empty((B, H, R, 128), np.float64)
    L = np.empty((B, H, R), np.float64)
    for b in range(B):
        for h in range(H):
            qh = dequant(q_codes[b, h], q_scales[b, h], gq)
            kh = dequant(k_codes[b, h], k_scales[b, h], gk)
            O[b, h], L[b, h] = attention_head(qh, kh, v_bits[b, h], scale, rows)
    return O, L


# -- training-time backward (fake quantisation, straight-through estimator) ------

def attention_backward_head(qhat: np.ndarray, khat: np.ndarray, v_bits: np.ndarray, dO: np.ndarray, scale=None,
                            O=None):
    """fp64 gradients of one head's attention at the dequantised Q and K.
    qhat, khat: float32 [N,128]; v_bits: bf16 bits [N,128]; dO: [N,128] (any
    float dtype, used in fp64); O: optional forward output [N,128] that D is
    taken from (default: the exact definition).  Returns (dqhat, dkhat, dv),
    fp64 [N,128]."""
    qhat = np.ascontiguousarray(qhat, dtype=np.float32)
    khat = np.ascontiguousarray(khat, dtype=np.float32)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    dO = np.ascontiguousarray(dO, dtype=np.float64)
    N = khat.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(128.0)
    dq, dk, dv = (np.empty((N, 128), np.float64) for _ in range(3))
    op = None
    if O is not None:
        O = np.ascontiguousarray(O, dtype=np.float64)
        op = _p(O)
    lib().oracle_attention_backward_head(_p(qhat), _p(khat), _p(v_bits), _p(dO), op, N, float(scale),
                                         _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def ste_grads(dqhat: np.ndarray, dkhat: np.ndarray, flags: int = 0):
    """Straight-through gradients of one head's prologue inputs from the
    gradients at the dequantised Q and K.  Returns (dq, dk), fp64 [N,128]."""
    dqhat = np.ascontiguousarray(dqhat, dtype=np.float64)
    dkhat = np.ascontiguousarray(dkhat, dtype=np.float64)
    N = dqhat.shape[0]
    dq, dk = np.empty((N, 128), np.float64), np.empty((N, 128), np.float64)
    lib().oracle_ste_grads(_p(dqhat), _p(dkhat), N, flags, _p(dq), _p(dk))
    return dq, dk


def attention_backward(q_codes, q_scales, k_codes, k_scales, v_bits, dO, gq=1.0, gk=1.0, scale=None, flags=0,
                       O=None):
    """Whole training-time backward over [B,H,N,...] quantised Q/K, bf16 V and
    dO: attention gradients at the dequantised Q and K, then the straight-
    through gradients of the bf16 Q and K inputs.  O: optional [B,H,N,128]
    forward output D is taken from.  Returns (dq, dk, dv), fp64 [B,H,N,128]."""
    B, H, N = q_codes.shape[:3]
    out = [np.empty((B, H, N, 128), np.float64) for _ in range(3)]
    for b in range(B):
        for h in range(H):
            qh = dequant(q_codes[b, h], q_scales[b, h], gq)
            kh = dequant(k_codes[b, h], k_scales[b, h], gk)
            dqh, dkh, out[2][b, h] = attention_backward_head(qh, kh, v_bits[b, h], dO[b, h], scale,
                                                             None if O is None else O[b, h])
            out[0][b, h], out[1][b, h] = ste_grads(dqh, dkh, flags)
    return tuple(out)


# -- sampled rows at full length ---------------------------------------------------

def _bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def attention_all_rows(qhat: np.ndarray, khat: np.ndarray, v_bits: np.ndarray, scale=None, chunk: int = 1024):
    """fp64 attention of every query row of one head at lengths where the
    scalar C loop of attention_head is too slow (FastVideo "Pika H3 Flex in
    FastVideo", section "FP4 attention": softmax(scale Q K^T) V over the
    dequantised Q and K).  Each row is its own softmax, so rows are taken
    `chunk` at a time, each by the plain definition (row max subtracted) with
    torch's fp64 CPU matrix products and exponentials.  Inputs and outputs as
    attention_head: (O [N,128] fp64, lse [N] fp64)."""
    import torch

    if scale is None:
        scale = 1.0 / np.sqrt(128.0)
    q = torch.from_numpy(np.ascontiguousarray(qhat, dtype=np.float32)).double()
    kT = torch.from_numpy(np.ascontiguousarray(khat, dtype=np.float32)).double().T.contiguous()
    v = torch.from_numpy(_bf16_bits_to_f64(v_bits))
    N = q.shape[0]
    O = torch.empty((N, 128), dtype=torch.float64)
    lse = torch.empty((N,), dtype=torch.float64)
    buf = torch.empty((min(chunk, N), kT.shape[1]), dtype=torch.float64)  # reused: no fresh pages per chunk
    for r0 in range(0, N, chunk):
        r1 = min(N, r0 + chunk)
        s = buf[: r1 - r0]
        torch.mm(q[r0:r1], kT, out=s)  # scores, then P in place
        s.mul_(scale)
        m = s.max(dim=1, keepdim=True).values
        s.sub_(m).exp_()
        l = s.sum(dim=1)
        O[r0:r1] = (s @ v) / l[:, None]
        lse[r0:r1] = m[:, 0] + torch.log(l)
    return O.numpy(), lse.numpy()


def attention_backward_rows(qhat: np.ndarray, khat: np.ndarray, v_bits: np.ndarray, dO: np.ndarray, O: np.ndarray,
                            O_exact: np.ndarray, lse: np.ndarray, rows_q, rows_k, scale=None, flags: int = 0):
    """Sampled rows of one head's training-time gradients -- what
    attention_backward_head followed by ste_grads gives -- at lengths where
    the N x N arrays are out of reach.  With P_ij = exp(scale qhat_i.khat_j -
    lse_i), D_i = dO_i.O_i from the supplied forward output O, and
    dS_ij = P_ij (dO_i.v_j - D_i):
      query rows i:  dQ^_i = scale sum_j dS_ij khat_j,
      key rows j:    dK^_j = scale sum_i dS_ij qhat_i,  dv_j = sum_i P_ij dO_i,
    then dq = c H dQ^ and dk = c H (dK^ - mean_k dK^_k), as in ste_grads.
    The key mean needs every row sum of dS; since the P_ij of a row sum to 1
    and sum_j P_ij v_j is the exact output, sum_j dS_ij = dO_i.O_exact_i - D_i
    (an exact rewrite of the sum), so the mean costs O(N d).  O_exact, lse:
    the exact forward of attention_all_rows.  Returns (dq [|rows_q|,128],
    dk [|rows_k|,128], dv [|rows_k|,128]), fp64."""
    import torch

    if scale is None:
        scale = 1.0 / np.sqrt(128.0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    q = torch.from_numpy(np.ascontiguousarray(qhat, dtype=np.float32)).double()
    k = torch.from_numpy(np.ascontiguousarray(khat, dtype=np.float32)).double()
    v = torch.from_numpy(_bf16_bits_to_f64(v_bits))
    g, Of, Oe, L = t(dO), t(O), t(O_exact), t(lse)
    I = torch.from_numpy(np.asarray(rows_q, dtype=np.int64))
    J = torch.from_numpy(np.asarray(rows_k, dtype=np.int64))
    N = q.shape[0]
    D = (g * Of).sum(dim=1)
    # query rows
    P = torch.exp((q[I] @ k.T) * scale - L[I][:, None])
    dS = P * (g[I] @ v.T - D[I][:, None])
    dqh = (dS @ k) * scale
    # key rows (the transposed products)
    PT = torch.exp((k[J] @ q.T) * scale - L[None, :])
    dST = PT * (v[J] @ g.T - D[None, :])
    dkh = (dST @ q) * scale
    dv = PT @ g
    if not flags & NO_SMOOTH_K:
        rowsum = (g * Oe).sum(dim=1) - D
        dkh = dkh - (rowsum @ q) * (scale / N)
    # the rotation of ste_grads; the centring is done above
    dq, _ = ste_grads(dqh.numpy(), np.zeros(dqh.shape), flags | NO_SMOOTH_K)
    _, dk = ste_grads(np.zeros(dkh.shape), dkh.numpy(), flags | NO_SMOOTH_K)
    return dq, dk, dv.numpy()
