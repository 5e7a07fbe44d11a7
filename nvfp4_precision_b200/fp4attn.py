"""Python binding of the CUDA library's C ABI (include/fp4attn.h).

Argument marshalling only: every step of the path runs in the library's
kernels.  torch supplies device memory and the current stream.  Importing
this module loads ``libfp4attn.so`` and raises if it is missing -- there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# FP4ATTN_BOUNDS_CHECK=1 selects the bounds-checked build of the same library
# (build.py --checked): every kernel checks its global stores, atomics and tile
# coordinates and reports FP4ATTN_ERR_RANGE instead of an out-of-range access.
LIB_PATH = os.path.join(_PKG, "libfp4attn_checked.so" if os.environ.get("FP4ATTN_BOUNDS_CHECK") == "1"
                        else "libfp4attn.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_CUDA = 3
ERR_RANGE = 4
ERR_TIMEOUT = 5
ERR_WORKSPACE = 6
NO_SMOOTH_K = 1
NO_HADAMARD = 2
DYNAMIC_GSCALE = 4

EXPORTS = (
    "fp4attn_workspace_bytes", "fp4attn_quantize_qk", "fp4attn_quantize_qk_ex", "fp4attn_quantize_qk_noalloc",
    "fp4attn_forward", "fp4attn_forward_ex", "fp4attn_forward_bf16qk", "fp4attn_forward_bf16qk_ex",
    "fp4attn_dequant", "fp4attn_dequant_bf16", "fp4attn_backward", "fp4attn_backward_ex",
    "fp4attn_backward_workspace_bytes",
    "fp4attn_read_status", "fp4attn_reset_status", "fp4attn_status_string", "fp4attn_encode_f32",
    "fp4attn_probe_qk_tile", "fp4attn_probe_pv_tile", "fp4attn_probe_wait_timeout", "fp4attn_probe_div6",
    "fp4attn_probe_withheld_key_sums", "fp4attn_probe_mma_rate",
)


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("D", ctypes.c_int32)]


class Strides(ctypes.Structure):
    """Element strides (b, h, n) of a [B,H,N,128] tensor whose channels are contiguous."""
    _fields_ = [("b", ctypes.c_int64), ("h", ctypes.c_int64), ("n", ctypes.c_int64)]


class Fp4AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library {LIB_PATH} is missing; build it with "
                          f"`python -m nvfp4_precision_b200.build` (there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, U32, U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64
    L.fp4attn_workspace_bytes.restype = ctypes.c_size_t
    L.fp4attn_workspace_bytes.argtypes = [Shape]
    L.fp4attn_quantize_qk.restype = ctypes.c_int
    L.fp4attn_quantize_qk.argtypes = [P, P, Shape, P, P, U32, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.fp4attn_quantize_qk_ex.restype = ctypes.c_int
    L.fp4attn_quantize_qk_ex.argtypes = [P, Strides, P, Strides, Shape, P, P, U32, P, P, P, P, P, P,
                                         ctypes.c_size_t, P]
    L.fp4attn_forward_ex.restype = ctypes.c_int
    L.fp4attn_forward_ex.argtypes = [P, P, P, P, P, P, P, Strides, Shape, ctypes.c_float, P, Strides, P, P,
                                     ctypes.c_size_t, P]
    L.fp4attn_forward_bf16qk_ex.restype = ctypes.c_int
    L.fp4attn_forward_bf16qk_ex.argtypes = [P, Strides, P, Strides, P, Strides, Shape, ctypes.c_float, P, Strides,
                                            P, P, ctypes.c_size_t, P]
    L.fp4attn_quantize_qk_noalloc.restype = ctypes.c_int
    L.fp4attn_quantize_qk_noalloc.argtypes = [P, P, Shape, P, P, U32, P, P, P, P, P, P, P]
    L.fp4attn_forward.restype = ctypes.c_int
    L.fp4attn_forward.argtypes = [P, P, P, P, P, P, P, Shape, ctypes.c_float, P, P, P, ctypes.c_size_t, P]
    L.fp4attn_forward_bf16qk.restype = ctypes.c_int
    L.fp4attn_forward_bf16qk.argtypes = [P, P, P, Shape, ctypes.c_float, P, P, P, ctypes.c_size_t, P]
    L.fp4attn_dequant_bf16.restype = ctypes.c_int
    L.fp4attn_dequant_bf16.argtypes = [P, P, P, Shape, P, P]
    L.fp4attn_backward_workspace_bytes.restype = ctypes.c_size_t
    L.fp4attn_backward_workspace_bytes.argtypes = [Shape]
    L.fp4attn_backward.restype = ctypes.c_int
    L.fp4attn_backward.argtypes = [P, P, P, P, P, P, P, P, P, P, Shape, ctypes.c_float, U32, P, P, P, P,
                                   ctypes.c_size_t, P]
    L.fp4attn_backward_ex.restype = ctypes.c_int
    L.fp4attn_backward_ex.argtypes = [P, P, P, P, P, P, P, P, P, Strides, P, Shape, ctypes.c_float, U32, P, P, P,
                                      P, ctypes.c_size_t, P]
    L.fp4attn_dequant.restype = ctypes.c_int
    L.fp4attn_dequant.argtypes = [P, P, P, Shape, P, P]
    L.fp4attn_read_status.restype = ctypes.c_int
    L.fp4attn_read_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int)]
    L.fp4attn_reset_status.restype = ctypes.c_int
    L.fp4attn_reset_status.argtypes = [P, P]
    L.fp4attn_status_string.restype = ctypes.c_char_p
    L.fp4attn_status_string.argtypes = [ctypes.c_int]
    L.fp4attn_encode_f32.restype = ctypes.c_int
    L.fp4attn_encode_f32.argtypes = [P, I64, P, P, P]
    L.fp4attn_probe_qk_tile.restype = ctypes.c_int
    L.fp4attn_probe_qk_tile.argtypes = [P, P, P, P, P, P]
    L.fp4attn_probe_pv_tile.restype = ctypes.c_int
    L.fp4attn_probe_pv_tile.argtypes = [P, P, P, P]
    L.fp4attn_probe_div6.restype = ctypes.c_int
    L.fp4attn_probe_mma_rate.restype = ctypes.c_int
    L.fp4attn_probe_mma_rate.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P]
    L.fp4attn_probe_div6.argtypes = [P, P]
    L.fp4attn_probe_wait_timeout.restype = ctypes.c_int
    L.fp4attn_probe_wait_timeout.argtypes = [P, U64, P]
    L.fp4attn_probe_withheld_key_sums.restype = ctypes.c_int
    L.fp4attn_probe_withheld_key_sums.argtypes = [P, P, Shape, P, P, P, P, P, ctypes.c_size_t, U64, P]
    return L


lib = _load()


def status_string(code: int) -> str:
    return lib.fp4attn_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != OK:
        raise Fp4AttnError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def shape_of(t: torch.Tensor) -> Shape:
    B, H, N, D = t.shape
    return Shape(B, H, N, D)


def strides_of(t: torch.Tensor) -> Strides:
    """Strides of a [B,H,N,128] tensor or view (e.g. ``x.transpose(1, 2)`` of a
    [B,N,H,128] tensor); the channels must be contiguous.  The library checks
    the rest (positive multiples of 8)."""
    assert t.dim() == 4 and t.stride(3) == 1, "the channel dimension must be contiguous"
    return Strides(t.stride(0), t.stride(1), t.stride(2))


def fp4attn_workspace_bytes(B: int, H: int, N: int, D: int = 128) -> int:
    return int(lib.fp4attn_workspace_bytes(Shape(B, H, N, D)))


def new_workspace(B: int, H: int, N: int, device="cuda") -> torch.Tensor:
    n = fp4attn_workspace_bytes(B, H, N)
    return torch.empty(n, dtype=torch.uint8, device=device)


def fp4attn_quantize_qk(q: torch.Tensor, k: torch.Tensor, q_gscale: Optional[torch.Tensor] = None,
                        k_gscale: Optional[torch.Tensor] = None, flags: int = 0, out: Optional[dict] = None,
                        k_mean: bool = True, workspace: Optional[torch.Tensor] = None, stream=None,
                        dynamic_gscale: bool = False) -> dict:
    """Smooth K + Hadamard + NVFP4 pack of bf16 [B,H,N,128] Q and K (any
    strides with contiguous channels).  dynamic_gscale=True computes each
    tensor's global scale from its transformed amax into q_gscale / k_gscale
    (allocated when None) instead of reading them.

    Returns dict(q_codes, q_scales, k_codes, k_scales, k_mean, workspace) and,
    with dynamic_gscale, q_gscale and k_gscale (fp32 device scalars to pass to
    fp4attn_forward)."""
    assert q.dtype == torch.bfloat16 and k.dtype == torch.bfloat16 and q.shape == k.shape
    B, H, N, D = q.shape
    dev = q.device
    if out is None:
        out = dict(q_codes=torch.empty((B, H, N, D // 2), dtype=torch.uint8, device=dev),
                   q_scales=torch.empty((B, H, N, D // 16), dtype=torch.uint8, device=dev),
                   k_codes=torch.empty((B, H, N, D // 2), dtype=torch.uint8, device=dev),
                   k_scales=torch.empty((B, H, N, D // 16), dtype=torch.uint8, device=dev),
                   k_mean=torch.empty((B, H, D), dtype=torch.float32, device=dev) if k_mean else None)
    if workspace is None:
        workspace = new_workspace(B, H, N, dev)
    if dynamic_gscale:
        flags = int(flags) | DYNAMIC_GSCALE
        q_gscale = torch.empty(1, dtype=torch.float32, device=dev) if q_gscale is None else q_gscale
        k_gscale = torch.empty(1, dtype=torch.float32, device=dev) if k_gscale is None else k_gscale
    rc = lib.fp4attn_quantize_qk_ex(_ptr(q), strides_of(q), _ptr(k), strides_of(k), Shape(B, H, N, D),
                                    _ptr(q_gscale), _ptr(k_gscale), int(flags), _ptr(out["q_codes"]),
                                    _ptr(out["q_scales"]), _ptr(out["k_codes"]), _ptr(out["k_scales"]),
                                    _ptr(out.get("k_mean")), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "fp4attn_quantize_qk_ex")
    out["workspace"] = workspace
    if dynamic_gscale:
        out["q_gscale"], out["k_gscale"] = q_gscale, k_gscale
    return out


def fp4attn_quantize_qk_noalloc(q: torch.Tensor, k: torch.Tensor, q_gscale: Optional[torch.Tensor] = None,
                                k_gscale: Optional[torch.Tensor] = None, flags: int = 0, out: Optional[dict] = None,
                                k_mean: bool = True, status: Optional[torch.Tensor] = None, stream=None) -> dict:
    """fp4attn_quantize_qk for callers that cannot allocate a workspace: the
    library's fixed scratch array is used instead (B*H <= 1024).  The outputs
    (and the optional int32 ``status`` tensor receiving the device status)
    are the caller's.  Returns dict(q_codes, q_scales, k_codes, k_scales,
    k_mean, status)."""
    assert q.dtype == torch.bfloat16 and k.dtype == torch.bfloat16 and q.shape == k.shape
    assert q.is_contiguous() and k.is_contiguous()
    B, H, N, D = q.shape
    dev = q.device
    if out is None:
        out = dict(q_codes=torch.empty((B, H, N, D // 2), dtype=torch.uint8, device=dev),
                   q_scales=torch.empty((B, H, N, D // 16), dtype=torch.uint8, device=dev),
                   k_codes=torch.empty((B, H, N, D // 2), dtype=torch.uint8, device=dev),
                   k_scales=torch.empty((B, H, N, D // 16), dtype=torch.uint8, device=dev),
                   k_mean=torch.empty((B, H, D), dtype=torch.float32, device=dev) if k_mean else None)
    rc = lib.fp4attn_quantize_qk_noalloc(_ptr(q), _ptr(k), Shape(B, H, N, D), _ptr(q_gscale), _ptr(k_gscale),
                                         int(flags), _ptr(out["q_codes"]), _ptr(out["q_scales"]),
                                         _ptr(out["k_codes"]), _ptr(out["k_scales"]), _ptr(out.get("k_mean")),
                                         _ptr(status), _stream(stream))
    _check(rc, "fp4attn_quantize_qk_noalloc")
    out["status"] = status
    return out


def fp4attn_forward(q_codes, q_scales, k_codes, k_scales, v: torch.Tensor, q_gscale=None, k_gscale=None,
                    softmax_scale: float = 0.0, o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    want_lse: bool = False, workspace: Optional[torch.Tensor] = None, stream=None):
    """Non-causal attention over NVFP4 Q/K and bf16 V [B,H,N,128] (any strides
    with contiguous channels; so may a caller-supplied O be).  Returns
    (O, lse or None); a new O is contiguous [B,H,N,128]."""
    assert v.dtype == torch.bfloat16
    B, H, N, D = v.shape
    if o is None:
        o = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=v.device)
    assert o.shape == v.shape and o.dtype == torch.bfloat16
    if want_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=v.device)
    if workspace is None:
        workspace = new_workspace(B, H, N, v.device)
        workspace.zero_()
    rc = lib.fp4attn_forward_ex(_ptr(q_codes), _ptr(q_scales), _ptr(k_codes), _ptr(k_scales), _ptr(q_gscale),
                                _ptr(k_gscale), _ptr(v), strides_of(v), Shape(B, H, N, D), float(softmax_scale),
                                _ptr(o), strides_of(o), _ptr(lse), _ptr(workspace), workspace.numel(),
                                _stream(stream))
    _check(rc, "fp4attn_forward_ex")
    return o, lse


def fp4attn_forward_bf16qk(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, softmax_scale: float = 0.0,
                           o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                           want_lse: bool = False, workspace: Optional[torch.Tensor] = None, stream=None):
    """Non-causal attention with bf16 Q, K, V [B,H,N,128] (no quantisation; any
    strides with contiguous channels): the BF16 counterpart of fp4attn_forward.
    Returns (O, lse or None); a new O is contiguous [B,H,N,128]."""
    for t in (q, k, v):
        assert t.dtype == torch.bfloat16 and t.shape == v.shape
    B, H, N, D = v.shape
    if o is None:
        o = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=v.device)
    assert o.shape == v.shape and o.dtype == torch.bfloat16
    if want_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=v.device)
    if workspace is None:
        workspace = new_workspace(B, H, N, v.device)
        workspace.zero_()
    rc = lib.fp4attn_forward_bf16qk_ex(_ptr(q), strides_of(q), _ptr(k), strides_of(k), _ptr(v), strides_of(v),
                                       Shape(B, H, N, D), float(softmax_scale), _ptr(o), strides_of(o), _ptr(lse),
                                       _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "fp4attn_forward_bf16qk_ex")
    return o, lse


def fp4attn_dequant(codes: torch.Tensor, scales: torch.Tensor, gscale: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    B, H, N, C = codes.shape  # C = D / 2 code bytes per row
    out = torch.empty((B, H, N, 2 * C), dtype=torch.float32, device=codes.device)
    rc = lib.fp4attn_dequant(_ptr(codes), _ptr(scales), _ptr(gscale), Shape(B, H, N, 2 * C), _ptr(out),
                             _stream(stream))
    _check(rc, "fp4attn_dequant")
    return out


def fp4attn_dequant_bf16(codes: torch.Tensor, scales: torch.Tensor, gscale: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """NVFP4 [B,H,N,D/2] codes + [B,H,N,D/16] scales -> bf16 [B,H,N,D] values."""
    B, H, N, C = codes.shape
    out = torch.empty((B, H, N, 2 * C), dtype=torch.bfloat16, device=codes.device)
    rc = lib.fp4attn_dequant_bf16(_ptr(codes), _ptr(scales), _ptr(gscale), Shape(B, H, N, 2 * C), _ptr(out),
                                  _stream(stream))
    _check(rc, "fp4attn_dequant_bf16")
    return out


def fp4attn_backward_workspace_bytes(B: int, H: int, N: int, D: int = 128) -> int:
    return int(lib.fp4attn_backward_workspace_bytes(Shape(B, H, N, D)))


def fp4attn_backward(q_codes, q_scales, k_codes, k_scales, v, o, dout, lse, softmax_scale: float = 0.0,
                     flags: int = 0, workspace: Optional[torch.Tensor] = None, stream=None,
                     q_gscale: Optional[torch.Tensor] = None, k_gscale: Optional[torch.Tensor] = None):
    """Straight-through backward of the FP4 attention (see include/fp4attn.h):
    the forward's NVFP4 Q and K (codes and scales from fp4attn_quantize_qk)
    and global scales (device scalars, None for 1), V, the forward's O, dL/dO
    (one layout of any strides with contiguous channels, e.g. views of
    [B,N,H,128] tensors) and fp32 lse [B,H,N].  Returns (dq, dk, dv,
    workspace): bf16 gradients of the bf16 Q, K, V inputs of the forward, in
    the layout of V."""
    st = strides_of(v)
    for t in (o, dout):
        assert t.dtype == torch.bfloat16 and t.shape == v.shape and t.stride() == v.stride(), \
            "v, o and dout must share one layout"
    assert v.dtype == torch.bfloat16
    assert lse.dtype == torch.float32 and lse.is_contiguous()
    B, H, N, D = v.shape
    assert q_codes.shape == (B, H, N, 64) and k_codes.shape == (B, H, N, 64)
    if workspace is None:
        workspace = torch.empty(fp4attn_backward_workspace_bytes(B, H, N), dtype=torch.uint8, device=v.device)
    dq, dk, dv = (torch.empty_strided(v.shape, v.stride(), dtype=torch.bfloat16, device=v.device) for _ in range(3))
    rc = lib.fp4attn_backward_ex(_ptr(q_codes), _ptr(q_scales), _ptr(k_codes), _ptr(k_scales), _ptr(q_gscale),
                                 _ptr(k_gscale), _ptr(v), _ptr(o), _ptr(dout), st, _ptr(lse), Shape(B, H, N, D),
                                 float(softmax_scale), int(flags), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                 workspace.numel(), _stream(stream))
    _check(rc, "fp4attn_backward_ex")
    return dq, dk, dv, workspace


class FP4AttentionSTE(torch.autograd.Function):
    """Training-time FP4 attention: the inference path forward (quantise,
    FP4 attention), straight-through backward (fp4attn_backward).  The device
    status words of both halves are checked on the host."""

    @staticmethod
    def forward(ctx, q, k, v, softmax_scale=0.0, flags=0, dynamic_gscale=False):
        # any layout with contiguous channels is used as it is (no copies);
        # O is allocated in V's layout, which the backward then uses throughout
        q, k, v = (t if t.stride(3) == 1 and t.stride(0) > 0 else t.contiguous() for t in (q, k, v))
        out = fp4attn_quantize_qk(q, k, flags=flags, k_mean=False, dynamic_gscale=dynamic_gscale)
        gq, gk = out.get("q_gscale"), out.get("k_gscale")
        o = torch.empty_strided(v.shape, v.stride(), dtype=torch.bfloat16, device=v.device)
        o, lse = fp4attn_forward(out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"], v, gq, gk,
                                 softmax_scale=softmax_scale, o=o, want_lse=True, workspace=out["workspace"])
        codes = (out["q_codes"], out["q_scales"], out["k_codes"], out["k_scales"])
        st = fp4attn_read_status(out["workspace"])
        if st != OK:
            raise Fp4AttnError(st, "FP4AttentionSTE.forward (device)")
        ctx.save_for_backward(*codes, v, o, lse, gq, gk)
        ctx.softmax_scale, ctx.flags = softmax_scale, flags
        return o

    @staticmethod
    def backward(ctx, do):
        qc, qs, kc, ks, v, o, lse, gq, gk = ctx.saved_tensors
        do = do.to(torch.bfloat16)
        if do.stride() != v.stride():
            do = torch.empty_strided(v.shape, v.stride(), dtype=torch.bfloat16, device=v.device).copy_(do)
        dq, dk, dv, ws = fp4attn_backward(qc, qs, kc, ks, v, o, do, lse, ctx.softmax_scale, ctx.flags,
                                          q_gscale=gq, k_gscale=gk)
        st = fp4attn_read_status(ws)
        if st != OK:
            raise Fp4AttnError(st, "FP4AttentionSTE.backward (device)")
        return dq, dk, dv, None, None, None


def fp4_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, softmax_scale: float = 0.0,
                  flags: int = 0, dynamic_gscale: bool = False) -> torch.Tensor:
    """Differentiable FP4 attention of bf16 [B,H,N,128] Q, K, V (fake
    quantisation with a straight-through backward); dynamic_gscale selects the
    amax-derived per-tensor scales."""
    return FP4AttentionSTE.apply(q, k, v, softmax_scale, flags, dynamic_gscale)


def fp4attn_read_status(workspace: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int(-1)
    _check(lib.fp4attn_read_status(_ptr(workspace), _stream(stream), ctypes.byref(v)), "fp4attn_read_status")
    return v.value


def fp4attn_reset_status(workspace: torch.Tensor, stream=None):
    _check(lib.fp4attn_reset_status(_ptr(workspace), _stream(stream)), "fp4attn_reset_status")


def fp4attn_encode_f32(x: torch.Tensor, stream=None):
    assert x.dtype == torch.float32 and x.is_contiguous()
    e2m1 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    e4m3 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(lib.fp4attn_encode_f32(_ptr(x), x.numel(), _ptr(e2m1), _ptr(e4m3), _stream(stream)), "fp4attn_encode_f32")
    return e2m1, e4m3


def fp4attn_probe_qk_tile(q_codes, q_scales, k_codes, k_scales, stream=None) -> torch.Tensor:
    s = torch.empty((128, 128), dtype=torch.float32, device=q_codes.device)
    _check(lib.fp4attn_probe_qk_tile(_ptr(q_codes), _ptr(q_scales), _ptr(k_codes), _ptr(k_scales), _ptr(s),
                                     _stream(stream)), "fp4attn_probe_qk_tile")
    return s


def fp4attn_probe_pv_tile(p: torch.Tensor, v: torch.Tensor, stream=None) -> torch.Tensor:
    o = torch.empty((128, 128), dtype=torch.float32, device=p.device)
    _check(lib.fp4attn_probe_pv_tile(_ptr(p), _ptr(v), _ptr(o), _stream(stream)), "fp4attn_probe_pv_tile")
    return o


def fp4attn_probe_div6(stream=None):
    """(number of mismatches, smallest mismatching bit pattern) of the device
    amax / 6 against the IEEE quotient over every non-negative finite fp32."""
    res = torch.zeros(2, dtype=torch.int32, device="cuda")
    _check(lib.fp4attn_probe_div6(_ptr(res), _stream(stream)), "fp4attn_probe_div6")
    r = res.cpu().numpy().view("uint32")
    return int(r[0]), int(r[1])


MMA_RATE_FLOPS_PER_GROUP = {0: 2 * 2 * 128 * 256 * 64, 1: 8 * 2 * 128 * 256 * 16}


def fp4attn_probe_mma_rate(mode: int, reps: int = 40000, stream=None) -> dict:
    """Back-to-back tcgen05 MMA throughput on every SM (mode 0: block-scaled
    FP4 M128 N256 K64; mode 1: BF16 M128 N256 K16), timed by CUDA events on
    the stream, with the SM clock CTA 0 saw: dict(ms, tflops, flop_per_clk_sm,
    sm_mhz)."""
    cycles = torch.zeros(1, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = stream if stream is not None else torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    _check(lib.fp4attn_probe_mma_rate(mode, reps, _ptr(cycles), _ptr(status), _stream(st)), "fp4attn_probe_mma_rate")
    e1.record(st)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    cyc = int(cycles.item())
    if int(status.item()) != 0 or cyc <= 0:
        raise RuntimeError(f"fp4attn_probe_mma_rate: status {int(status.item())}, cycles {cyc}")
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    flops = MMA_RATE_FLOPS_PER_GROUP[mode] * reps
    return {"ms": ms, "tflops": flops * sms / (ms * 1e-3) / 1e12, "flop_per_clk_sm": flops / cyc,
            "sm_mhz": cyc / (ms * 1e3)}


def fp4attn_probe_wait_timeout(limit_ns: int, stream=None) -> int:
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(lib.fp4attn_probe_wait_timeout(_ptr(status), int(limit_ns), _stream(stream)), "fp4attn_probe_wait_timeout")
    return int(status.item())


def fp4attn_probe_withheld_key_sums(q: torch.Tensor, k: torch.Tensor, limit_ns: int, stream=None) -> int:
    """The prologue with its key-sum tiles withheld: returns the device status
    after the run (FP4ATTN_ERR_TIMEOUT when the K tiles' bounded wait gave up)."""
    assert q.dtype == torch.bfloat16 and k.dtype == torch.bfloat16 and q.shape == k.shape
    assert q.is_contiguous() and k.is_contiguous()
    B, H, N, D = q.shape
    dev = q.device
    qc = torch.empty((B, H, N, 64), dtype=torch.uint8, device=dev)
    qs = torch.empty((B, H, N, 8), dtype=torch.uint8, device=dev)
    kc = torch.empty_like(qc)
    ks = torch.empty_like(qs)
    ws = new_workspace(B, H, N)
    _check(lib.fp4attn_probe_withheld_key_sums(_ptr(q), _ptr(k), Shape(B, H, N, D), _ptr(qc), _ptr(qs), _ptr(kc),
                                               _ptr(ks), _ptr(ws), ws.numel(), int(limit_ns), _stream(stream)),
           "fp4attn_probe_withheld_key_sums")
    return fp4attn_read_status(ws)
