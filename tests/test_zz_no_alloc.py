"""The quantisation entry point that allocates nothing
(fp4attn_quantize_qk_noalloc): for callers that cannot allocate device memory
for a workspace (cudaMalloc may synchronise the whole device, or another
allocator owns the memory), the library's fixed scratch array stands in for
it.  Its results must equal those of fp4attn_quantize_qk with a workspace --
bit for bit, as every prologue result is -- on consecutive calls that share
the scratch.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from nvfp4_precision_b200 import synth

pytestmark = pytest.mark.gpu

KEYS = ("q_codes", "q_scales", "k_codes", "k_scales", "k_mean")


def _fa():
    from nvfp4_precision_b200 import fp4attn
    return fp4attn


def _inputs(name, B, H, N, seed):
    d = synth.generate(synth.custom(name, B, H, N, seed=seed, k_offset_std=2.0, n_outliers=2,
                                    outlier_factor=20.0), ("q", "k"))
    return d["q"].cuda(), d["k"].cuda()


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    fa = _fa()
    calls = [("a", 1, 2, 512, 1), ("a", 1, 2, 512, 1), ("b", 2, 3, 1000, 2), ("a", 1, 2, 512, 1)]
    for i, (name, B, H, N, seed) in enumerate(calls):
        q, k = _inputs(name, B, H, N, seed)
        ref = fa.fp4attn_quantize_qk(q, k)
        assert fa.fp4attn_read_status(ref["workspace"]) == 0
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        got = fa.fp4attn_quantize_qk_noalloc(q, k, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {i}: device status {int(status.item())}"
        for key in KEYS:
            assert torch.equal(got[key], ref[key]), f"call {i} ({name}): {key} differs"


def test_noalloc_flags_and_global_scales_match():
    fa = _fa()
    q, k = _inputs("flags", 1, 2, 300, 3)
    gq = torch.tensor([0.37], dtype=torch.float32, device="cuda")
    gk = torch.tensor([3.1], dtype=torch.float32, device="cuda")
    for flags in (fa.NO_SMOOTH_K, fa.NO_HADAMARD, 0):
        ref = fa.fp4attn_quantize_qk(q, k, gq, gk, flags=flags)
        got = fa.fp4attn_quantize_qk_noalloc(q, k, gq, gk, flags=flags)
        torch.cuda.synchronize()
        for key in KEYS:
            assert torch.equal(got[key], ref[key]), f"flags={flags}: {key} differs"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    fa = _fa()
    p = torch.empty(16, dtype=torch.uint8, device="cuda")
    ptr = fa._ptr(p)
    rc = fa.lib.fp4attn_quantize_qk_noalloc(ptr, ptr, fa.Shape(1, 1025, 128, 128), None, None, 0,
                                            ptr, ptr, ptr, ptr, None, None, None)
    assert rc == fa.ERR_UNSUPPORTED
    rc = fa.lib.fp4attn_quantize_qk_noalloc(ptr, ptr, fa.Shape(32, 33, 128, 128), None, None, 0,
                                            ptr, ptr, ptr, ptr, None, None, None)
    assert rc == fa.ERR_UNSUPPORTED


def test_noalloc_device_errors_reach_the_status_word_and_are_cleared_by_the_next_call():
    """The shared scratch keeps the last call's contents, so each call must
    clear its status word: a call with a non-finite global scale reports
    FP4ATTN_ERR_RANGE through status_dev, and the good call after it reports 0.
    An empty shape (N = 0) launches nothing and also reports 0."""
    fa = _fa()
    q, k = _inputs("err", 1, 2, 256, 5)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    bad = torch.tensor([float("inf")], dtype=torch.float32, device="cuda")
    fa.fp4attn_quantize_qk_noalloc(q, k, bad, None, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == fa.ERR_RANGE
    ref = fa.fp4attn_quantize_qk(q, k)
    got = fa.fp4attn_quantize_qk_noalloc(q, k, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for key in KEYS:
        assert torch.equal(got[key], ref[key]), f"after an error: {key} differs"
    fa.fp4attn_quantize_qk_noalloc(q, k, bad, None, status=status)
    e = torch.empty((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    fa.fp4attn_quantize_qk_noalloc(e, e, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
