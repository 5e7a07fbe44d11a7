"""GPU parity of the quantisation prologue (smooth K + Hadamard + NVFP4 pack)
and of the device codecs, bit-exact against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_precision_b200 import synth

from gpu_helpers import fa, gpu_prologue, oracle_prologue

pytestmark = pytest.mark.gpu

KEYS = ("q_codes", "q_scales", "k_codes", "k_scales", "k_mean")


def assert_prologue_equal(g, o, what):
    assert g["status"] == 0, f"{what}: device status {g['status']}"
    for key in KEYS:
        if not np.array_equal(g[key], o[key]):
            bad = np.argwhere(g[key] != o[key])
            raise AssertionError(f"{what}: {key} differs at {bad.shape[0]} places, first {bad[:3].tolist()}")


def test_block_scale_quotient_is_the_ieee_quotient_for_every_input():
    """amax / 6 by a multiply and an FMA refinement: with the IEEE divide
    below 2^-123 every non-negative finite fp32 amax gives the IEEE
    quotient's bits, and without it (the prologue's block scale) every amax
    gives the UE4M3 byte of the IEEE quotient."""
    count, first = fa().fp4attn_probe_div6()
    assert count == 0, f"{count} mismatches, first at bits {first:#010x}"


def test_device_codecs_match_oracle_over_every_fp32_bit_pattern():
    """The device E2M1 and UE4M3 conversions against the oracle's codecs on
    every one of the 2^32 fp32 bit patterns except NaNs (which no finite input
    of the prologue produces), both signs, subnormals, zeros and infinities
    included.  UE4M3 is compared on the non-negative half only: the quantiser
    converts t = amax/6/g >= +0, and negative zero keeps its sign bit in E4M3."""
    chunk = 1 << 27
    for c0 in range(0, 1 << 32, chunk):
        bits = np.arange(c0, c0 + chunk, dtype=np.uint64).astype(np.uint32)
        x = bits.view(np.float32)
        keep = ~np.isnan(x)
        xt = torch.from_numpy(x).cuda()
        e2m1, e4m3 = fa().fp4attn_encode_f32(xt)
        e2m1 = e2m1.cpu().numpy()[keep]
        want = oracle.e2m1_encode(x[keep])
        bad = np.nonzero(e2m1 != want)[0]
        assert bad.size == 0, [(hex(int(bits[keep][i])), int(e2m1[i]), int(want[i])) for i in bad[:8]]
        nonneg = keep & ((bits >> 31) == 0)
        if nonneg.any():
            e4 = e4m3.cpu().numpy()[nonneg]
            want4 = oracle.ue4m3_encode(x[nonneg])
            bad = np.nonzero(e4 != want4)[0]
            assert bad.size == 0, [(hex(int(bits[nonneg][i])), int(e4[i]), int(want4[i])) for i in bad[:8]]


@pytest.mark.parametrize("name,B,H,N,extra", [
    ("one_row", 1, 1, 1, {}),
    ("ragged127", 1, 3, 127, dict(k_offset_std=2.0)),
    ("ragged1000", 2, 2, 1000, dict(k_offset_std=2.0, n_outliers=2, outlier_factor=20.0)),
    ("heavy_tail", 1, 4, 4096, dict(dist="student_t3", n_outliers=4, outlier_factor=50.0)),
])
def test_prologue_bit_exact_small(name, B, H, N, extra):
    d = synth.generate(synth.custom(name, B, H, N, seed=100 + N, **extra), ("q", "k"))
    assert_prologue_equal(gpu_prologue(d), oracle_prologue(d), name)


@pytest.mark.parametrize("flags", [0, 1, 2, 3])
def test_prologue_bit_exact_tiny_all_flags(flags):
    d = synth.generate(synth.WORKLOADS["tiny"], ("q", "k"))
    assert_prologue_equal(gpu_prologue(d, flags=flags), oracle_prologue(d, flags=flags), f"tiny flags={flags}")


def test_prologue_bit_exact_global_scales():
    d = synth.generate(synth.WORKLOADS["tiny"], ("q", "k"))
    g = gpu_prologue(d, gq=0.37, gk=3.1)
    o = oracle_prologue(d, gq=np.float32(0.37), gk=np.float32(3.1))
    assert_prologue_equal(g, o, "tiny g!=1")


def test_prologue_bit_exact_mid():
    d = synth.generate(synth.WORKLOADS["mid"], ("q", "k"))
    assert_prologue_equal(gpu_prologue(d), oracle_prologue(d), "mid")


def test_prologue_key_permutation_gives_permuted_codes():
    """The key mean is an exact integer sum: permuting keys permutes the codes."""
    d = synth.generate(synth.custom("perm", 1, 2, 3000, seed=9, k_offset_std=2.0), ("q", "k"))
    g1 = gpu_prologue(d)
    perm = torch.from_numpy(np.random.default_rng(0).permutation(3000))
    d2 = dict(q=d["q"], k=d["k"][:, :, perm].contiguous())
    g2 = gpu_prologue(d2)
    assert np.array_equal(g2["k_mean"], g1["k_mean"])
    assert np.array_equal(g2["k_codes"], g1["k_codes"][:, :, perm.numpy()])
    assert np.array_equal(g2["k_scales"], g1["k_scales"][:, :, perm.numpy()])


@pytest.mark.parametrize("name", ["clip5s", "prologue_stress"])
def test_prologue_bit_exact_full_size(name):
    d = synth.generate(synth.WORKLOADS[name], ("q", "k"))
    assert_prologue_equal(gpu_prologue(d), oracle_prologue(d), name)


def test_dequant_matches_oracle():
    d = synth.generate(synth.WORKLOADS["tiny"], ("q", "k"))
    o = oracle_prologue(d)
    codes = torch.from_numpy(o["k_codes"]).cuda()
    scales = torch.from_numpy(o["k_scales"]).cuda()
    for g in (None, 0.75):
        gt = None if g is None else torch.tensor([g], dtype=torch.float32, device="cuda")
        got = fa().fp4attn_dequant(codes, scales, gt).cpu().numpy()
        want = oracle.dequant(o["k_codes"], o["k_scales"], 1.0 if g is None else g)
        assert np.array_equal(got, want)


def test_range_errors_are_reported():
    d = synth.generate(synth.custom("bad", 1, 1, 256, seed=3), ("q", "k"))
    k = d["k"].clone()
    k[0, 0, 5, 7] = 2.0 ** 21
    assert gpu_prologue(dict(q=d["q"], k=k))["status"] == fa().ERR_RANGE
    q = d["q"].clone()
    q[0, 0, 9, 1] = float("nan")
    assert gpu_prologue(dict(q=q, k=d["k"]))["status"] == fa().ERR_RANGE
    assert gpu_prologue(d, gq=-1.0)["status"] == fa().ERR_RANGE
    assert gpu_prologue(d)["status"] == 0


def test_empty_shapes_are_no_ops():
    q = torch.zeros((1, 0, 128, 128), dtype=torch.bfloat16, device="cuda")
    out = fa().fp4attn_quantize_qk(q, q)
    assert fa().fp4attn_read_status(out["workspace"]) == 0
    q = torch.zeros((2, 3, 0, 128), dtype=torch.bfloat16, device="cuda")
    out = fa().fp4attn_quantize_qk(q, q)
    assert out["q_codes"].numel() == 0


def test_withheld_key_sums_time_out_and_the_kernel_returns():
    """Failure detection without a GPU fault: the prologue runs with its
    key-sum tiles withheld, so every head's K tiles wait for column sums that
    never arrive.  The wait is bounded (1 ms here): the status word must read
    FP4ATTN_ERR_TIMEOUT, the kernel must return, and the context must stay
    usable -- the ordinary prologue right after it is still bit-exact."""
    d = synth.generate(synth.custom("withheld", 1, 3, 1000, seed=11, k_offset_std=2.0), ("q", "k"))
    q, k = d["q"].cuda(), d["k"].cuda()
    assert fa().fp4attn_probe_withheld_key_sums(q, k, 1_000_000) == fa().ERR_TIMEOUT
    torch.cuda.synchronize()
    assert_prologue_equal(gpu_prologue(d), oracle_prologue(d), "after a timed-out launch")
