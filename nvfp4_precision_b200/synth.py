"""Seeded synthetic inputs for the FP4 attention path.

This module is shared by the CPU oracle's tests and by the CUDA path's tests
and benchmark.  It only draws random numbers and casts them to bf16; it holds
none of the method's arithmetic (no mean, no Hadamard, no quantisation).

The workloads follow the FastVideo "Pika H3 Flex in FastVideo" page, section
"FP4 attention" (long non-causal video+audio sequences, head dim 128) and the
toy heads described there (per-channel key bias, a few scaled-up channels).
Real Flex activations are not available, so these distributions stand in for
them.

Recipe (per config):
  * one ``numpy.random.SeedSequence(seed)`` is spawned into independent child
    streams, in this fixed order: [offset] + [Q heads] + [K heads] + [V heads];
    each child drives a ``Generator(PCG64(child))``;
  * offset stream: the per-channel key offset ``[B, H, 128] ~ N(0, 2^2)``
    (drawn only when the config has one), then the outlier channel indices
    ``choice(128, n_outliers, replace=False)`` (same channels for Q and K and
    for every head);
  * one stream per (tensor, b, h): the ``[N, 128]`` block of that head, drawn
    as float32 standard normals (Student-t with 3 degrees of freedom for the
    heavy-tailed prologue stress config); rows of the audio tail are drawn
    from the same stream and multiplied by the tail standard deviation;
  * Q and K outlier channels are multiplied by the outlier factor; the key
    offset is added to K; everything is cast to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np
import torch

D = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    seed: int
    dist: str = "normal"          # "normal" or "student_t3"
    n_outliers: int = 0
    outlier_factor: float = 1.0
    k_offset_std: float = 0.0     # 0 disables the per-channel key offset
    tail_rows: int = 0            # audio-token tail length (last rows)
    tail_std: float = 1.0
    with_v: bool = True

    @property
    def shape(self):
        return (self.B, self.H, self.N, D)

    def describe(self) -> str:
        return (f"B{self.B} H{self.H} N{self.N} d{D} {self.dist}"
                f" offset_std={self.k_offset_std} outliers={self.n_outliers}x{self.outlier_factor:g}"
                f" tail={self.tail_rows}@{self.tail_std} seed={self.seed}")


# The workloads: tiny correctness, mid, 5-second clip (with a ~1k audio
# tail), 15-second clip (the 109k-token headline), eight heads of it, and the
# heavy-tailed quantisation-prologue stress case.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 512, seed=0, k_offset_std=2.0),
    "mid": Workload("mid", 1, 8, 8192, seed=1, n_outliers=2, outlier_factor=20.0, k_offset_std=2.0),
    "clip5s": Workload("clip5s", 1, 48, 36864, seed=2, n_outliers=2, outlier_factor=20.0,
                       k_offset_std=2.0, tail_rows=1024, tail_std=0.5),
    "clip15s": Workload("clip15s", 1, 48, 109568, seed=3, n_outliers=2, outlier_factor=20.0,
                        k_offset_std=2.0),
    # the 15-second clip's recipe and head length with eight heads: the
    # headline's per-head access pattern in a few GB of device memory, for
    # hardware-counter captures of one launch
    "clip15s_8heads": Workload("clip15s_8heads", 1, 8, 109568, seed=3, n_outliers=2, outlier_factor=20.0,
                               k_offset_std=2.0),
    "prologue_stress": Workload("prologue_stress", 1, 48, 109568, seed=4, dist="student_t3",
                                n_outliers=4, outlier_factor=50.0, with_v=False),
}


def custom(name: str, B: int, H: int, N: int, seed: int, **kw) -> Workload:
    """A workload of any shape with the same recipe (used for edge cases)."""
    return Workload(name, B, H, N, seed, **kw)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _draw_head(child: np.random.SeedSequence, w: Workload, tail: bool) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(child))
    if w.dist == "normal":
        x = g.standard_normal((w.N, D), dtype=np.float32)
    elif w.dist == "student_t3":
        x = g.standard_t(3.0, size=(w.N, D)).astype(np.float32)
    else:
        raise ValueError(f"unknown distribution {w.dist!r}")
    if tail and w.tail_rows > 0:
        x[w.N - w.tail_rows:] *= np.float32(w.tail_std)
    return x


def generate(w: Workload, tensors=("q", "k", "v"), heads=None) -> dict:
    """Return CPU bf16 tensors ``[B, H, N, 128]`` for the requested names.

    The draw for every (tensor, head) comes from its own child stream, so a
    tensor's values do not depend on which other tensors or heads were
    requested.  ``heads`` (flat b*H + h indices) restricts the draw to those
    heads; the result then has shape ``[1, len(heads), N, 128]``.
    """
    BH = w.B * w.H
    root = np.random.SeedSequence(w.seed)
    children = root.spawn(1 + 3 * BH)
    g0 = np.random.Generator(np.random.PCG64(children[0]))
    offset = None
    if w.k_offset_std > 0:
        offset = (g0.standard_normal((BH, D)) * w.k_offset_std).astype(np.float32)
    outl = None
    if w.n_outliers > 0:
        outl = np.sort(g0.choice(D, size=w.n_outliers, replace=False))

    sel = list(range(BH)) if heads is None else [int(h) for h in heads]
    out = {}
    index = {"q": 0, "k": 1, "v": 2}
    for name in tensors:
        if name == "v" and not w.with_v:
            continue
        t = index[name]
        res = torch.empty((len(sel), w.N, D), dtype=torch.bfloat16)

        def work(i, t=t, name=name, res=res):
            bh = sel[i]
            x = _draw_head(children[1 + t * BH + bh], w, tail=True)
            if outl is not None and name in ("q", "k"):
                x[:, outl] *= np.float32(w.outlier_factor)
            if offset is not None and name == "k":
                x += offset[bh][None, :]
            res[i] = torch.from_numpy(x).to(torch.bfloat16)

        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(len(sel))))
        out[name] = res.view(w.B, w.H, w.N, D) if heads is None else res.view(1, len(sel), w.N, D)
    out["outlier_channels"] = outl
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw uint16 bit patterns of a CPU bf16 tensor, as a numpy array."""
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(bits: np.ndarray, shape) -> torch.Tensor:
    """Inverse of :func:`bf16_bits`."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).reshape(shape)


def sample_rows(N: int, per_head: int, seed: int, tail_rows: int = 0, n_tail: int = 0) -> np.ndarray:
    """Seeded query-row sample for large workloads: row 0, row N-1, ``n_tail``
    rows of the audio tail, and the rest uniform without replacement."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 7919])))
    fixed = {0, N - 1}
    if tail_rows and n_tail:
        fixed |= set(int(r) for r in g.choice(np.arange(N - tail_rows, N), size=n_tail, replace=False))
    rest = per_head - len(fixed)
    pool = np.setdiff1d(np.arange(N), np.fromiter(fixed, dtype=np.int64))
    extra = g.choice(pool, size=max(0, rest), replace=False) if rest > 0 else np.array([], dtype=np.int64)
    return np.sort(np.concatenate([np.fromiter(fixed, dtype=np.int64), extra.astype(np.int64)]))


def toy_heads(n_heads: int, seed: int, N: int = 32, d: int = 64, k_bias_std: float = 2.0, n_scaled: int = 2,
              scale_factor: float = 20.0) -> dict:
    """The page's toy heads: ``d`` channels (64: four 16-value blocks), ``N``
    keys and as many queries, Gaussian values, a per-channel key bias shared by
    the keys of a head, and ``n_scaled`` channels scaled up in Q and K.

    Same recipe as :func:`generate` with its own stream order: one
    ``SeedSequence(seed)`` spawned into [bias and channels] + [Q] + [K] + [V];
    the bias ``[n_heads, d] ~ N(0, k_bias_std^2)``, then the scaled channels
    ``choice(d, n_scaled, replace=False)`` (shared by Q, K and every head),
    then Q, K, V ``[n_heads, N, d]`` as float32 standard normals; scale the
    channels, add the bias to K, cast to bf16 (round to nearest even).
    Returns CPU bf16 tensors q, k, v ``[n_heads, N, d]`` and the channels."""
    children = np.random.SeedSequence([seed, 64]).spawn(4)
    g0 = np.random.Generator(np.random.PCG64(children[0]))
    bias = (g0.standard_normal((n_heads, d)) * k_bias_std).astype(np.float32)
    chans = np.sort(g0.choice(d, size=n_scaled, replace=False)) if n_scaled else np.array([], dtype=np.int64)
    out = {}
    for i, name in enumerate(("q", "k", "v")):
        x = np.random.Generator(np.random.PCG64(children[1 + i])).standard_normal((n_heads, N, d), dtype=np.float32)
        if name in ("q", "k") and n_scaled:
            x[:, :, chans] *= np.float32(scale_factor)
        if name == "k":
            x += bias[:, None, :]
        out[name] = torch.from_numpy(x).to(torch.bfloat16)
    out["scaled_channels"] = chans
    return out
