"""Seeded synthetic inputs and the workload table.

This module holds no attention arithmetic: it only draws random tensors and
describes shapes.  Both the CUDA path (tests, benchmark) and the CPU oracle are
fed from it, so both sides see identical bf16/fp32 values.

Generator (a reading: the workloads give seeds but no generator):
``torch.Generator('cpu').manual_seed(seed)``, then ``torch.randn`` in fp32 in
the order Q, K, V, dO, then rounding to bf16 (round to nearest even) when the
workload is bf16.  For the GQA workload, after the four draws a permutation of
the B*Hkv*N flattened K rows is drawn from the same generator and the first
round(1%) of them are multiplied by 8 before rounding, so that some rows meet
a much larger score late in the key order.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "allowed_pairs", "flops"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Hkv: int
    N: int
    d: int
    dtype: str  # "bf16" or "fp32"
    causal: bool
    window: int  # -1: none; w >= 0: keys with |i-j| <= w
    seed: int
    boost_frac: float = 0.0  # fraction of K rows scaled by 8 (GQA workload)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "fp32_n256_d64": Workload("fp32_n256_d64", 1, 1, 1, 256, 64, "fp32", False, -1, 0),
    "bf16_b4h16_n2048_d64": Workload("bf16_b4h16_n2048_d64", 4, 16, 16, 2048, 64, "bf16", False, -1, 1),
    "bf16_causal_b2h16_n8192_d128": Workload("bf16_causal_b2h16_n8192_d128", 2, 16, 16, 8192, 128,
                                             "bf16", True, -1, 2),
    "bf16_gqa_causal_h32kv8_n16384_d128": Workload("bf16_gqa_causal_h32kv8_n16384_d128", 1, 32, 8,
                                                   16384, 128, "bf16", True, -1, 3, 0.01),
    "bf16_window128_h16_n32768_d64": Workload("bf16_window128_h16_n32768_d64", 1, 16, 16, 32768, 64,
                                              "bf16", False, 128, 4),
    # not one of the stated workloads: a small-batch long-sequence case (too few
    # query blocks to fill the GPU) used to measure the split-KV forward
    "bf16_causal_b1h2_n16384_d128": Workload("bf16_causal_b1h2_n16384_d128", 1, 2, 2, 16384, 128, "bf16", True, -1, 5),
}
HEADLINE = "bf16_causal_b2h16_n8192_d128"


def make_inputs(w: Workload, device="cpu"):
    """Return dict(q, k, v, do) as torch tensors in the workload dtype on ``device``.

    Layouts: q, do [B,H,N,d]; k, v [B,Hkv,N,d]; all contiguous.
    """
    g = torch.Generator("cpu").manual_seed(w.seed)
    q = torch.randn((w.B, w.H, w.N, w.d), generator=g, dtype=torch.float32)
    k = torch.randn((w.B, w.Hkv, w.N, w.d), generator=g, dtype=torch.float32)
    v = torch.randn((w.B, w.Hkv, w.N, w.d), generator=g, dtype=torch.float32)
    do = torch.randn((w.B, w.H, w.N, w.d), generator=g, dtype=torch.float32)
    if w.boost_frac > 0:
        rows = w.B * w.Hkv * w.N
        perm = torch.randperm(rows, generator=g)
        sel = perm[: int(round(w.boost_frac * rows))]
        kf = k.view(rows, w.d)
        kf[sel] *= 8.0
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out = {}
    for name, t in (("q", q), ("k", k), ("v", v), ("do", do)):
        out[name] = t.to(dt).to(device).contiguous()
    return out


def allowed_pairs(N: int, causal: bool, window: int) -> int:
    """Number of (query, key) pairs the mask keeps in one head (closed form)."""
    if window < 0:
        return N * (N + 1) // 2 if causal else N * N
    w = min(window, N - 1)
    if causal:  # keys i-w..i
        return (w + 1) * N - w * (w + 1) // 2
    # keys i-w..i+w clipped to [0, N)
    return (2 * w + 1) * N - w * (w + 1)


def flops(w: Workload) -> tuple[float, float]:
    """(forward, backward) algorithmic flops of the whole workload.

    Forward counts the two matmuls, 4*d flops per kept (query, key) pair; the
    backward counts 2.5x that.  For full and causal masks this is 4*N^2*d per
    head, halved for causal; the metric's own formula halves exactly (N^2/2)
    rather than counting the N/2 diagonal pairs, so causal uses N^2/2.
    """
    heads = w.B * w.H
    if w.window < 0:
        pairs = w.N * w.N / (2.0 if w.causal else 1.0)
    else:
        pairs = float(allowed_pairs(w.N, w.causal, w.window))
    fwd = 4.0 * w.d * pairs * heads
    return fwd, 2.5 * fwd


def block_mask(N: int, density: float, seed: int, causal: bool):
    """Seeded 0/1 mask over 128 x 128 blocks ([nb, nb], uint8) for measuring
    block-sparse attention: each block on with probability `density`; under a
    causal mask the upper triangle is dropped and the diagonal kept on."""
    import numpy as np
    nb = (N + 127) // 128
    m = (np.random.default_rng(seed).random((nb, nb)) < density).astype(np.uint8)
    if causal:
        m = np.tril(m)
        np.fill_diagonal(m, 1)
    return m


def block_pairs(N: int, mask, causal: bool) -> int:
    """(query, key) pairs a causal (or unmasked) attention keeps inside the
    blocks `mask` switches on, for one head."""
    nb = mask.shape[0]
    total = 0
    for i in range(nb):
        ri = min(128, N - 128 * i)
        for j in range(nb):
            if not mask[i, j]:
                continue
            cj = min(128, N - 128 * j)
            if not causal or j < i:
                total += ri * cj if (not causal or j < i) else 0
            elif j == i:
                total += ri * (ri + 1) // 2
    return total
