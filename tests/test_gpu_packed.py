"""GPU parity of the packed variable-length entry points (fa_fwd_packed /
fa_bwd_packed): sequences concatenated along the token axis, offsets on the
host.  Each sequence must equal the oracle's attention of that sequence alone,
and the deterministic outputs must equal the padded-layout path bit for bit."""
import numpy as np
import pytest
import torch

import exact_io_aware_online_b200 as fa

from parity_util import compare, np64
from oracle import ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from exact_io_aware_online_b200 import _build
    _build.build()
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


def packed_inputs(lens, H, Hkv, d, dtype, seed):
    """q, k, v, dO as [T, heads, d], iid N(0,1) from a seeded CPU generator."""
    T = sum(lens)
    g = torch.Generator("cpu").manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.randn((T, H, d), generator=g).to(dt)
    k = torch.randn((T, Hkv, d), generator=g).to(dt)
    v = torch.randn((T, Hkv, d), generator=g).to(dt)
    do = torch.randn((T, H, d), generator=g).to(dt)
    return q, k, v, do


def offsets(lens):
    return [0] + list(np.cumsum(lens))


CASES = [
    # name, lens, H, Hkv, d, dtype, causal, window
    ("causal_gqa_d128", [700, 1, 0, 383], 4, 2, 128, "bf16", True, -1),
    ("window_d64", [257, 900], 2, 2, 64, "bf16", False, 100),
    ("full_d64_gqa", [130, 64, 999], 2, 1, 64, "bf16", False, -1),
    ("fp32_causal", [300, 77], 2, 1, 64, "fp32", True, -1),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_packed_matches_oracle_per_sequence(case):
    name, lens, H, Hkv, d, dtype, causal, window = case
    q, k, v, do = packed_inputs(lens, H, Hkv, d, dtype, 81)
    cu = offsets(lens)
    scale = 1.0 / d ** 0.5
    o, lse = fa.fwd_packed(q.cuda(), k.cuda(), v.cuda(), cu, scale, causal, window)
    dq, dk, dv = fa.bwd_packed(q.cuda(), k.cuda(), v.cuda(), o, lse, do.cuda(), cu, scale, causal, window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    for b, L in enumerate(lens):
        if L == 0:
            continue
        sl = slice(cu[b], cu[b + 1])
        as4 = lambda t: t[sl].transpose(0, 1).unsqueeze(0)  # noqa: E731  [1, heads, L, d]
        want_o, want_l = ref.forward(as4(q), as4(k), as4(v), scale, causal, window)
        gq, gk, gv = ref.backward(as4(q), as4(k), as4(v), as4(do), scale, causal, window)
        compare("O", np64(as4(o.cpu())), want_o, dtype)
        compare("LSE", np64(lse[H * cu[b]:H * cu[b + 1]].view(1, H, L).cpu()), want_l, dtype)
        compare("dQ", np64(as4(dq.cpu())), gq, dtype)
        compare("dK", np64(as4(dk.cpu())), gk, dtype)
        compare("dV", np64(as4(dv.cpu())), gv, dtype)


def test_packed_equals_padded_lengths_bitwise():
    lens, H, Hkv, d = [600, 1, 383], 4, 2, 128
    q, k, v, do = (t.cuda() for t in packed_inputs(lens, H, Hkv, d, "bf16", 82))
    cu = offsets(lens)
    B, N = len(lens), max(lens)

    def pad(t):
        out = torch.zeros((B, t.shape[1], N, d), dtype=t.dtype, device=t.device)
        for b, L in enumerate(lens):
            out[b, :, :L] = t[cu[b]:cu[b + 1]].transpose(0, 1)
        return out

    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o1, l1 = fa.fwd_packed(q, k, v, cu, causal=True)
    g1 = fa.bwd_packed(q, k, v, o1, l1, do, cu, causal=True)
    qp, kp, vp, dop = pad(q), pad(k), pad(v), pad(do)
    o2, l2 = fa.fwd_varlen(qp, kp, vp, sl, causal=True)
    g2 = fa.bwd_varlen(qp, kp, vp, o2, l2, dop, sl, causal=True)
    torch.cuda.synchronize()
    for b, L in enumerate(lens):
        seg = slice(cu[b], cu[b + 1])
        assert torch.equal(o1[seg].transpose(0, 1), o2[b, :, :L])
        assert torch.equal(l1[H * cu[b]:H * cu[b + 1]].view(H, L), l2[b, :, :L])
        assert torch.equal(g1[1][seg].transpose(0, 1), g2[1][b, :, :L])
        assert torch.equal(g1[2][seg].transpose(0, 1), g2[2][b, :, :L])


def _short_lens(n, hi, seed):
    """n sequence lengths in [0, hi], seeded, with a few empty and one-token ones."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, hi + 1, size=n).tolist()
    lens[0], lens[n // 2], lens[-1] = 0, 1, hi
    return lens


@pytest.mark.parametrize("d,causal,window", [(64, True, -1), (128, False, -1), (64, False, 40)])
def test_many_short_sequences_in_one_launch(d, causal, window):
    """Hundreds of short sequences (tiles that end inside a sequence, empty and
    one-token sequences, sequences that start mid-tile) against the oracle,
    sequence by sequence, with the offsets handed over as a CUDA tensor."""
    lens, H, Hkv = _short_lens(300, 200, 83 + d), 2, 1
    q, k, v, do = packed_inputs(lens, H, Hkv, d, "bf16", 84)
    cu = offsets(lens)
    cu_dev = torch.tensor(cu, dtype=torch.int32, device="cuda")
    scale = 1.0 / d ** 0.5
    o, lse = fa.fwd_packed(q.cuda(), k.cuda(), v.cuda(), cu_dev, scale, causal, window)
    dq, dk, dv = fa.bwd_packed(q.cuda(), k.cuda(), v.cuda(), o, lse, do.cuda(), cu_dev, scale, causal, window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    o, lse, dq, dk, dv = (t.cpu() for t in (o, lse, dq, dk, dv))
    for b, L in enumerate(lens):
        if L == 0:
            continue
        sl = slice(cu[b], cu[b + 1])
        as4 = lambda t: t[sl].transpose(0, 1).unsqueeze(0)  # noqa: E731  [1, heads, L, d]
        want_o, want_l = ref.forward(as4(q), as4(k), as4(v), scale, causal, window)
        gq, gk, gv = ref.backward(as4(q), as4(k), as4(v), as4(do), scale, causal, window)
        compare("O", np64(as4(o)), want_o, "bf16")
        compare("LSE", np64(lse[H * cu[b]:H * cu[b + 1]].view(1, H, L)), want_l, "bf16")
        compare("dQ", np64(as4(dq)), gq, "bf16")
        compare("dK", np64(as4(dk)), gk, "bf16")
        compare("dV", np64(as4(dv)), gv, "bf16")


def test_packed_writes_nothing_outside_its_rows():
    """Outputs sit inside larger buffers holding a sentinel: rows before the
    first token and after the last one (and the logsumexp around its T * H
    values) must keep it, whichever way a tile's rows are stored."""
    lens, H, Hkv, d, pad = [5, 130, 0, 257, 1, 77], 2, 1, 128, 300
    q, k, v, do = (t.cuda() for t in packed_inputs(lens, H, Hkv, d, "bf16", 85))
    cu = offsets(lens)
    T = cu[-1]
    sent = -7.0
    big = lambda heads: torch.full((T + 2 * pad, heads, d), sent, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    ob, dqb, dkb, dvb = big(H), big(H), big(Hkv), big(Hkv)
    lb = torch.full((T * H + 2 * 1024,), sent, dtype=torch.float32, device="cuda")
    mid = slice(pad, pad + T)
    o, lse = fa.fwd_packed(q, k, v, cu, causal=True, out=ob[mid], lse=lb[1024:1024 + T * H])
    fa.bwd_packed(q, k, v, o, lse, do, cu, causal=True, grads=(dqb[mid], dkb[mid], dvb[mid]))
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    for name, t in (("O", ob), ("dQ", dqb), ("dK", dkb), ("dV", dvb)):
        assert bool((t[:pad] == sent).all()) and bool((t[pad + T:] == sent).all()), name
        assert bool(torch.isfinite(t[mid].float()).all()), name
    assert bool((lb[:1024] == sent).all()) and bool((lb[1024 + T * H:] == sent).all())
