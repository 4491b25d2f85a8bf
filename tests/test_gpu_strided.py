"""GPU parity of the strided-layout entry points (fa_fwd_strided /
fa_bwd_strided): [B, N, H, d] ("BSHD") buffers, slices of longer buffers and
outputs with a padded row pitch.  The layout only changes addressing, so the
results must equal the oracle within the usual tolerances and, for the
deterministic outputs (O, LSE, dK, dV), equal the contiguous path bit for bit."""
import numpy as np
import pytest
import torch

import exact_io_aware_online_b200 as fa
from exact_io_aware_online_b200 import workloads as W

from parity_util import compare, np64
from oracle import ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from exact_io_aware_online_b200 import _build
    _build.build()
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


def bshd(t):
    """Device copy of a [B, h, N, d] tensor stored as [B, N, h, d], returned as a [B, h, N, d] view."""
    B, h, N, d = t.shape
    buf = torch.empty((B, N, h, d), dtype=t.dtype, device="cuda")
    buf.copy_(t.transpose(1, 2))
    return buf.transpose(1, 2)


def oracle_check(x, w, causal, window, o, lse, dq, dk, dv, lens=None):
    want_o, want_l = ref.forward(x["q"], x["k"], x["v"], w.scale, causal, window, seqlens=lens)
    gq, gk, gv = ref.backward(x["q"], x["k"], x["v"], x["do"], w.scale, causal, window, seqlens=lens)
    got_l = np64(lse)
    dead = ~np.isfinite(want_l)
    assert np.all(np.isneginf(got_l[dead]))
    got_l[dead] = 0.0
    want_l = np.where(dead, 0.0, want_l)
    compare("O", np64(o), want_o, w.dtype)
    compare("LSE", got_l, want_l, w.dtype)
    compare("dQ", np64(dq), gq, w.dtype)
    compare("dK", np64(dk), gk, w.dtype)
    compare("dV", np64(dv), gv, w.dtype)


CASES = [
    # name, B, H, Hkv, N, d, dtype, causal, window
    ("bshd_causal_gqa_d128", 2, 4, 2, 700, 128, "bf16", True, -1),
    ("bshd_full_d64", 2, 3, 3, 520, 64, "bf16", False, -1),
    ("bshd_window_d128", 1, 2, 1, 900, 128, "bf16", False, 100),
    ("bshd_fp32_d64", 2, 2, 1, 300, 64, "fp32", True, -1),
    # more units than SMs, five key tiles each at most: the persistent forward on 4-D maps
    ("bshd_many_units_causal_d128", 16, 8, 4, 1000, 128, "bf16", True, -1),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_bshd_matches_oracle_and_contiguous_path(case):
    name, B, H, Hkv, N, d, dtype, causal, window = case
    w = W.Workload(name, B, H, Hkv, N, d, dtype, causal, window, 61)
    x = W.make_inputs(w)
    q, k, v, do = (bshd(x[n]) for n in ("q", "k", "v", "do"))
    assert q.stride() == (N * H * d, d, H * d, 1)
    o, lse = fa.fwd_strided(q, k, v, w.scale, causal, window)
    assert o.stride() == q.stride()
    dq, dk, dv = fa.bwd_strided(q, k, v, o, lse, do, w.scale, causal, window)
    assert dq.stride() == q.stride() and dk.stride() == k.stride()
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    oracle_check(x, w, causal, window, o, lse, dq, dk, dv)
    # same arithmetic as the contiguous path
    qc, kc, vc, doc = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o2, l2 = fa.fwd(qc, kc, vc, w.scale, causal, window)
    g2 = fa.bwd(qc, kc, vc, o2, l2, doc, w.scale, causal, window)
    torch.cuda.synchronize()
    assert torch.equal(o.contiguous(), o2) and torch.equal(lse, l2)
    assert torch.equal(dk.contiguous(), g2[1]) and torch.equal(dv.contiguous(), g2[2])


def test_slices_of_longer_buffers_and_padded_pitch_outputs():
    """Inputs are the first N rows of [B, h, Ncap, d] buffers (a cache of
    capacity Ncap); outputs go to buffers with a row pitch of d + 64 whose
    extra columns hold a canary that must survive."""
    B, H, Hkv, N, d, Ncap = 2, 4, 1, 650, 128, 1000
    w = W.Workload("slices", B, H, Hkv, N, d, "bf16", True, -1, 62)
    x = W.make_inputs(w)

    def cache(t):
        buf = torch.full((t.shape[0], t.shape[1], Ncap, d), 7.0, dtype=t.dtype, device="cuda")
        buf[:, :, :N] = t.cuda()
        return buf[:, :, :N]

    def pitched(like):
        buf = torch.full((like.shape[0], like.shape[1], N, d + 64), 3.0, dtype=like.dtype, device="cuda")
        return buf, buf[..., :d]

    q, k, v, do = (cache(x[n]) for n in ("q", "k", "v", "do"))
    ob, o = pitched(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    fa.fwd_strided(q, k, v, w.scale, True, out=o, lse=lse)
    (dqb, dq), (dkb, dk), (dvb, dv) = pitched(q), pitched(k), pitched(v)
    fa.bwd_strided(q, k, v, o, lse, do, w.scale, True, grads=(dq, dk, dv))
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    for buf in (ob, dqb, dkb, dvb):
        assert (buf[..., d:] == 3.0).all(), "wrote outside the output layout"
    oracle_check(x, w, True, -1, o, lse, dq, dk, dv)


def test_bshd_with_padded_lengths():
    B, H, Hkv, N, d = 3, 2, 1, 600, 64
    lens = [600, 211, 0]
    w = W.Workload("bshd_varlen", B, H, Hkv, N, d, "bf16", True, -1, 63)
    x = W.make_inputs(w)
    for b, L in enumerate(lens):  # garbage in the padding
        for t, val in (("q", 30.0), ("k", -30.0), ("v", 9.0), ("do", 5.0)):
            x[t][b, :, L:] = val
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    q, k, v, do = (bshd(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd_strided(q, k, v, w.scale, True, seqlens=sl)
    dq, dk, dv = fa.bwd_strided(q, k, v, o, lse, do, w.scale, True, seqlens=sl)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    oracle_check(x, w, True, -1, o, lse, dq, dk, dv, lens=lens)
    for b, L in enumerate(lens):
        assert (o[b, :, L:] == 0).all() and (dq[b, :, L:] == 0).all()
        assert (dk[b, :, L:] == 0).all() and (dv[b, :, L:] == 0).all()


def test_bshd_headline_shape_sampled_head():
    """The causal B=2 H=16 N=8192 d=128 workload in [B, N, H, d] layout; one
    sampled head against the oracle, every output against the contiguous path."""
    w = W.WORKLOADS[W.HEADLINE]
    x = W.make_inputs(w)
    q, k, v, do = (bshd(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd_strided(q, k, v, w.scale, True)
    dq, dk, dv = fa.bwd_strided(q, k, v, o, lse, do, w.scale, True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    qc, kc, vc, doc = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o2, l2 = fa.fwd(qc, kc, vc, w.scale, True)
    g2 = fa.bwd(qc, kc, vc, o2, l2, doc, w.scale, True)
    torch.cuda.synchronize()
    assert torch.equal(o.contiguous(), o2) and torch.equal(lse, l2)
    assert torch.equal(dk.contiguous(), g2[1]) and torch.equal(dv.contiguous(), g2[2])
    s_ = (slice(1, 2), slice(11, 12))
    want_o, want_l = ref.forward(x["q"][s_], x["k"][s_], x["v"][s_], w.scale, True)
    gq, gk, gv = ref.backward(x["q"][s_], x["k"][s_], x["v"][s_], x["do"][s_], w.scale, True)
    compare("O", np64(o[s_]), want_o, "bf16")
    compare("LSE", np64(lse[s_]), want_l, "bf16")
    compare("dQ", np64(dq[s_]), gq, "bf16")
    compare("dK", np64(dk[s_]), gk, "bf16")
    compare("dV", np64(dv[s_]), gv, "bf16")
