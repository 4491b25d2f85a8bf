"""GPU parity of the padded variable-length entry points: batch entry b holds
seqlens[b] valid tokens; padding (filled with large garbage here) must not
leak, padded rows come out zero (LSE -inf)."""
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


def _lens(n, hi, seed):
    """Seeded lengths in [0, hi], the first three forced to 0, 1 and hi."""
    g = torch.Generator().manual_seed(seed)
    lens = torch.randint(0, hi + 1, (n,), generator=g).tolist()
    lens[:3] = [0, 1, hi]
    return lens


CASES = [
    # name, B, H, Hkv, N, d, dtype, causal, window, lens
    ("causal_d128", 3, 2, 1, 700, 128, "bf16", True, -1, [700, 383, 1]),
    ("full_d64_gqa", 2, 4, 2, 1000, 64, "bf16", False, -1, [130, 999]),
    ("window_d128", 2, 2, 2, 900, 128, "bf16", False, 100, [900, 257]),
    ("zero_length", 2, 1, 1, 300, 64, "bf16", True, -1, [0, 300]),
    ("fp32_causal", 2, 2, 1, 300, 64, "fp32", True, -1, [300, 77]),
    # Many short units (at most a few key tiles each, more units than SMs): the
    # forward runs persistent CTAs over several units each, including padding
    # pairs with no key tile (O = 0, LSE = -inf) and empty sequences.
    ("many_units_causal_d64", 40, 8, 2, 700, 64, "bf16", True, -1, _lens(40, 700, 61)),
    ("many_units_window_d128", 24, 4, 4, 1500, 128, "bf16", False, 64, _lens(24, 1500, 62)),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_varlen_matches_oracle(case):
    name, B, H, Hkv, N, d, dtype, causal, window, lens = case
    w = W.Workload(name, B, H, Hkv, N, d, dtype, causal, window, 51)
    x = W.make_inputs(w)
    for b, L in enumerate(lens):  # garbage in the padding
        for t, val in (("q", 30.0), ("k", -30.0), ("v", 9.0), ("do", 5.0)):
            x[t][b, :, L:] = val
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd_varlen(q, k, v, sl, w.scale, causal, window)
    dq, dk, dv = fa.bwd_varlen(q, k, v, o, lse, do, sl, w.scale, causal, window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    want_o, want_l = ref.forward(x["q"], x["k"], x["v"], w.scale, causal, window, seqlens=lens)
    gq, gk, gv = ref.backward(x["q"], x["k"], x["v"], x["do"], w.scale, causal, window, seqlens=lens)
    got_l = np64(lse)
    dead = ~np.isfinite(want_l)
    assert np.all(np.isneginf(got_l[dead]))
    got_l[dead] = 0.0
    want_l = np.where(dead, 0.0, want_l)
    compare("O", np64(o), want_o, dtype)
    compare("LSE", got_l, want_l, dtype)
    compare("dQ", np64(dq), gq, dtype)
    compare("dK", np64(dk), gk, dtype)
    compare("dV", np64(dv), gv, dtype)
    for b, L in enumerate(lens):
        assert (o[b, :, L:] == 0).all() and (dq[b, :, L:] == 0).all()
        assert (dk[b, :, L:] == 0).all() and (dv[b, :, L:] == 0).all()


def test_varlen_full_lengths_equal_dense():
    w = W.Workload("dense_eq", 2, 2, 1, 600, 128, "bf16", True, -1, 52)
    x = {n: t.cuda() for n, t in W.make_inputs(w).items()}
    sl = torch.tensor([600, 600], dtype=torch.int32, device="cuda")
    o1, l1 = fa.fwd(x["q"], x["k"], x["v"], w.scale, True)
    o2, l2 = fa.fwd_varlen(x["q"], x["k"], x["v"], sl, w.scale, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    g1 = fa.bwd(x["q"], x["k"], x["v"], o1, l1, x["do"], w.scale, True)
    g2 = fa.bwd_varlen(x["q"], x["k"], x["v"], o1, l1, x["do"], sl, w.scale, True)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])


def test_varlen_headline_shape_sampled_head():
    w = W.WORKLOADS[W.HEADLINE]
    x = W.make_inputs(w)
    lens = [8192, 5000]
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd_varlen(q, k, v, sl, w.scale, True)
    dq, dk, dv = fa.bwd_varlen(q, k, v, o, lse, do, sl, w.scale, True)
    torch.cuda.synchronize()
    s_ = (slice(1, 2), slice(6, 7))
    want_o, want_l = ref.forward(x["q"][s_], x["k"][s_], x["v"][s_], w.scale, True, seqlens=[5000])
    gq, gk, gv = ref.backward(x["q"][s_], x["k"][s_], x["v"][s_], x["do"][s_], w.scale, True, seqlens=[5000])
    got_l = np64(lse[s_])
    got_l[..., 5000:] = 0.0
    want_l[..., 5000:] = 0.0
    compare("O", np64(o[s_]), want_o, "bf16")
    compare("LSE", got_l, want_l, "bf16")
    compare("dQ", np64(dq[s_]), gq, "bf16")
    compare("dK", np64(dk[s_]), gk, "bf16")
    compare("dV", np64(dv[s_]), gv, "bf16")
