"""GPU parity of block-sparse attention (0/1 mask over 128 x 128 blocks)
against the CPU oracle, and against the dense kernels when every block is on."""
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


def _mask(shape, density, seed, empty_row=None, empty_col=None):
    m = (np.random.default_rng(seed).random(shape) < density).astype(np.uint8)
    if empty_row is not None:
        m[..., empty_row, :] = 0
    if empty_col is not None:
        m[..., :, empty_col] = 0
    return m


CASES = [
    # name, B, H, Hkv, N, d, dtype, causal, window, per_head, density
    ("shared_full_d128", 1, 2, 2, 1000, 128, "bf16", False, -1, False, 0.5),
    ("perhead_causal_gqa_d128", 1, 4, 2, 900, 128, "bf16", True, -1, True, 0.6),
    ("perhead_d64_ragged", 2, 2, 1, 777, 64, "bf16", False, -1, True, 0.4),
    ("shared_window_d64", 1, 2, 2, 1500, 64, "bf16", False, 200, False, 0.7),
    ("fp32_perhead_causal", 1, 2, 1, 600, 64, "fp32", True, -1, True, 0.5),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_blocksparse_matches_oracle(case):
    name, B, H, Hkv, N, d, dtype, causal, window, per_head, density = case
    w = W.Workload(name, B, H, Hkv, N, d, dtype, causal, window, 41)
    x = W.make_inputs(w)
    nb = (N + 127) // 128
    shape = (B, H, nb, nb) if per_head else (nb, nb)
    m = _mask(shape, density, 7, empty_row=1, empty_col=nb - 1)  # a query block and a key block fully off
    mt = torch.from_numpy(m).cuda()
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd_blocksparse(q, k, v, mt, w.scale, causal, window)
    dq, dk, dv = fa.bwd_blocksparse(q, k, v, o, lse, do, mt, w.scale, causal, window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    want_o, want_l = ref.forward(x["q"], x["k"], x["v"], w.scale, causal, window, block_mask=m)
    gq, gk, gv = ref.backward(x["q"], x["k"], x["v"], x["do"], w.scale, causal, window, block_mask=m)
    dead = ~np.isfinite(want_l)
    assert dead.any()  # the switched-off query block
    got_l = np64(lse)
    assert np.all(np.isneginf(got_l[dead]))
    got_l[dead] = 0.0
    want_l = np.where(dead, 0.0, want_l)
    compare("O", np64(o), want_o, dtype)
    compare("LSE", got_l, want_l, dtype)
    compare("dQ", np64(dq), gq, dtype)
    compare("dK", np64(dk), gk, dtype)
    compare("dV", np64(dv), gv, dtype)


def test_all_blocks_on_equals_dense_kernels():
    w = W.Workload("dense_eq", 1, 2, 1, 1100, 128, "bf16", True, -1, 42)
    x = {n: t.cuda() for n, t in W.make_inputs(w).items()}
    nb = (w.N + 127) // 128
    ones = torch.ones((nb, nb), dtype=torch.uint8, device="cuda")
    o1, l1 = fa.fwd(x["q"], x["k"], x["v"], w.scale, True)
    o2, l2 = fa.fwd_blocksparse(x["q"], x["k"], x["v"], ones, w.scale, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    g1 = fa.bwd(x["q"], x["k"], x["v"], o1, l1, x["do"], w.scale, True)
    g2 = fa.bwd_blocksparse(x["q"], x["k"], x["v"], o1, l1, x["do"], ones, w.scale, True)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    assert (g1[0].float() - g2[0].float()).abs().max().item() <= 2e-2 * g1[0].float().abs().max().item()


def test_blocksparse_headline_shape_sampled_head():
    w = W.WORKLOADS[W.HEADLINE]
    x = W.make_inputs(w)
    nb = w.N // 128
    m = np.tril(_mask((nb, nb), 0.5, 9))
    np.fill_diagonal(m, 1)
    mt = torch.from_numpy(m).cuda()
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd_blocksparse(q, k, v, mt, w.scale, True)
    dq, dk, dv = fa.bwd_blocksparse(q, k, v, o, lse, do, mt, w.scale, True)
    torch.cuda.synchronize()
    sl = (slice(1, 2), slice(3, 4))
    want_o, want_l = ref.forward(x["q"][sl], x["k"][sl], x["v"][sl], w.scale, True, block_mask=m)
    gq, gk, gv = ref.backward(x["q"][sl], x["k"][sl], x["v"][sl], x["do"][sl], w.scale, True, block_mask=m)
    compare("O", np64(o[sl]), want_o, "bf16")
    compare("LSE", np64(lse[sl]), want_l, "bf16")
    compare("dQ", np64(dq[sl]), gq, "bf16")
    compare("dK", np64(dk[sl]), gk, "bf16")
    compare("dV", np64(dv[sl]), gv, "bf16")
