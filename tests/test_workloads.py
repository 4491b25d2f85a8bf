"""Host-side checks of the workload table and the seeded generator."""
import numpy as np
import pytest
import torch

from exact_io_aware_online_b200 import workloads as W
from oracle import ref


@pytest.mark.parametrize("n", [1, 2, 7, 64, 130])
@pytest.mark.parametrize("causal,window", [(False, -1), (True, -1), (False, 0), (False, 3), (True, 5), (False, 200)])
def test_allowed_pairs_closed_form(n, causal, window):
    brute = int(ref.allowed(np.arange(n), np.arange(n), causal, window).sum())
    assert W.allowed_pairs(n, causal, window) == brute


def test_window_workload_pair_count():
    w = W.WORKLOADS["bf16_window128_h16_n32768_d64"]
    assert W.allowed_pairs(w.N, w.causal, w.window) == 8_404_864


def test_headline_flops():
    w = W.WORKLOADS[W.HEADLINE]
    fwd, bwd = W.flops(w)
    assert fwd == 4 * 8192 ** 2 * 128 / 2 * 32
    assert bwd == 2.5 * fwd


def test_generator_is_seeded_and_rounded():
    w = W.WORKLOADS["fp32_n256_d64"].with_(dtype="bf16", N=32)
    a = W.make_inputs(w)
    b = W.make_inputs(w)
    for k in ("q", "k", "v", "do"):
        assert a[k].dtype == torch.bfloat16
        assert torch.equal(a[k], b[k])
    g = torch.Generator("cpu").manual_seed(w.seed)
    q = torch.randn((1, 1, 32, 64), generator=g)
    assert torch.equal(a["q"], q.to(torch.bfloat16))


def test_boosted_rows():
    w = W.WORKLOADS["bf16_gqa_causal_h32kv8_n16384_d128"].with_(N=256, dtype="fp32")
    x = W.make_inputs(w)
    norms = x["k"].reshape(-1, 128).norm(dim=1)
    big = int((norms > 40).sum())
    assert big == round(0.01 * 8 * 256)


@pytest.mark.parametrize("N,causal,density", [(300, True, 0.5), (300, False, 0.5), (1000, True, 0.3), (129, False, 1.0)])
def test_block_pairs_matches_brute_force(N, causal, density):
    m = W.block_mask(N, density, 3, causal)
    brute = int(ref.allowed(np.arange(N), np.arange(N), causal, -1, m).sum())
    assert W.block_pairs(N, m, causal) == brute
