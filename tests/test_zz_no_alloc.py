"""fa_bwd_noalloc: the backward entry point for callers that cannot allocate
device memory (for example a plugin inside a host application that owns all
device allocations, or a loop where a cudaMalloc is not allowed).  It must give
the same gradients as fa_bwd, whose workspace the caller allocates, while
taking its scratch from the library's fixed built-in array.

This file is collected last on purpose: it runs after every other test, and
passes as well when run on its own in a fresh process.
"""
import ctypes

import pytest
import torch

import exact_io_aware_online_b200 as fa
from exact_io_aware_online_b200 import _build
from exact_io_aware_online_b200 import workloads as W

from parity_util import F32_TOL, GRAD_REL

SCRATCH_BYTES = 16 * 1024 * 1024  # FA_BWD_NOALLOC_SCRATCH_BYTES in include/fa.h
A = 0x7f0000010000  # aligned fake address; rejected calls never touch it


@pytest.fixture(scope="module")
def L():
    _build.build()
    return fa.lib()


def _call_noalloc(L, x, o, lse, grads, w):
    B, H, N, d = x["q"].shape
    dq, dk, dv = grads
    return L.fa_bwd_noalloc(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), o.data_ptr(),
                            x["do"].data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                            B, H, w.Hkv, N, d, ctypes.c_float(w.scale), int(w.causal), w.window,
                            fa.FA_BF16 if w.dtype == "bf16" else fa.FA_FP32,
                            torch.cuda.current_stream().cuda_stream)


def test_noalloc_rejects_problems_beyond_its_scratch(L):
    # bf16, d=128: 520 bytes per padded row; 32256 rows fit, 32384 do not.
    ok_rows, big_rows = 32256, 32384
    assert L.fa_bwd_workspace_size(1, 1, ok_rows, 128, 0) <= SCRATCH_BYTES
    assert L.fa_bwd_workspace_size(1, 1, big_rows, 128, 0) > SCRATCH_BYTES
    args = [A] * 9 + [1, 1, 1, big_rows, 128, ctypes.c_float(0.088), 1, -1, 0, None]
    assert L.fa_bwd_noalloc(*args) == 4  # FA_ERR_WORKSPACE, nothing enqueued
    args = [A] * 9 + [1, 2, 3, 64, 128, ctypes.c_float(0.088), 1, -1, 0, None]
    assert L.fa_bwd_noalloc(*args) == 1  # H % Hkv != 0


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_noalloc_matches_fa_bwd_on_two_calls_in_a_row(L, dtype):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    # The second call is smaller than the first, so it runs over scratch that
    # still holds the first call's values: what must start at zero is cleared
    # by every call itself.
    shapes = ([dict(B=1, H=4, Hkv=2, N=1000, d=128), dict(B=1, H=2, Hkv=1, N=300, d=128)] if dtype == "bf16"
              else [dict(B=1, H=2, Hkv=1, N=256, d=64), dict(B=1, H=1, Hkv=1, N=100, d=64)])
    for call, (seed, shape) in enumerate(zip((21, 22), shapes)):
        w = W.Workload(f"noalloc{call}", shape["B"], shape["H"], shape["Hkv"], shape["N"], shape["d"], dtype,
                       True, -1, seed)
        x = {k: t.cuda() for k, t in W.make_inputs(w).items()}
        o, lse = fa.fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.window)
        want = fa.bwd(x["q"], x["k"], x["v"], o, lse, x["do"], w.scale, w.causal, w.window)
        got = (torch.full_like(x["q"], float("nan")), torch.full_like(x["k"], float("nan")),
               torch.full_like(x["v"], float("nan")))
        assert _call_noalloc(L, x, o, lse, got, w) == 0
        torch.cuda.synchronize()
        assert fa.device_status() == 0
        for name, g, r in zip(("dQ", "dK", "dV"), got, want):
            g, r = g.double(), r.double()
            assert torch.isfinite(g).all(), name
            err = (g - r).abs().max().item()
            if dtype == "fp32":
                assert err <= F32_TOL, (call, name, err)
            else:
                assert err / r.abs().max().item() <= GRAD_REL, (call, name, err)
