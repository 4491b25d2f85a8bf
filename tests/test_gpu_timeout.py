"""Failure detection on the GPU without a fault: a wait that nothing completes.

With fa_debug_set_stall on, the sm_100a kernels never issue their first tile
load, so every CTA's wait for it runs out after the (shortened) wait limit.  The
call must come back, fa_last_device_status() must report FA_ERR_TIMEOUT, and the
context must stay usable: the next normal call matches the CPU oracle.  No trap,
no device assert, no bad address and no endless loop is involved -- every wait
in the kernels is bounded, and a CTA that gives up drains its own copies and
tensor-core operations before it frees its tensor memory and returns.
"""
import time

import pytest
import torch

import exact_io_aware_online_b200 as fa
from exact_io_aware_online_b200 import _build
from exact_io_aware_online_b200 import workloads as W

from parity_util import check_groups, gpu_run, oracle_groups

FA_ERR_TIMEOUT = 6
LIMIT_NS = 20_000_000  # 20 ms instead of the default two seconds


@pytest.mark.gpu
@pytest.mark.parametrize("d,B,H", [(128, 1, 4), (64, 1, 4), (128, 40, 2)],
                         ids=["d128", "d64", "d128_persistent_forward"])
def test_stalled_load_reports_timeout_then_recovers(d, B, H):
    """B=40 H=2: 160 short units (three key tiles at most) on fewer CTAs than
    units, so the forward runs its persistent kernel and every role leaves
    the unit loop on the abort."""
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    _build.build()
    w = W.Workload(f"stall_d{d}_b{B}", B, H, H // 2, 384, d, "bf16", True, -1, 31)
    x = W.make_inputs(w)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    assert fa.device_status() == 0
    fa.debug_set_wait_limit(LIMIT_NS)
    fa.debug_set_stall(True)
    try:
        t0 = time.perf_counter()
        o, lse = fa.fwd(q, k, v, w.scale, w.causal, w.window)
        assert fa.device_status() == FA_ERR_TIMEOUT  # synchronises: the kernel returned
        o.zero_()
        lse.zero_()
        fa.bwd(q, k, v, o, lse, do, w.scale, w.causal, w.window)
        assert fa.device_status() == FA_ERR_TIMEOUT
        assert time.perf_counter() - t0 < 30.0
    finally:
        fa.debug_set_stall(False)
        fa.debug_set_wait_limit(0)
    assert fa.device_status() == 0  # the status word was cleared by the reads above
    got = gpu_run(w, x)  # asserts a clean status itself
    groups = [(b, kh) for b in sorted({0, w.B - 1}) for kh in range(w.Hkv)]
    want = oracle_groups(w, x, groups)
    check_groups(w, got, want)
