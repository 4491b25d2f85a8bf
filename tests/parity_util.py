"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI,
run the CPU oracle on the same seeded inputs, and compare with the stated
tolerances.

Tolerances (the workloads' targets, with the readings needed to apply them):
  fp32 path:  max |x - ref| <= 1e-5 for O, LSE, dQ, dK, dV.
  bf16 path:  O:   |o - ref| <= 1e-2 + ulp_bf16(ref)/2 element-wise (the
                   output is rounded to bf16, and half an ulp of bf16 exceeds
                   1e-2 once |O| >= 4, so the rounding of the stored value is
                   added to the bound);
              LSE: |lse - ref| <= 1e-3 * max(1, |ref|);
              dQ, dK, dV: max |g - ref| / max |ref| <= 2e-2 per tensor.
"""
from __future__ import annotations

import numpy as np
import torch

import exact_io_aware_online_b200 as fa
from exact_io_aware_online_b200 import workloads as W
from oracle import ref

F32_TOL = 1e-5
O_TOL = 1e-2
LSE_REL = 1e-3
GRAD_REL = 2e-2


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 8), 0.0)  # ulp = 2^(e-7); half of it


def np64(t) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def _worst(err, got, want, bound, k=5):
    flat = np.argsort((err - bound).ravel())[::-1][:k]
    rows = []
    for f in flat:
        idx = np.unravel_index(f, err.shape)
        b = bound if np.isscalar(bound) else bound[idx]
        rows.append(f"{tuple(int(i) for i in idx)}: got {got[idx]:.6g} want {want[idx]:.6g} bound {b:.3g}")
    return "; ".join(rows)


def compare(name: str, got: np.ndarray, want: np.ndarray, dtype: str) -> float:
    """Asserts the tolerance for output `name`; returns the headline error."""
    assert got.shape == want.shape, (name, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    err = np.abs(got - want)
    if dtype == "fp32":
        m = float(err.max()) if err.size else 0.0
        assert m <= F32_TOL, f"{name}: max abs err {m:.3e} > {F32_TOL:.3e}; {_worst(err, got, want, F32_TOL)}"
        return m
    if name == "O":
        bound = O_TOL + bf16_half_ulp(want)
        bad = err > bound
        assert not bad.any(), (f"O: {int(bad.sum())} elements over bound, max err {float(err.max()):.3e}; "
                               f"{_worst(err, got, want, bound)}")
        return float(err.max())
    if name == "LSE":
        rel = err / np.maximum(1.0, np.abs(want))
        m = float(rel.max())
        assert m <= LSE_REL, f"LSE: max rel err {m:.3e} > {LSE_REL}"
        return m
    scale = float(np.abs(want).max())
    m = float(err.max()) / (scale if scale > 0 else 1.0)
    assert m <= GRAD_REL, f"{name}: max err / max |ref| = {m:.3e} > {GRAD_REL}"
    return m


def gpu_run(w: W.Workload, inputs: dict, device="cuda"):
    """fwd + bwd through the C ABI; returns dict of device tensors."""
    q, k, v, do = (inputs[n].to(device) for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, w.scale, w.causal, w.window)
    dq, dk, dv = fa.bwd(q, k, v, o, lse, do, w.scale, w.causal, w.window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


def oracle_groups(w: W.Workload, inputs: dict, groups, row_block: int = 2048):
    """Oracle outputs for whole GQA groups: groups = [(b, kv_head), ...].

    Returns {(b, kh): dict(o, lse, dq [g heads], dk, dv)} computed from the
    exact same (bf16-rounded) values the GPU saw.  row_block: the oracle's row
    blocking (it changes no value; small blocks keep a narrow band cheap).
    """
    g = w.H // w.Hkv
    out = {}
    for b, kh in groups:
        hs = slice(kh * g, (kh + 1) * g)
        q = inputs["q"][b:b + 1, hs]
        do = inputs["do"][b:b + 1, hs]
        k = inputs["k"][b:b + 1, kh:kh + 1]
        v = inputs["v"][b:b + 1, kh:kh + 1]
        o, lse = ref.forward(q, k, v, w.scale, w.causal, w.window, row_block=row_block)
        dq, dk, dv = ref.backward(q, k, v, do, w.scale, w.causal, w.window, row_block=row_block)
        out[(b, kh)] = dict(o=o[0], lse=lse[0], dq=dq[0], dk=dk[0, 0], dv=dv[0, 0])
    return out


def check_groups(w: W.Workload, gpu: dict, want: dict) -> dict:
    g = w.H // w.Hkv
    worst = {}
    for (b, kh), r in want.items():
        hs = slice(kh * g, (kh + 1) * g)
        pairs = (("O", np64(gpu["o"][b, hs]), r["o"]), ("LSE", np64(gpu["lse"][b, hs]), r["lse"]),
                 ("dQ", np64(gpu["dq"][b, hs]), r["dq"]), ("dK", np64(gpu["dk"][b, kh]), r["dk"]),
                 ("dV", np64(gpu["dv"][b, kh]), r["dv"]))
        for name, got, exp in pairs:
            e = compare(name, got, exp, w.dtype)
            worst[name] = max(worst.get(name, 0.0), e)
    return worst
