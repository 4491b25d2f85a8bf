"""The pins in test_oracle.py are chosen so that plausible mistakes in the
oracle fail at least one of them.  Each case here plants one mistake in a copy
of the oracle's arithmetic (on the CPU, by patching the module under test) and
checks that a pin that does not depend on the oracle itself catches it."""
import math

import numpy as np
import pytest

from oracle import ref

RNG = np.random.default_rng(0)


def _inputs(n=6, d=3, h=1):
    return [RNG.standard_normal((1, h, n, d)) for _ in range(4)]


def _fd_error(fwd, bwd, causal=False, window=-1):
    """max relative error of bwd against central differences of fwd."""
    q, k, v, do = _inputs()
    dq, dk, dv = bwd(q, k, v, do, 0.75, causal, window)
    eps, worst = 1e-6, 0.0
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            args = {"q": q, "k": k, "v": v}
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args[name] = xp
            lp = float((fwd(args["q"], args["k"], args["v"], 0.75, causal, window)[0] * do).sum())
            args[name] = xm
            lm = float((fwd(args["q"], args["k"], args["v"], 0.75, causal, window)[0] * do).sum())
            num[idx] = (lp - lm) / (2 * eps)
        worst = max(worst, np.abs(num - g).max() / max(1.0, np.abs(g).max()))
    return worst


def _worked_example_error(fwd):
    q = np.array([[1, 0], [0, 1], [1, 1], [0, 0]], float)[None, None]
    v = np.array([[1, 1], [2, 0], [0, 2], [1, 1]], float)[None, None]
    o, _ = fwd(q, q, v, 1 / math.sqrt(2))
    return float(np.abs(o[0, 0, 0] - [0.830, 1.170]).max())


def test_unmodified_oracle_passes_the_pins():
    assert _fd_error(ref.forward, ref.backward) < 1e-6
    assert _worked_example_error(ref.forward) < 1e-3


@pytest.mark.parametrize("mutation", ["dS sign", "missing D term", "dK scale", "dQ uses V", "dV transposed"])
def test_backward_mutations_fail_finite_differences(mutation):
    def bwd(q, k, v, do, scale, causal=False, window=-1):
        q, k, v, do = (np.asarray(t, float) for t in (q, k, v, do))
        n = q.shape[2]
        rows = np.arange(n)
        p, _, _ = ref.attention_probs(q[0, 0], k[0, 0], scale, rows, rows, causal, window)
        dp = do[0, 0] @ v[0, 0].T
        dmat = ref.row_dot(p, dp)[:, None]
        ds = p * (dp - dmat)
        if mutation == "dS sign":
            ds = p * (dmat - dp)
        if mutation == "missing D term":
            ds = p * dp
        dq = scale * ds @ (v[0, 0] if mutation == "dQ uses V" else k[0, 0])
        dk = (1.0 if mutation == "dK scale" else scale) * ds.T @ q[0, 0]
        dv = (p @ do[0, 0]) if mutation == "dV transposed" else (p.T @ do[0, 0])
        return dq[None, None], dk[None, None], dv[None, None]

    assert _fd_error(ref.forward, bwd) > 1e-3


@pytest.mark.parametrize("mutation", ["exp(s + m)", "scale dropped", "max as normaliser",
                                      "softmax over queries", "P times Q"])
def test_forward_mutations_fail_a_pin(mutation):
    def fwd(q, k, v, scale, causal=False, window=-1):
        q, k, v = (np.asarray(t, float) for t in (q, k, v))
        s = (1.0 if mutation == "scale dropped" else scale) * (q[0, 0] @ k[0, 0].T)
        axis = 0 if mutation == "softmax over queries" else 1
        m = s.max(axis=axis, keepdims=True)
        e = np.exp(s + m) if mutation == "exp(s + m)" else np.exp(s - m)
        denom = e.max(axis=axis, keepdims=True) if mutation == "max as normaliser" else e.sum(axis=axis, keepdims=True)
        return ((e / denom) @ (q[0, 0] if mutation == "P times Q" else v[0, 0]))[None, None], None

    if mutation == "exp(s + m)":
        # exp(s + m) / sum exp(s + m) is still the softmax in exact arithmetic; the
        # safe-softmax pin (a large logit must not overflow) is what catches it
        q = np.array([[400.0, 0.0]])[None, None]
        with np.errstate(over="ignore", invalid="ignore"):
            o, _ = fwd(q, q, np.ones((1, 1, 1, 2)), 1.0)
        assert not np.isfinite(o).all()
        o_ref, _ = ref.forward(q, q, np.ones((1, 1, 1, 2)), 1.0)
        assert np.isfinite(o_ref).all()
        return
    assert _worked_example_error(fwd) > 1e-3


def test_mask_mutation_fails_the_page_table():
    rows = np.arange(6)
    wrong = np.abs(rows[:, None] - rows[None, :]) < 1  # "< w" instead of "<= w"
    right = ref.allowed(rows, rows, False, 1)
    assert (wrong != right).any()
