"""Pins for the CPU oracle, checked against things other than the oracle itself.

Each test names what fixes the expected value: a number printed on the pages
(fixtures under tests/golden/), a closed form, an identity from the pages, an
invariance, finite differences, or a library routine used only as a cross-check.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MODES = [(False, -1), (True, -1), (False, 1), (True, 2), (False, 0)]


def _worked():
    with open(os.path.join(GOLDEN, "worked_example_n4_d2.json")) as f:
        g = json.load(f)
    q = np.array(g["Q"], float)[None, None]
    k = np.array(g["K"], float)[None, None]
    v = np.array(g["V"], float)[None, None]
    return g, q, k, v


def _rand(shape, seed, dtype=np.float64):
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


# --------------------------------------------------------------------------
# Worked example N=4, d=2 ("Flash attention and efficient attention", worked
# example "Flash Attention Forward Pass (Simplified)").
# --------------------------------------------------------------------------
def test_worked_example_output_row0():
    g, q, k, v = _worked()
    tol = g["tolerance"]
    o, lse = ref.forward(q, k, v, 1 / math.sqrt(2))
    np.testing.assert_allclose(o[0, 0, 0], g["merged"]["O"], atol=tol)
    # l printed relative to the row maximum m = 1/sqrt(2): l = exp(LSE - m)
    m = 1 / math.sqrt(2)
    assert abs(math.exp(lse[0, 0, 0] - m) - g["merged"]["l"]) < tol
    np.testing.assert_allclose(o[0, 0, 0] * math.exp(lse[0, 0, 0] - m),
                               g["merged"]["numerator"], atol=tol)


def test_worked_example_block_statistics_merge_to_oracle():
    """Block stats (Step 2) and the merge (Step 3), restated here, against the
    printed numbers and against the oracle's two-pass result."""
    g, q, k, v = _worked()
    tol = g["tolerance"]
    s = (q[0, 0, 0] @ k[0, 0].T) / math.sqrt(2)
    blocks = []
    for bi, name in enumerate(("block1", "block2")):
        sb = s[2 * bi: 2 * bi + 2]
        m = sb.max()
        e = np.exp(sb - m)
        l = e.sum()
        ot = e @ v[0, 0, 2 * bi: 2 * bi + 2]
        exp_ = g[name]
        np.testing.assert_allclose(sb, exp_["scores"], atol=tol)
        assert abs(m - exp_["m"]) < tol and abs(l - exp_["l"]) < tol
        np.testing.assert_allclose(e, exp_["exps"], atol=tol)
        np.testing.assert_allclose(ot, exp_["Otilde"], atol=tol)
        blocks.append((m, l, ot))
    (m1, l1, o1), (m2, l2, o2) = blocks
    mn = max(m1, m2)
    l = math.exp(m1 - mn) * l1 + math.exp(m2 - mn) * l2
    o = (math.exp(m1 - mn) * o1 + math.exp(m2 - mn) * o2) / l
    assert abs(l - g["merged"]["l"]) < tol
    o_ref, lse_ref = ref.forward(q, k, v, 1 / math.sqrt(2))
    np.testing.assert_allclose(o, o_ref[0, 0, 0], rtol=0, atol=1e-14)
    assert abs(mn + math.log(l) - lse_ref[0, 0, 0]) < 1e-14


def test_worked_example_rescale_factor_and_row_sums():
    g, q, k, v = _worked()
    assert abs(math.exp(1 / math.sqrt(2) - math.sqrt(2)) - g["rescale_example"]["factor"]) < 1e-3
    o, lse = ref.forward(q, k, v, 1 / math.sqrt(2))
    # every V row sums to 2, softmax weights sum to 1 -> every O row sums to 2
    np.testing.assert_allclose(o[0, 0].sum(axis=1), 2.0, atol=1e-14)
    # derived pin: LSE of row 0 = 1/sqrt(2) + ln(2 * (1 + e^{-1/sqrt 2}))
    assert abs(lse[0, 0, 0] - (1 / math.sqrt(2) + math.log(2 * (1 + math.exp(-1 / math.sqrt(2)))))) < 1e-14
    assert abs(lse[0, 0, 0] - 1.801087) < 1e-6


def test_local_window_mask_matches_page_table():
    rows = [l for l in open(os.path.join(GOLDEN, "local_window_n6_w3.txt")) if not l.startswith("#")]
    table = np.array([[int(x) for x in r.split()] for r in rows if r.strip()], dtype=bool)
    # the page's w = 3 (itself + one neighbour per side) is half-width 1
    got = ref.allowed(np.arange(6), np.arange(6), causal=False, window=1)
    assert table.shape == (6, 6)
    assert (got == table).all()


# --------------------------------------------------------------------------
# Identities from the pages
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal,window", MODES)
def test_merge_identity_any_split(causal, window):
    """Step 3 merge of per-block (m, l, Otilde), for every split point of the key
    axis and for a three-way split, equals the oracle's two-pass result."""
    n, d = 23, 5
    q, k, v = _rand((1, 1, n, d), 1), _rand((1, 1, n, d), 2), _rand((1, 1, n, d), 3)
    scale = 0.7
    o_ref, lse_ref = ref.forward(q, k, v, scale, causal, window)
    s = scale * (q[0, 0] @ k[0, 0].T)
    ok = ref.allowed(np.arange(n), np.arange(n), causal, window)
    s = np.where(ok, s, -np.inf)

    def block(lo, hi):
        sb = s[:, lo:hi]
        m = sb.max(axis=1)
        ms = np.where(np.isfinite(m), m, 0.0)
        e = np.exp(sb - ms[:, None])
        return m, e.sum(axis=1), e @ v[0, 0, lo:hi]

    def merge(parts):
        mn = np.max([p[0] for p in parts], axis=0)
        fac = [np.where(np.isfinite(p[0]), np.exp(np.where(np.isfinite(p[0]), p[0], 0.0) - mn), 0.0)
               for p in parts]
        l = sum(f * p[1] for f, p in zip(fac, parts))
        o = sum(f[:, None] * p[2] for f, p in zip(fac, parts)) / l[:, None]
        return o, mn + np.log(l)

    splits = [[(0, c), (c, n)] for c in range(1, n)] + [[(0, 5), (5, 13), (13, n)]]
    for sp in splits:
        o, lse = merge([block(lo, hi) for lo, hi in sp])
        np.testing.assert_allclose(o, o_ref[0, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref[0, 0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,window", MODES)
def test_probability_rows_sum_to_one_and_zero_where_masked(causal, window):
    n, d = 17, 4
    q, k = _rand((n, d), 4), _rand((n, d), 5)
    rows = np.arange(n)
    p, m, l = ref.attention_probs(q, k, 0.5, rows, rows, causal, window)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    ok = ref.allowed(rows, rows, causal, window)
    assert (p[~ok] == 0).all()
    assert (p[ok] > 0).all()


def test_no_allowed_key_row():
    p, m, l = ref.attention_probs(np.ones((1, 2)), np.ones((1, 2)), 1.0,
                                  np.array([0]), np.array([5]), True, -1)
    assert (p == 0).all() and m[0] == -np.inf and l[0] == 0


def test_permutation_invariance_noncausal():
    b, h, n, d = 1, 2, 19, 6
    q, k, v, do = (_rand((b, h, n, d), s) for s in (10, 11, 12, 13))
    perm = np.random.default_rng(7).permutation(n)
    o1, l1 = ref.forward(q, k, v, 0.4)
    o2, l2 = ref.forward(q, k[:, :, perm], v[:, :, perm], 0.4)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)
    dq1, dk1, dv1 = ref.backward(q, k, v, do, 0.4)
    dq2, dk2, dv2 = ref.backward(q, k[:, :, perm], v[:, :, perm], do, 0.4)
    np.testing.assert_allclose(dq1, dq2, atol=1e-12)
    np.testing.assert_allclose(dk1[:, :, perm], dk2, atol=1e-12)
    np.testing.assert_allclose(dv1[:, :, perm], dv2, atol=1e-12)


# --------------------------------------------------------------------------
# Closed forms and special cases
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal,window", MODES)
def test_zero_queries_give_mean_of_allowed_values(causal, window):
    n, d = 13, 3
    q = np.zeros((1, 1, n, d))
    k, v = _rand((1, 1, n, d), 20), _rand((1, 1, n, d), 21)
    o, lse = ref.forward(q, k, v, 1.3, causal, window)
    for i in range(n):
        keys = [j for j in range(n) if (not causal or j <= i) and (window < 0 or abs(i - j) <= window)]
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, keys].mean(axis=0), atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(len(keys))) < 1e-14


def test_causal_first_row_is_first_value():
    n, d = 9, 4
    q, k, v = (_rand((1, 1, n, d), s) for s in (30, 31, 32))
    o, lse = ref.forward(q, k, v, 0.9, causal=True)
    np.testing.assert_array_equal(o[0, 0, 0], v[0, 0, 0])
    assert lse[0, 0, 0] == 0.9 * float(q[0, 0, 0] @ k[0, 0, 0])


def test_single_allowed_key_gives_zero_dq():
    n, d = 7, 3
    q, k, v, do = (_rand((1, 1, n, d), s) for s in (40, 41, 42, 43))
    o, lse = ref.forward(q, k, v, 0.8, window=0)
    np.testing.assert_array_equal(o, v)
    dq, dk, dv = ref.backward(q, k, v, do, 0.8, window=0)
    np.testing.assert_array_equal(dq, 0.0)
    np.testing.assert_array_equal(dk, 0.0)
    np.testing.assert_array_equal(dv, do)


def test_row_dot_equals_do_dot_o():
    """D_i = sum_j P_ij dP_ij equals dO_i . O_i (the shortcut the GPU uses)."""
    n, d = 15, 5
    q, k, v, do = (_rand((n, d), s) for s in (50, 51, 52, 53))
    rows = np.arange(n)
    p, _, _ = ref.attention_probs(q, k, 0.6, rows, rows, True, 3)
    o = p @ v
    dp = do @ v.T
    np.testing.assert_allclose(ref.row_dot(p, dp), (do * o).sum(axis=1), atol=1e-12)


def test_gqa_equals_repeated_kv_heads():
    b, h, hkv, n, d = 1, 4, 2, 11, 3
    q, do = _rand((b, h, n, d), 60), _rand((b, h, n, d), 61)
    k, v = _rand((b, hkv, n, d), 62), _rand((b, hkv, n, d), 63)
    kr, vr = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
    o1, l1 = ref.forward(q, k, v, 0.5, True)
    o2, l2 = ref.forward(q, kr, vr, 0.5, True)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)
    dq1, dk1, dv1 = ref.backward(q, k, v, do, 0.5, True)
    dq2, dk2, dv2 = ref.backward(q, kr, vr, do, 0.5, True)
    np.testing.assert_allclose(dq1, dq2, atol=1e-14)
    np.testing.assert_allclose(dk1, dk2.reshape(b, hkv, 2, n, d).sum(axis=2), atol=1e-13)
    np.testing.assert_allclose(dv1, dv2.reshape(b, hkv, 2, n, d).sum(axis=2), atol=1e-13)


def test_row_blocking_does_not_change_values():
    n, d = 37, 4
    q, k, v, do = (_rand((1, 2, n, d), s) for s in (70, 71, 72, 73))
    for causal, window in MODES:
        o1, l1 = ref.forward(q, k, v, 0.5, causal, window, row_block=5)
        o2, l2 = ref.forward(q, k, v, 0.5, causal, window)
        np.testing.assert_allclose(o1, o2, atol=1e-14)
        np.testing.assert_allclose(l1, l2, atol=1e-14)
        g1 = ref.backward(q, k, v, do, 0.5, causal, window, row_block=6)
        g2 = ref.backward(q, k, v, do, 0.5, causal, window)
        for a, b in zip(g1, g2):
            np.testing.assert_allclose(a, b, atol=1e-13)


# --------------------------------------------------------------------------
# Backward against central finite differences of L = sum(dO * O)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal,window", MODES)
@pytest.mark.parametrize("g", [1, 2])
def test_backward_matches_finite_differences(causal, window, g):
    b, hkv, n, d = 1, 1, 6, 3
    h = hkv * g
    q, do = _rand((b, h, n, d), 80), _rand((b, h, n, d), 81)
    k, v = _rand((b, hkv, n, d), 82), _rand((b, hkv, n, d), 83)
    scale = 0.75
    dq, dk, dv = ref.backward(q, k, v, do, scale, causal, window)

    def loss(q_, k_, v_):
        o, _ = ref.forward(q_, k_, v_, scale, causal, window)
        return float((o * do).sum())

    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = loss(args["q"], args["k"], args["v"])
            args[name] = xm
            lm = loss(args["q"], args["k"], args["v"])
            num[idx] = (lp - lm) / (2 * eps)
        err = np.abs(num - grad).max() / max(1.0, np.abs(grad).max())
        assert err < 1e-6, (name, err)


# --------------------------------------------------------------------------
# Library cross-check (never the oracle itself)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal,window", MODES)
def test_forward_agrees_with_torch_sdpa_fp64(causal, window):
    b, h, n, d = 1, 2, 64, 16
    q, k, v = (torch.randn(b, h, n, d, dtype=torch.float64, generator=torch.Generator().manual_seed(s))
               for s in (90, 91, 92))
    mask = torch.from_numpy(ref.allowed(np.arange(n), np.arange(n), causal, window))
    want = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=0.3)
    o, _ = ref.forward(q, k, v, 0.3, causal, window)
    np.testing.assert_allclose(o, want.numpy(), atol=1e-12)


def test_forward_agrees_with_torch_sdpa_at_fp32_workload_shape():
    """Same shape as the fp32 workload (N=256, d=64, scale 1/8)."""
    gen = torch.Generator().manual_seed(5)
    q, k, v, do = (torch.randn(1, 1, 256, 64, dtype=torch.float64, generator=gen) for _ in range(4))
    qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
    want = torch.nn.functional.scaled_dot_product_attention(qr, kr, vr, scale=0.125)
    want.backward(do)
    o, _ = ref.forward(q, k, v, 0.125)
    np.testing.assert_allclose(o, want.detach().numpy(), atol=1e-12)
    dq, dk, dv = ref.backward(q, k, v, do, 0.125)
    np.testing.assert_allclose(dq, qr.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, kr.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, vr.grad.numpy(), atol=1e-11)


# --------------------------------------------------------------------------
# Block-sparse masks (128 x 128 blocks)
# --------------------------------------------------------------------------
def test_block_mask_all_ones_equals_dense():
    n, d = 300, 8
    q, k, v, do = (_rand((1, 2, n, d), s) for s in (100, 101, 102, 103))
    nb = (n + 127) // 128
    ones = np.ones((nb, nb), dtype=np.uint8)
    for causal, window in MODES:
        o1, l1 = ref.forward(q, k, v, 0.3, causal, window)
        o2, l2 = ref.forward(q, k, v, 0.3, causal, window, block_mask=ones)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)
        g1 = ref.backward(q, k, v, do, 0.3, causal, window)
        g2 = ref.backward(q, k, v, do, 0.3, causal, window, block_mask=ones)
        for a, b in zip(g1, g2):
            np.testing.assert_array_equal(a, b)


def test_block_diagonal_mask_equals_independent_blocks():
    """With only diagonal blocks on, each 128-row block is its own attention
    problem: the result equals the dense oracle run on each block alone."""
    n, d = 333, 6
    q, k, v, do = (_rand((1, 1, n, d), s) for s in (110, 111, 112, 113))
    nb = (n + 127) // 128
    diag = np.eye(nb, dtype=np.uint8)
    o, lse = ref.forward(q, k, v, 0.4, block_mask=diag)
    dq, dk, dv = ref.backward(q, k, v, do, 0.4, block_mask=diag)
    for bi in range(nb):
        sl = slice(128 * bi, min(n, 128 * (bi + 1)))
        ob, lb = ref.forward(q[:, :, sl], k[:, :, sl], v[:, :, sl], 0.4)
        gq, gk, gv = ref.backward(q[:, :, sl], k[:, :, sl], v[:, :, sl], do[:, :, sl], 0.4)
        np.testing.assert_allclose(o[:, :, sl], ob, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, sl], lb, atol=1e-13)
        np.testing.assert_allclose(dq[:, :, sl], gq, atol=1e-13)
        np.testing.assert_allclose(dk[:, :, sl], gk, atol=1e-13)
        np.testing.assert_allclose(dv[:, :, sl], gv, atol=1e-13)


def test_block_mask_fully_masked_rows_and_per_head_masks():
    n, d = 260, 4
    q, k, v, do = (_rand((1, 2, n, d), s) for s in (120, 121, 122, 123))
    bm = np.zeros((1, 2, 3, 3), dtype=np.uint8)
    bm[0, 0] = np.tril(np.ones((3, 3)))
    bm[0, 1, 0, 0] = 1  # head 1: only block (0, 0); rows >= 128 see nothing
    o, lse = ref.forward(q, k, v, 0.5, block_mask=bm)
    assert np.all(o[0, 1, 128:] == 0) and np.all(lse[0, 1, 128:] == -np.inf)
    dq, dk, dv = ref.backward(q, k, v, do, 0.5, block_mask=bm)
    assert np.all(dq[0, 1, 128:] == 0)
    o_dense, _ = ref.forward(q[:, 1:2, :128], k[:, 1:2, :128], v[:, 1:2, :128], 0.5)
    np.testing.assert_allclose(o[0, 1, :128], o_dense[0, 0], atol=1e-13)
    # head 0: block-causal mask = causal at block granularity, a superset of causal
    o_c, _ = ref.forward(q[:, :1], k[:, :1], v[:, :1], 0.5, causal=True, block_mask=bm[:, :1])
    o_cc, _ = ref.forward(q[:, :1], k[:, :1], v[:, :1], 0.5, causal=True)
    np.testing.assert_allclose(o_c, o_cc, atol=1e-13)


# --------------------------------------------------------------------------
# Padding / variable lengths
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal,window", MODES)
def test_seqlens_equal_truncated_problems(causal, window):
    """Each batch entry with L_b valid tokens equals the attention of its
    first L_b rows alone; padded rows are zero (LSE -inf), and whatever the
    padding holds does not matter."""
    b, h, n, d = 3, 2, 40, 5
    q, k, v, do = (_rand((b, h, n, d), s) for s in (130, 131, 132, 133))
    lens = [40, 17, 1]
    o, lse = ref.forward(q, k, v, 0.6, causal, window, seqlens=lens)
    gq, gk, gv = ref.backward(q, k, v, do, 0.6, causal, window, seqlens=lens)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for bi, L in enumerate(lens):  # garbage in the padding
        q2[bi, :, L:] = 1e3
        k2[bi, :, L:] = -1e3
        v2[bi, :, L:] = 7.0
    o2, lse2 = ref.forward(q2, k2, v2, 0.6, causal, window, seqlens=lens)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    for bi, L in enumerate(lens):
        ob, lb = ref.forward(q[bi:bi + 1, :, :L], k[bi:bi + 1, :, :L], v[bi:bi + 1, :, :L], 0.6, causal, window)
        np.testing.assert_allclose(o[bi:bi + 1, :, :L], ob, atol=1e-14)
        np.testing.assert_allclose(lse[bi:bi + 1, :, :L], lb, atol=1e-14)
        assert np.all(o[bi, :, L:] == 0) and np.all(lse[bi, :, L:] == -np.inf)
        g = ref.backward(q[bi:bi + 1, :, :L], k[bi:bi + 1, :, :L], v[bi:bi + 1, :, :L], do[bi:bi + 1, :, :L], 0.6,
                         causal, window)
        np.testing.assert_allclose(gq[bi:bi + 1, :, :L], g[0], atol=1e-13)
        np.testing.assert_allclose(gk[bi:bi + 1, :, :L], g[1], atol=1e-13)
        np.testing.assert_allclose(gv[bi:bi + 1, :, :L], g[2], atol=1e-13)
        assert np.all(gq[bi, :, L:] == 0) and np.all(gk[bi, :, L:] == 0) and np.all(gv[bi, :, L:] == 0)


# --------------------------------------------------------------------------
# Fewer queries than keys (decode): query i sits at position Nk - Nq + i
# ("FlashAttention" guide page, "Key takeaways": generation needs its own kernel
# mapping, with the same computation).
# --------------------------------------------------------------------------
def test_decode_brute_force_tiny():
    """Each query row written out with explicit loops: softmax over the keys its
    position may see, then the weighted sum of V rows."""
    nq, nk, d, scale = 2, 5, 3, 0.7
    q, k, v = (_rand((1, 1, n, d), s) for n, s in ((nq, 140), (nk, 141), (nk, 142)))
    for causal, window in ((True, -1), (False, 1), (True, 1), (False, -1)):
        o, lse = ref.forward(q, k, v, scale, causal, window)
        for i in range(nq):
            pos = nk - nq + i
            keys = [j for j in range(nk) if (not causal or j <= pos) and (window < 0 or abs(pos - j) <= window)]
            s = [scale * sum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(d)) for j in keys]
            mx = max(s)
            w = [math.exp(x - mx) for x in s]
            tot = sum(w)
            for c in range(d):
                want = sum(wj * v[0, 0, j, c] for wj, j in zip(w, keys)) / tot
                assert abs(o[0, 0, i, c] - want) < 1e-12
            assert abs(lse[0, 0, i] - (mx + math.log(tot))) < 1e-12


@pytest.mark.parametrize("causal,window", MODES)
def test_decode_rows_are_the_last_rows_of_the_full_problem(causal, window):
    """The Nq newest queries against all Nk keys give exactly the last Nq rows
    of the Nk x Nk problem, whatever the earlier queries are."""
    b, h, hkv, nk, nq, d = 2, 4, 2, 37, 5, 6
    k, v = (_rand((b, hkv, nk, d), s) for s in (143, 144))
    q_full = _rand((b, h, nk, d), 145)
    o_full, l_full = ref.forward(q_full, k, v, 0.45, causal, window)
    o, lse = ref.forward(q_full[:, :, nk - nq:], k, v, 0.45, causal, window)
    np.testing.assert_allclose(o, o_full[:, :, nk - nq:], atol=1e-14)
    np.testing.assert_allclose(lse, l_full[:, :, nk - nq:], atol=1e-14)


def test_single_newest_query_causal_sees_every_key():
    k, v = (_rand((1, 2, 29, 4), s) for s in (146, 147))
    q = _rand((1, 2, 1, 4), 148)
    oc, lc = ref.forward(q, k, v, 0.5, True)
    of, lf = ref.forward(q, k, v, 0.5, False)
    np.testing.assert_allclose(oc, of, atol=1e-15)
    np.testing.assert_allclose(lc, lf, atol=1e-15)


def test_decode_rejects_more_queries_than_keys():
    with pytest.raises(ValueError):
        ref.forward(_rand((1, 1, 6, 2), 1), _rand((1, 1, 5, 2), 2), _rand((1, 1, 5, 2), 3), 1.0)
