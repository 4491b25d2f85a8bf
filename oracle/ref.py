"""CPU fp64 oracle for exact softmax attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code with the CUDA library and imports nothing from the package.

What it computes, and where each step is stated:

* Scores, probabilities, output -- "Flash attention and efficient attention",
  section "The Standard Attention Problem": S = Q K^T, P = softmax(S / sqrt(d_k)),
  O = P V.  The scale is an explicit argument (the pages fold 1/sqrt(d_k) into
  the softmax; callers pass 1/sqrt(d) for that reading).
* Safe softmax -- same page, "Derivation: Incremental Softmax", Step 1: the
  row maximum is subtracted before exponentiating.  This oracle is the plain
  two-pass form (max, then exp/sum); the tiled, online form that the GPU runs is
  equal to it in exact arithmetic (page "FlashAttention paper", section
  "Exact, not approximate").
* Masks -- causal keeps keys j <= i ("FlashAttention" guide page, section
  "Tiling through SRAM": a causal mask alters which tiles are visited, never the result of the rule); the local
  window keeps |i - j| <= w, which reproduces the N=6, w=3 matrix of the
  "Flash attention and efficient attention" page, worked example
  "Local Attention Window" (there w counts the token and one neighbour on each
  side, i.e. half-width 1 here).
* Saved softmax metadata -- the per-row natural-log logsumexp of the scaled,
  masked scores, LSE_i = m_i + ln(sum_j exp(S_ij - m_i)).  The pages say only
  that a small amount of per-row softmax state is kept for training
  ("FlashAttention" guide page, "Tiling through SRAM"); this is the plainest
  reading.
* Backward -- the pages say only that S and P are recomputed from Q, K, V
  ("Flash attention and efficient attention", section "Backward Pass:
  Recomputation").  The formulas below are the textbook softmax Jacobian for
  the loss L = sum(dO * O):
      dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij,
      dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
  D is taken from P and dP on purpose (not as rowsum(dO * O)).
* GQA -- query head h reads kv head h // (H / Hkv); the gradients of a kv
  head sum over its query heads.  The guide page only names grouped-query
  attention, so this contiguous grouping is a reading.
* Block-sparse attention -- "FlashAttention paper" page, section "What it does
  not claim": block sparsity is a separate extension of the same algorithm.
  Reading: a 0/1 mask M over 128 x 128 blocks of the score matrix (per head or
  shared), and a key is allowed only if the causal / window predicate holds
  AND M[i // 128][j // 128] = 1.
* Padding / variable lengths -- "FlashAttention" guide page, "Tiling through
  SRAM": padding only alters how the tiles are laid out, not what is computed.  Reading: batch entry b
  holds L_b <= N valid tokens at the start of its [N, d] rows; keys >= L_b are
  never attended to and padded query rows (>= L_b) give O = 0, LSE = -inf and
  zero gradients, i.e. each batch entry is the attention of its first L_b
  rows alone.
* Fully masked rows (impossible in the shipped dense workloads, where the
  diagonal is always allowed; possible under a block mask) give O = 0,
  LSE = -inf and zero gradients.
* Fewer queries than keys (decode) -- "FlashAttention" guide page, "Key
  takeaways": processing a whole prompt and generating one token at a time
  call for different kernels that compute the same thing.  Reading:
  the Nq queries are the newest Nq tokens of a length-Nk sequence, so query i
  sits at position Nk - Nq + i and the causal / window predicate is applied to
  that position (forward only; Nq <= Nk).

Implementation notes, none of which changes a value: rows are processed in
blocks (each row's softmax is still computed over its whole key range at once),
and with a causal or window mask only keys that can be allowed for a block are
materialised; every other key contributes exactly zero.
"""
from __future__ import annotations

import numpy as np

__all__ = ["allowed", "attention_probs", "forward", "backward", "row_dot"]


BLOCK = 128  # block size of block-sparse masks (rows and columns)


def allowed(rows: np.ndarray, cols: np.ndarray, causal: bool, window: int, block_mask=None) -> np.ndarray:
    """Boolean mask a[i, j]: may query ``rows[i]`` attend to key ``cols[j]``?

    causal -> j <= i; window >= 0 -> |i - j| <= window; window = -1 -> no band;
    block_mask (2-D 0/1 array over 128 x 128 blocks) -> block (i//128, j//128) on.
    """
    r = np.asarray(rows)[:, None]
    c = np.asarray(cols)[None, :]
    ok = np.ones((r.shape[0], c.shape[1]), dtype=bool)
    if causal:
        ok &= c <= r
    if window >= 0:
        ok &= np.abs(r - c) <= window
    if block_mask is not None:
        bm = np.asarray(block_mask).astype(bool)
        ok &= bm[(r // BLOCK), (c // BLOCK)]
    return ok


def _key_range(r0: int, r1: int, n: int, causal: bool, window: int) -> tuple[int, int]:
    lo, hi = 0, n
    if causal:
        hi = min(hi, r1)
    if window >= 0:
        lo = max(lo, r0 - window)
        hi = min(hi, r1 + window)
    return lo, max(lo, hi)


def _scores(q_rows, k_keys, scale, rows, keys, causal, window, block_mask=None):
    s = scale * (q_rows @ k_keys.T)
    ok = allowed(rows, keys, causal, window, block_mask)
    s = np.where(ok, s, -np.inf)
    return s, ok


def attention_probs(q_rows, k_keys, scale, rows, keys, causal, window, block_mask=None):
    """Safe softmax of the masked, scaled scores of one head.

    Returns (P, m, l): P[i, j] probabilities, m the row max of the scaled
    scores, l = sum_j exp(S_ij - m_i).  Rows with no allowed key get P = 0,
    m = -inf, l = 0.
    """
    s, ok = _scores(q_rows, k_keys, scale, rows, keys, causal, window, block_mask)
    m = s.max(axis=1) if s.shape[1] else np.full(s.shape[0], -np.inf)
    dead = ~np.isfinite(m)
    m_safe = np.where(dead, 0.0, m)
    e = np.where(ok, np.exp(s - m_safe[:, None]), 0.0)
    l = e.sum(axis=1)
    p = np.where(l[:, None] > 0, e / np.where(l > 0, l, 1.0)[:, None], 0.0)
    return p, m, l


def _as64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor; upcast exactly from its dtype
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def _heads(q, k):
    b, h, n, d = q.shape
    hkv = k.shape[1]
    if h % hkv:
        raise ValueError("H must be a multiple of Hkv")
    return b, h, hkv, n, d, h // hkv


def _head_mask(block_mask, b, h):
    if block_mask is None:
        return None
    bm = np.asarray(block_mask)
    return bm if bm.ndim == 2 else bm[b, h]


def forward(q, k, v, scale: float, causal: bool = False, window: int = -1,
            heads=None, row_block: int = 2048, block_mask=None, seqlens=None):
    """O [B,H,Nq,d] and LSE [B,H,Nq] in fp64.

    q: [B,H,Nq,d]; k, v: [B,Hkv,Nk,d] with Nq <= Nk (Nq < Nk: decode reading
    above).  ``heads`` optionally restricts the work to a list of (b, h) pairs;
    other heads are left as NaN.  ``block_mask``: 0/1 over 128 x 128 blocks,
    shape [nb, nb] (all heads) or [B, H, nb, nb].  ``seqlens``: optional [B]
    valid lengths (padding reading above).  Both need Nq == Nk.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    b_, h_, _, nq_full, d, g = _heads(q, k)
    nk_full = k.shape[2]
    if nq_full > nk_full or (nq_full != nk_full and (seqlens is not None or block_mask is not None)):
        raise ValueError("need Nq <= Nk, and Nq == Nk with seqlens or a block mask")
    qoff = nk_full - nq_full  # position of query row 0
    o = np.full(q.shape, np.nan)
    lse = np.full(q.shape[:3], np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(b_) for h in range(h_)]
    for b, h in todo:
        kvh = h // g
        nq = nq_full if seqlens is None else int(seqlens[b])
        nk = nk_full if seqlens is None else int(seqlens[b])
        o[b, h, nq:] = 0.0
        lse[b, h, nq:] = -np.inf
        for r0 in range(0, nq, row_block):
            r1 = min(nq, r0 + row_block)
            lo, hi = _key_range(qoff + r0, qoff + r1, nk, causal, window)
            rows, keys = np.arange(qoff + r0, qoff + r1), np.arange(lo, hi)
            p, m, l = attention_probs(q[b, h, r0:r1], k[b, kvh, lo:hi], scale,
                                      rows, keys, causal, window, _head_mask(block_mask, b, h))
            o[b, h, r0:r1] = p @ v[b, kvh, lo:hi]
            with np.errstate(divide="ignore"):
                lse[b, h, r0:r1] = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return o, lse


def row_dot(p: np.ndarray, dp: np.ndarray) -> np.ndarray:
    """D_i = sum_j P_ij dP_ij (the softmax-Jacobian row term)."""
    return (p * dp).sum(axis=1)


def backward(q, k, v, do, scale: float, causal: bool = False, window: int = -1,
             heads=None, row_block: int = 2048, block_mask=None, seqlens=None):
    """dQ [B,H,N,d], dK and dV [B,Hkv,N,d] of L = sum(dO * O), in fp64.

    S and P are recomputed from Q and K (no saved forward state is used).
    With ``heads`` only those (b, h) query heads contribute: dQ of other heads
    is NaN and dK/dV hold only the listed heads' contributions.
    """
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    b_, h_, _, n_full, d, g = _heads(q, k)
    dq = np.full(q.shape, np.nan)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    todo = heads if heads is not None else [(b, h) for b in range(b_) for h in range(h_)]
    for b, h in todo:
        kvh = h // g
        n = n_full if seqlens is None else int(seqlens[b])
        dq[b, h, n:] = 0.0
        for r0 in range(0, n, row_block):
            r1 = min(n, r0 + row_block)
            lo, hi = _key_range(r0, r1, n, causal, window)
            rows, keys = np.arange(r0, r1), np.arange(lo, hi)
            kk, vv = k[b, kvh, lo:hi], v[b, kvh, lo:hi]
            qq, dd = q[b, h, r0:r1], do[b, h, r0:r1]
            p, _, _ = attention_probs(qq, kk, scale, rows, keys, causal, window, _head_mask(block_mask, b, h))
            dv[b, kvh, lo:hi] += p.T @ dd
            dp = dd @ vv.T
            ds = p * (dp - row_dot(p, dp)[:, None])
            dq[b, h, r0:r1] = scale * (ds @ kk)
            dk[b, kvh, lo:hi] += scale * (ds.T @ qq)
    return dq, dk, dv
