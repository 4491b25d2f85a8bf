"""GPU parity of fa_fwd_decode: Nq <= Nk queries, the newest Nq positions of
the sequence, against the oracle's reading of the same (query i at position
Nk - Nq + i), on seeded synthetic inputs."""
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


def decode_inputs(B, H, Hkv, Nq, Nk, d, seed):
    """Q, K, V in the workloads' recipe (iid N(0,1) from a seeded CPU generator,
    then bf16), with Nq query rows and Nk key rows."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, Nk, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, Nk, d), generator=g).to(torch.bfloat16)
    return q, k, v


CASES = [
    # name, B, H, Hkv, Nq, Nk, d, causal, window, splits
    ("one_token_gqa_d128", 2, 8, 2, 1, 3000, 128, True, -1, 4),
    ("few_tokens_window_d64", 1, 4, 4, 5, 700, 64, False, 100, 3),
    ("ragged_tiles_causal_d128", 1, 2, 1, 300, 1000, 128, True, -1, 2),
    ("full_noncausal_d64", 2, 2, 1, 17, 513, 64, False, -1, 5),
    ("causal_window_d128", 1, 2, 2, 40, 2048, 128, True, 200, 16),
    ("square_one_split", 1, 2, 1, 600, 600, 128, True, -1, 1),
    ("packed_rows_span_pairs", 1, 8, 1, 70, 900, 64, True, 300, 2),   # 8 x 70 packed rows cross 256-row pairs
    ("packed_window_d128", 2, 6, 2, 33, 1500, 128, False, 64, 4),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(case):
    name, B, H, Hkv, Nq, Nk, d, causal, window, S = case
    q, k, v = decode_inputs(B, H, Hkv, Nq, Nk, d, 71)
    o, lse = fa.fwd_decode(q.cuda(), k.cuda(), v.cuda(), S, 1.0 / d ** 0.5, causal, window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    want_o, want_l = ref.forward(q, k, v, 1.0 / d ** 0.5, causal, window)
    compare("O", np64(o), want_o, "bf16")
    compare("LSE", np64(lse), want_l, "bf16")


def test_square_decode_equals_splitkv_bitwise():
    """With Nq == Nk and one query head per kv head (so the packing of query
    heads is the identity) the decode instantiation does exactly what the
    split-KV forward does."""
    w = W.Workload("sq", 2, 4, 4, 900, 128, "bf16", True, -1, 72)
    x = {n: t.cuda() for n, t in W.make_inputs(w).items()}
    o1, l1 = fa.fwd_splitkv(x["q"], x["k"], x["v"], 3, w.scale, True)
    o2, l2 = fa.fwd_decode(x["q"], x["k"], x["v"], 3, w.scale, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_long_cache_sampled_heads():
    """One new token per sequence against a 32768-token cache, B=8, 32 query
    heads on 8 kv heads, d=128, causal; sampled heads against the oracle."""
    B, H, Hkv, Nq, Nk, d = 8, 32, 8, 1, 32768, 128
    q, k, v = decode_inputs(B, H, Hkv, Nq, Nk, d, 73)
    o, lse = fa.fwd_decode(q.cuda(), k.cuda(), v.cuda(), None, 1.0 / d ** 0.5, True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    for b, h in ((0, 0), (3, 13), (7, 31)):
        kh = h // (H // Hkv)
        want_o, want_l = ref.forward(q[b:b + 1, h:h + 1], k[b:b + 1, kh:kh + 1], v[b:b + 1, kh:kh + 1],
                                     1.0 / d ** 0.5, True)
        compare("O", np64(o[b:b + 1, h:h + 1]), want_o, "bf16")
        compare("LSE", np64(lse[b:b + 1, h:h + 1]), want_l, "bf16")
