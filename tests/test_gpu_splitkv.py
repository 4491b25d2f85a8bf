"""GPU parity of the split-KV forward (partial online-softmax states per key
chunk, merged with the block-merge identity) against the CPU oracle."""
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


CASES = [
    # name, B, H, Hkv, N, d, causal, window, splits
    ("n1_one_chunk_empty", 1, 1, 1, 1, 64, False, -1, 2),
    ("n1000_causal_s3", 1, 2, 1, 1000, 128, True, -1, 3),
    ("n4096_full_d64_s4", 1, 2, 2, 4096, 64, False, -1, 4),
    ("n700_causal_gqa_s16_many_empty", 2, 4, 2, 700, 128, True, -1, 16),
    ("n2048_window100_s2", 1, 2, 2, 2048, 128, False, 100, 2),
    ("n3000_causal_gqa4_s5", 1, 4, 1, 3000, 128, True, -1, 5),
    ("n1500_causal_window300_d64_s3", 1, 2, 1, 1500, 64, True, 300, 3),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_splitkv_matches_oracle(case):
    name, B, H, Hkv, N, d, causal, window, S = case
    w = W.Workload(name, B, H, Hkv, N, d, "bf16", causal, window, 31)
    x = W.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.fwd_splitkv(q, k, v, S, w.scale, causal, window)
    o1, lse1 = fa.fwd(q, k, v, w.scale, causal, window)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    want_o, want_l = ref.forward(x["q"], x["k"], x["v"], w.scale, causal, window)
    compare("O", np64(o), want_o, "bf16")
    compare("LSE", np64(lse), want_l, "bf16")
    # and close to the unsplit kernel (same tolerance against each other)
    compare("O", np64(o), np64(o1).astype("float64"), "bf16")


def test_splitkv_is_deterministic():
    w = W.Workload("det", 1, 2, 1, 1300, 128, "bf16", True, -1, 32)
    x = {n: t.cuda() for n, t in W.make_inputs(w).items()}
    a = fa.fwd_splitkv(x["q"], x["k"], x["v"], 4, w.scale, True)
    b = fa.fwd_splitkv(x["q"], x["k"], x["v"], 4, w.scale, True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_splitkv_small_batch_long_sequence_sampled_head():
    w = W.WORKLOADS["bf16_causal_b1h2_n16384_d128"]
    x = W.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.fwd_splitkv(q, k, v, 4, w.scale, True)
    torch.cuda.synchronize()
    want_o, want_l = ref.forward(x["q"][:, 1:2], x["k"][:, 1:2], x["v"][:, 1:2], w.scale, True)
    compare("O", np64(o[:, 1:2]), want_o, "bf16")
    compare("LSE", np64(lse[:, 1:2]), want_l, "bf16")
