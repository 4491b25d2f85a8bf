"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol the header declares, and rejects bad arguments on the host before
touching the device (so fake, never-dereferenced pointer values are safe)."""
import ctypes
import subprocess

import pytest

import exact_io_aware_online_b200 as fa
from exact_io_aware_online_b200 import _build

A = 0x7f0000010000  # a 16-byte aligned fake device address (never dereferenced on these paths)


@pytest.fixture(scope="module")
def L():
    _build.build()
    return fa.lib()


def test_header_declares_expected_entry_points():
    names = fa.exported_names()
    for n in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_last_device_status", "fa_status_string",
              "fa_version", "fa_set_timing_events", "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_size", "fa_fwd_blocksparse", "fa_bwd_blocksparse", "fa_fwd_varlen", "fa_bwd_varlen", "fa_fwd_strided", "fa_bwd_strided", "fa_fwd_decode", "fa_fwd_packed", "fa_bwd_packed",
              "fa_fwd_decode_workspace_size", "fa_bwd_packed_workspace_size", "fa_bwd_noalloc",
              "fa_debug_set_wait_limit", "fa_debug_set_stall"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in fa.exported_names():
        assert n in exported, n
        assert getattr(L, n) is not None


def test_status_strings_and_version(L):
    assert L.fa_version() == 101
    for code in range(7):
        assert L.fa_status_string(code)
    assert L.fa_status_string(99) == b"unknown status"


def _fwd(L, **kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=2, Hkv=1, N=16, d=64, scale=0.125, causal=0, window=-1, dtype=0)
    a.update(kw)
    return L.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Hkv"], a["N"], a["d"],
                    ctypes.c_float(a["scale"]), a["causal"], a["window"], a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(v=None), 1), (dict(o=None), 1), (dict(lse=None), 1),
    (dict(B=0), 1), (dict(H=0), 1), (dict(Hkv=0), 1), (dict(N=0), 1), (dict(N=-5), 1),
    (dict(H=3, Hkv=2), 1), (dict(scale=0.0), 1), (dict(scale=-1.0), 1), (dict(scale=float("nan")), 1),
    (dict(scale=float("inf")), 1), (dict(window=-2), 1), (dict(dtype=7), 1),
    (dict(d=32), 2), (dict(d=96), 2), (dict(d=256), 2),
    (dict(q=A + 8), 3), (dict(k=A + 4), 3), (dict(o=A + 2), 3), (dict(lse=A + 12), 3),
])
def test_fwd_rejects_bad_arguments(L, kw, code):
    assert _fwd(L, **kw) == code


def _bwd(L, ws=A, ws_bytes=None, **kw):
    a = dict(B=1, H=2, Hkv=1, N=16, d=64, scale=0.125, causal=0, window=-1, dtype=0)
    a.update(kw)
    if ws_bytes is None:
        ws_bytes = L.fa_bwd_workspace_size(a["B"], a["H"], a["N"], a["d"], a["dtype"] if a["dtype"] in (0, 1) else 0)
    ptrs = [kw.get(n, A) for n in ("q", "k", "v", "o", "do", "lse", "dq", "dk", "dv")]
    return L.fa_bwd(*ptrs, ws, ws_bytes, a["B"], a["H"], a["Hkv"], a["N"], a["d"], ctypes.c_float(a["scale"]),
                    a["causal"], a["window"], a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(do=None), 1), (dict(lse=None), 1), (dict(dq=None), 1), (dict(dv=None), 1),
    (dict(H=4, Hkv=3), 1), (dict(window=-3), 1), (dict(scale=0.0), 1), (dict(d=80), 2),
    (dict(dk=A + 8), 3), (dict(do=A + 4), 3),
    (dict(ws=None), 4), (dict(ws_bytes=16), 4), (dict(ws=A + 8), 3),
])
def test_bwd_rejects_bad_arguments(L, kw, code):
    assert _bwd(L, **kw) == code


def test_bwd_workspace_one_byte_short_is_rejected(L):
    need = L.fa_bwd_workspace_size(2, 4, 300, 128, 0)
    assert _bwd(L, ws_bytes=need - 1, B=2, H=4, Hkv=2, N=300, d=128) == 4


@pytest.mark.parametrize("B,H,N,d", [(1, 1, 1, 64), (2, 16, 8192, 128), (1, 32, 16384, 128), (3, 5, 130, 64)])
def test_workspace_size_closed_form(L, B, H, N, d):
    def a256(x):
        return (x + 255) // 256 * 256
    np_ = (N + 127) // 128 * 128
    rows = B * H * np_
    assert L.fa_bwd_workspace_size(B, H, N, d, 0) == a256(rows * 4) * 2 + a256(rows * d * 4)
    assert L.fa_bwd_workspace_size(B, H, N, d, 1) == a256(B * H * N * 4)
    assert L.fa_bwd_workspace_size(B, H, N, 96, 0) == 0
    assert L.fa_bwd_workspace_size(0, H, N, d, 0) == 0


def test_python_helpers_fail_loudly_without_cuda():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(Exception):
        fa.fwd(q, q, q)


def _split(L, ws=A, ws_bytes=None, **kw):
    a = dict(B=1, H=2, Hkv=1, N=300, d=128, scale=0.088, causal=1, window=-1, splits=3, dtype=0)
    a.update(kw)
    if ws_bytes is None:
        ws_bytes = L.fa_fwd_splitkv_workspace_size(a["B"], a["H"], a["N"], a["d"], max(1, min(16, a["splits"])))
    ptrs = [kw.get(n, A) for n in ("q", "k", "v", "o", "lse")]
    return L.fa_fwd_splitkv(*ptrs, a["B"], a["H"], a["Hkv"], a["N"], a["d"], ctypes.c_float(a["scale"]),
                            a["causal"], a["window"], a["splits"], ws, ws_bytes, a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(lse=None), 1), (dict(splits=0), 1), (dict(splits=17), 1), (dict(H=3, Hkv=2), 1),
    (dict(dtype=1), 2), (dict(d=96), 2), (dict(ws=None), 4), (dict(ws_bytes=100), 4), (dict(ws=A + 8), 3),
    (dict(o=A + 4), 3),
])
def test_splitkv_rejects_bad_arguments(L, kw, code):
    assert _split(L, **kw) == code


@pytest.mark.parametrize("B,H,N,d,S", [(1, 1, 1, 64, 1), (2, 16, 8192, 128, 4), (1, 3, 300, 64, 16)])
def test_splitkv_workspace_closed_form(L, B, H, N, d, S):
    def a256(x):
        return (x + 255) // 256 * 256
    nq2 = (N + 255) // 256 * 256
    assert L.fa_fwd_splitkv_workspace_size(B, H, N, d, S) == a256(S * B * H * nq2 * d * 4) + a256(S * B * H * nq2 * 16)
    assert L.fa_fwd_splitkv_workspace_size(B, H, N, d, 0) == 0
    assert L.fa_fwd_splitkv_workspace_size(B, H, N, d, 17) == 0


def test_blocksparse_rejects_bad_arguments(L):
    f = ctypes.c_float(0.125)
    # null mask, negative stride, misaligned q, bad head ratio
    assert L.fa_fwd_blocksparse(A, A, A, A, A, 1, 2, 1, 300, 64, f, 1, -1, None, 0, 0, None) == 1
    assert L.fa_fwd_blocksparse(A, A, A, A, A, 1, 2, 1, 300, 64, f, 1, -1, A, -1, 0, None) == 1
    assert L.fa_fwd_blocksparse(A + 8, A, A, A, A, 1, 2, 1, 300, 64, f, 1, -1, A, 0, 0, None) == 3
    assert L.fa_fwd_blocksparse(A, A, A, A, A, 1, 3, 2, 300, 64, f, 1, -1, A, 0, 0, None) == 1
    need = L.fa_bwd_workspace_size(1, 2, 300, 64, 0)
    assert L.fa_bwd_blocksparse(*([A] * 10), need, 1, 2, 1, 300, 64, f, 1, -1, None, 0, 0, None) == 1
    assert L.fa_bwd_blocksparse(*([A] * 10), need - 1, 1, 2, 1, 300, 64, f, 1, -1, A, 0, 0, None) == 4


def test_varlen_rejects_bad_arguments(L):
    f = ctypes.c_float(0.125)
    assert L.fa_fwd_varlen(A, A, A, A, A, 2, 2, 1, 300, 64, f, 1, -1, None, 0, None) == 1
    assert L.fa_fwd_varlen(A, A, A, A, A, 2, 2, 1, 300, 96, f, 1, -1, A, 0, None) == 2
    assert L.fa_fwd_varlen(A, A + 4, A, A, A, 2, 2, 1, 300, 64, f, 1, -1, A, 0, None) == 3
    need = L.fa_bwd_workspace_size(2, 2, 300, 64, 1)
    assert L.fa_bwd_varlen(*([A] * 10), need, 2, 2, 1, 300, 64, f, 1, -1, None, 1, None) == 1
    assert L.fa_bwd_varlen(*([A] * 10), need - 1, 2, 2, 1, 300, 64, f, 1, -1, A, 1, None) == 4


def _strides(rows):
    arr = (fa._Strides * len(rows))()
    for n, (b, h, r) in enumerate(rows):
        arr[n] = fa._Strides(b, h, r)
    return arr


def test_strided_rejects_bad_arguments(L):
    f = ctypes.c_float(0.125)
    B, H, Hkv, N, d = 2, 4, 2, 300, 64
    q = (H * N * d, N * d, d)          # contiguous [B, H, N, d]
    kv = (Hkv * N * d, N * d, d)
    bshd = (N * H * d, d, H * d)       # [B, N, H, d] seen as [B, H, N, d]

    def fwd(rows, dtype=0, dd=d):
        return L.fa_fwd_strided(A, A, A, A, A, ctypes.addressof(rows) if rows is not None else None,
                                B, H, Hkv, N, dd, f, 1, -1, None, dtype, None)

    assert fwd(None) == 1
    assert fwd(_strides([q, kv, kv, (q[0], q[1], 0)])) == 1            # zero row stride
    assert fwd(_strides([(q[0], q[1], -d), kv, kv, q])) == 1           # negative stride
    assert fwd(_strides([q, kv, (kv[0], kv[1], d + 4), q])) == 3       # 8-byte pitch: not 16-byte aligned
    assert fwd(_strides([q, kv, kv, (q[0], q[1], d // 2)])) == 1       # output rows overlap
    assert fwd(_strides([q, kv, kv, (q[0], d, d)])) == 1               # output heads overlap rows
    assert fwd(_strides([q, kv, kv, (N * d, N * d, d)])) == 1          # output batch entries overlap heads
    assert fwd(_strides([q, kv, kv, (1 << 40, q[1], d)])) == 1         # beyond the tensor-map range
    assert fwd(_strides([q, kv, kv, bshd]), dd=96) == 2                # d still 64 or 128
    # fp32: strides must be multiples of 4 elements
    assert fwd(_strides([q, kv, (kv[0], kv[1], d + 2), q]), dtype=1) == 3
    need = L.fa_bwd_workspace_size(B, H, N, d, 0)
    good = [q, kv, kv, q, q, q, kv, kv]

    def bwd(rows, ws=need):
        return L.fa_bwd_strided(*([A] * 9), ctypes.addressof(rows) if rows is not None else None, A, ws,
                                B, H, Hkv, N, d, f, 1, -1, None, 0, None)

    assert bwd(None) == 1
    assert bwd(_strides(good), ws=need - 1) == 4
    bad = list(good)
    bad[6] = (kv[0], kv[1], d // 2)                                     # dk rows overlap
    assert bwd(_strides(bad)) == 1
    bad = list(good)
    bad[4] = (q[0], q[1], d + 4)                                        # dout pitch misaligned
    assert bwd(_strides(bad)) == 3


def test_strided_helper_requires_contiguous_last_axis():
    import torch
    x = torch.zeros(1, 2, 8, 64).transpose(2, 3)
    with pytest.raises(ValueError):
        fa._strides_of(x)
    st = fa._strides_of(torch.zeros(2, 8, 3, 64).transpose(1, 2))
    assert (st[0].batch, st[0].head, st[0].row) == (8 * 3 * 64, 64, 3 * 64)


def test_decode_rejects_bad_arguments(L):
    f = ctypes.c_float(0.125)
    need = L.fa_fwd_decode_workspace_size(2, 8, 2, 3, 128, 4)
    assert need == L.fa_fwd_splitkv_workspace_size(2, 2, 12, 128, 4)  # 4 heads x 3 rows per kv head
    assert L.fa_fwd_decode_workspace_size(2, 8, 2, 0, 128, 4) == 0
    assert L.fa_fwd_decode_workspace_size(2, 8, 2, 3, 128, 17) == 0

    def call(**kw):
        a = dict(q=A, B=2, H=8, Hkv=2, Nq=3, Nk=1000, d=128, splits=4, ws=need, dtype=0)
        a.update(kw)
        return L.fa_fwd_decode(a["q"], A, A, A, A, a["B"], a["H"], a["Hkv"], a["Nq"], a["Nk"], a["d"], f, 1, -1,
                               a["splits"], A, a["ws"], a["dtype"], None)

    assert call(q=None) == 1
    assert call(Nq=0) == 1
    assert call(Nq=1001) == 1                  # more queries than keys
    assert call(splits=0) == 1 and call(splits=17) == 1
    assert call(H=7) == 1                      # H % Hkv
    assert call(d=96) == 2
    assert call(dtype=1) == 2                  # bf16 only
    assert call(q=A + 8) == 3
    assert call(ws=need - 1) == 4


def test_decode_split_heuristic():
    # 64 units (B=8 x 8 kv heads, 4 x 1 packed rows each): 16 chunks fill 7 waves to 98.8%
    assert fa.decode_splits(8, 32, 8, 1, 32768) == 16
    assert fa.decode_splits(1, 1, 1, 1, 300) == 3          # at most one chunk per key tile
    assert fa.decode_splits(37, 4, 1, 1, 1 << 20) == 4      # 37 x 4 = 148: one full wave
    assert fa.decode_splits(148, 8, 8, 1, 32768) == 1


def test_packed_rejects_bad_arguments(L):
    f = ctypes.c_float(0.125)

    def cu(*vals):
        return (ctypes.c_int * len(vals))(*vals)

    def fwd(offsets, B, **kw):
        a = dict(q=A, H=4, Hkv=2, d=128, dtype=0)
        a.update(kw)
        return L.fa_fwd_packed(a["q"], A, A, A, A, offsets, a.get("dev", A), B, a["H"], a["Hkv"], a["d"], f, 1, -1,
                               a["dtype"], None)

    assert fwd(None, 2) == 1
    assert fwd(cu(1, 5, 9), 2) == 1          # first offset must be 0
    assert fwd(cu(0, 9, 5), 2) == 1          # offsets must not decrease
    assert fwd(cu(0, 5, 9), 0) == 1          # B >= 1
    assert fwd(cu(0, 5, 9), 2, H=3) == 1     # H % Hkv
    assert fwd(cu(0, 5, 9), 2, d=96) == 2
    assert fwd(cu(0, 5, 9), 2, q=A + 8) == 3
    assert fwd(cu(0, 5, 9), 2, dev=None) == 1      # bf16 reads the offsets on the device
    assert fwd(cu(0, 5, 9), 2, dev=A + 4) == 1     # ... from a 16-byte aligned copy
    assert fwd(cu(0, 0, 0), 2) == 0                # no tokens: nothing to launch
    # bf16: every sequence's rows in whole 128-row tiles at 128-aligned starts,
    # 128 * (ceil(T / 128) + B) rows per head; fp32: the longest sequence
    need = L.fa_bwd_packed_workspace_size(cu(0, 300, 301, 1000), 3, 4, 128, 0)
    assert need == L.fa_bwd_workspace_size(1, 4, 128 * (8 + 3), 128, 0)
    assert L.fa_bwd_packed_workspace_size(cu(0, 300, 301, 1000), 3, 4, 128, 1) == \
        L.fa_bwd_workspace_size(1, 4, 699, 128, 1)
    assert L.fa_bwd_packed_workspace_size(cu(0, 5, 4), 2, 4, 128, 0) == 0
    assert L.fa_bwd_packed(*([A] * 9), cu(0, 300, 301, 1000), A, A, need - 1, 3, 4, 2, 128, f, 1, -1, 0,
                           None) == 4


def test_seqlens_helper_rejects_copies():
    """A non-contiguous or host seqlens tensor is rejected rather than copied
    to a temporary whose memory the allocator could hand out again before the
    kernel reads it."""
    torch = pytest.importorskip("torch")
    with pytest.raises(TypeError):
        fa._seqlens_ptr(torch.zeros(4, dtype=torch.int32), 4)        # host memory
    with pytest.raises(TypeError):
        fa._seqlens_ptr(torch.zeros(4, dtype=torch.int64), 4)        # wrong dtype


def test_python_helpers_validate_before_the_c_layer():
    """Sizes come from q alone, so every other tensor is checked against it
    (shape, dtype, device, contiguity) before any pointer reaches the library."""
    torch = pytest.importorskip("torch")
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        fa.fwd(q, torch.zeros(1, 1, 7, 64, dtype=torch.bfloat16), k)     # fewer key rows than q
    with pytest.raises(ValueError, match="shape"):
        fa.fwd(q, k, torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16))    # head dim mismatch
    with pytest.raises(TypeError):
        fa.fwd(q, k.float(), k)                                          # dtype mismatch
    with pytest.raises(ValueError, match="CUDA"):
        fa.fwd(q, k, k)                                                  # host tensors never reach a kernel
    with pytest.raises(ValueError, match="shape"):
        fa.bwd(q, k, k, q, torch.zeros(1, 2, 8), torch.zeros(1, 2, 9, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="shape"):
        fa.fwd_decode(q, torch.zeros(1, 1, 20, 64, dtype=torch.bfloat16), k)   # v rows differ from k
    with pytest.raises(ValueError, match="tokens"):
        fa.fwd_packed(torch.zeros(10, 2, 64, dtype=torch.bfloat16), torch.zeros(10, 1, 64, dtype=torch.bfloat16),
                      torch.zeros(10, 1, 64, dtype=torch.bfloat16), [0, 4, 9])
    with pytest.raises(ValueError):
        fa._mask_args(torch.zeros(2, 2, dtype=torch.uint8), 1, 2, 300, torch.device("cpu"))  # 300 rows need 3 blocks
