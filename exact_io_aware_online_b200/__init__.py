"""Exact IO-aware online-softmax attention for B200 (sm_100a).

The compute lives in ``libfa.so`` (CUDA kernels behind the C ABI of
``include/fa.h``).  This package only marshals arguments: ``lib()`` loads the
shared library with ctypes and the ``fwd`` / ``bwd`` helpers allocate outputs
with PyTorch and pass raw device pointers and the current stream.  There is no
CPU fallback: if the library is missing or a call fails, an error is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

__all__ = ["lib", "FAError", "FA_BF16", "FA_FP32", "fwd", "bwd", "bwd_workspace_size", "device_status",
           "exported_names", "set_timing_events", "bwd_noalloc", "fwd_splitkv", "fwd_blocksparse", "bwd_blocksparse", "fwd_varlen", "bwd_varlen", "fwd_strided", "bwd_strided",
           "fwd_decode", "decode_splits", "fwd_packed", "bwd_packed", "debug_set_wait_limit", "debug_set_stall",
           "LIB_PATH", "HEADER_PATH"]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa.so")
HEADER_PATH = os.path.join(os.path.dirname(HERE), "include", "fa.h")

FA_BF16, FA_FP32 = 0, 1
STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_MISALIGNED",
          4: "FA_ERR_WORKSPACE", 5: "FA_ERR_CUDA", 6: "FA_ERR_TIMEOUT"}

_lib = None


class FAError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}" if what else STATUS.get(code, str(code)))


def exported_names() -> list[str]:
    """Function names declared in include/fa.h."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_]+\**\s+\**(fa_[a-z_0-9]+)\s*\(", text, re.M)))


def lib() -> ctypes.CDLL:
    """Load libfa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_io_aware_online_b200._build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp]
    L.fa_fwd.restype = i
    L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, i, i, vp]
    L.fa_bwd.restype = i
    L.fa_bwd_workspace_size.argtypes = [i, i, i, i, i]
    L.fa_bwd_workspace_size.restype = sz
    L.fa_last_device_status.argtypes = [vp]
    L.fa_last_device_status.restype = i
    L.fa_status_string.argtypes = [i]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_version.argtypes = []
    L.fa_version.restype = i
    L.fa_set_timing_events.argtypes = [vp, vp]
    L.fa_set_timing_events.restype = None
    L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp]
    L.fa_bwd_noalloc.restype = i
    L.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp, sz, i, vp]
    L.fa_fwd_splitkv.restype = i
    L.fa_fwd_splitkv_workspace_size.argtypes = [i, i, i, i, i]
    L.fa_fwd_splitkv_workspace_size.restype = sz
    ll = ctypes.c_longlong
    L.fa_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, ll, i, vp]
    L.fa_fwd_blocksparse.restype = i
    L.fa_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, i, vp, ll, i, vp]
    L.fa_bwd_blocksparse.restype = i
    L.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, i, vp]
    L.fa_fwd_varlen.restype = i
    L.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, i, vp, i, vp]
    L.fa_bwd_varlen.restype = i
    L.fa_fwd_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, sz, i, vp]
    L.fa_fwd_decode.restype = i
    L.fa_fwd_decode_workspace_size.argtypes = [i, i, i, i, i, i]
    L.fa_fwd_decode_workspace_size.restype = sz
    L.fa_fwd_packed.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
    L.fa_fwd_packed.restype = i
    L.fa_bwd_packed_workspace_size.argtypes = [vp, i, i, i, i]
    L.fa_bwd_packed_workspace_size.restype = sz
    L.fa_bwd_packed.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, i, i, vp]
    L.fa_bwd_packed.restype = i
    L.fa_fwd_strided.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, i, vp]
    L.fa_fwd_strided.restype = i
    L.fa_bwd_strided.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, i, vp, i, vp]
    L.fa_bwd_strided.restype = i
    L.fa_debug_set_wait_limit.argtypes = [ctypes.c_ulonglong]
    L.fa_debug_set_wait_limit.restype = i
    L.fa_debug_set_stall.argtypes = [i]
    L.fa_debug_set_stall.restype = i
    _lib = L
    return L


# ---------------------------------------------------------------------------
# torch-facing helpers (argument marshalling only)
# ---------------------------------------------------------------------------
def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float32:
        return FA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_ptr(device) -> int:
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def _check(code: int, what: str):
    if code != 0:
        raise FAError(code, what)


def _on(device, fn, *args):
    """Calls a library entry point with `device` current: the C ABI enqueues on
    the stream it is given and rejects a stream of another device than the
    current one."""
    import torch
    with torch.cuda.device(device):
        return fn(*args)


def _validate(like, *specs):
    """Each (tensor, shape, name, contiguous) must have that shape, the dtype of
    `like`, live on like's CUDA device and (unless the helper takes strided
    layouts) be contiguous.  Shapes and dtypes are checked for all tensors
    before placement.  The C entry points receive only pointers and sizes, so a
    mismatch here would let a kernel read or write outside a buffer."""
    for t, shape, name, _ in specs:
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
        if t.dtype != like.dtype:
            raise TypeError(f"{name}: dtype {t.dtype}, expected {like.dtype}")
    for t, _, name, contiguous in specs:
        if not t.is_cuda or t.device != like.device:
            raise ValueError(f"{name}: must be on the CUDA device of q, got {t.device} (q: {like.device})")
        if contiguous and not t.is_contiguous():
            raise ValueError(f"{name}: must be contiguous (the *_strided helpers take other layouts)")


def _same(t, shape, like, name: str, contiguous: bool = True):
    _validate(like, (t, shape, name, contiguous))


def _check_qkv(q, k, v, contiguous: bool = True, kv_rows=None, extra=()):
    """q [B,H,N,d]; k, v [B,Hkv,kv_rows or N,d] of q's dtype and device, plus
    the (tensor, shape, name) triples in `extra`."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D [batch, heads, rows, head_dim]")
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    rows = N if kv_rows is None else kv_rows
    specs = [(q, (B, H, N, d), "q"), (k, (B, Hkv, rows, d), "k"), (v, (B, Hkv, rows, d), "v"), *extra]
    _validate(q, *[(t, sh, nm, contiguous) for t, sh, nm in specs])
    return B, H, Hkv, N, d


def _check_lse(lse, shape, q):
    import torch
    if lse.dtype != torch.float32 or tuple(lse.shape) != tuple(shape) or not lse.is_cuda or lse.device != q.device \
            or not lse.is_contiguous():
        raise ValueError(f"lse: must be a contiguous float32 tensor of shape {tuple(shape)} on {q.device}")


def _bwd_specs(q, k, o, do, grads):
    """(tensor, shape, name) triples of the backward's other tensors."""
    specs = [(o, q.shape, "o"), (do, q.shape, "do")]
    if grads is not None:
        dq, dk, dv = grads
        specs += [(dq, q.shape, "dq"), (dk, k.shape, "dk"), (dv, k.shape, "dv")]
    return specs


def _check_workspace(ws, device):
    import torch
    if ws.dtype != torch.uint8 or not ws.is_cuda or ws.device != device or not ws.is_contiguous():
        raise ValueError("workspace: must be a contiguous torch.uint8 tensor on the inputs' device")


def bwd_workspace_size(B: int, H: int, N: int, d: int, dtype_code: int) -> int:
    return int(lib().fa_bwd_workspace_size(B, H, N, d, dtype_code))


def fwd(q, k, v, scale: float | None = None, causal: bool = False, window: int = -1, out=None, lse=None):
    """O, LSE = attention(q [B,H,N,d], k/v [B,Hkv,N,d]); outputs allocated if not given."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v)
    if out is not None:
        _same(out, q.shape, q, "out")
    if lse is not None:
        _check_lse(lse, (B, H, N), q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    code = _on(q.device, lib().fa_fwd, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                        B, H, Hkv, N, d, float(scale), int(bool(causal)), int(window), _dtype_code(q),
                        _stream_ptr(q.device))
    _check(code, "fa_fwd")
    return o, l


def fwd_splitkv(q, k, v, num_splits: int, scale: float | None = None, causal: bool = False, window: int = -1,
                out=None, lse=None, workspace=None):
    """fwd() with each query block's key range split into `num_splits` chunks
    (partials merged on the device); bf16 only."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v)
    if out is not None:
        _same(out, q.shape, q, "out")
    if lse is not None:
        _check_lse(lse, (B, H, N), q)
    if workspace is not None:
        _check_workspace(workspace, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    need = int(lib().fa_fwd_splitkv_workspace_size(B, H, N, d, int(num_splits)))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device) if workspace is None else workspace
    code = _on(q.device, lib().fa_fwd_splitkv, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                                B, H, Hkv, N, d, float(scale), int(bool(causal)), int(window), int(num_splits),
                                ws.data_ptr(), ws.numel(), _dtype_code(q), _stream_ptr(q.device))
    _check(code, "fa_fwd_splitkv")
    return o, l


def decode_splits(B: int, H: int, Hkv: int, Nq: int, Nk: int, sms: int = 148) -> int:
    """Key chunks per query tile for fwd_decode().  The kernel runs one CTA per
    (kv head, 256 packed query rows, chunk), all of about the same length, so
    the count is chosen for whole waves over the SMs: the largest share of
    busy SM slots in the last wave, at most 16 chunks and at most one per
    128-key tile."""
    units = B * Hkv * (((H // Hkv) * Nq + 255) // 256)
    best, best_eff = 1, -1.0
    for s in range(1, min(16, (Nk + 127) // 128) + 1):
        ctas = units * s
        eff = ctas / (sms * -(-ctas // sms))
        if eff > best_eff + 1e-9:
            best, best_eff = s, eff
    return best


def fwd_decode(q, k, v, num_splits: int | None = None, scale: float | None = None, causal: bool = False,
               window: int = -1, out=None, lse=None, workspace=None):
    """O, LSE for q [B,H,Nq,d] against k/v [B,Hkv,Nk,d], Nq <= Nk: the queries
    are the newest Nq positions (see fa_fwd_decode in fa.h); bf16 only."""
    import torch
    if k.dim() != 4:
        raise ValueError("k must be 4-D [batch, kv heads, keys, head_dim]")
    B, H, Hkv, Nq, d = _check_qkv(q, k, v, kv_rows=k.shape[2])
    Nk = k.shape[2]
    if out is not None:
        _same(out, q.shape, q, "out")
    if lse is not None:
        _check_lse(lse, (B, H, Nq), q)
    if workspace is not None:
        _check_workspace(workspace, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    S = decode_splits(B, H, Hkv, Nq, Nk) if num_splits is None else int(num_splits)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    need = int(lib().fa_fwd_decode_workspace_size(B, H, Hkv, Nq, d, S))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device) if workspace is None else workspace
    code = _on(q.device, lib().fa_fwd_decode, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                               B, H, Hkv, Nq, Nk, d, float(scale), int(bool(causal)), int(window), S,
                               ws.data_ptr(), ws.numel(), _dtype_code(q), _stream_ptr(q.device))
    _check(code, "fa_fwd_decode")
    return o, l


def bwd(q, k, v, o, lse, do, scale: float | None = None, causal: bool = False, window: int = -1,
        workspace=None, grads=None):
    """dQ, dK, dV of sum(do * o); workspace and gradients allocated if not given."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v, extra=_bwd_specs(q, k, o, do, grads))
    _check_lse(lse, (B, H, N), q)
    if workspace is not None:
        _check_workspace(workspace, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    code_t = _dtype_code(q)
    need = bwd_workspace_size(B, H, N, d, code_t)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    code = _on(q.device, lib().fa_bwd, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws.numel(),
                        B, H, Hkv, N, d, float(scale), int(bool(causal)), int(window), code_t,
                        _stream_ptr(q.device))
    _check(code, "fa_bwd")
    return dq, dk, dv


def bwd_noalloc(q, k, v, o, lse, do, scale: float | None = None, causal: bool = False, window: int = -1,
                grads=None):
    """bwd() for callers that cannot allocate device memory: the library's
    built-in scratch array replaces the workspace (see fa_bwd_noalloc in fa.h).
    Pass preallocated `grads`=(dq, dk, dv) to keep the call allocation-free."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v, extra=_bwd_specs(q, k, o, do, grads))
    _check_lse(lse, (B, H, N), q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    code = _on(q.device, lib().fa_bwd_noalloc, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                B, H, Hkv, N, d, float(scale), int(bool(causal)), int(window), _dtype_code(q),
                                _stream_ptr(q.device))
    _check(code, "fa_bwd_noalloc")
    return dq, dk, dv


def _mask_args(block_mask, B, H, N, device):
    """(device pointer, head stride) for a uint8 block mask of shape [nb, nb]
    (shared) or [B, H, nb, nb] (per query head), nb = ceil(N / 128)."""
    import torch
    if block_mask.dtype != torch.uint8 or not block_mask.is_contiguous():
        raise TypeError("block_mask must be a contiguous torch.uint8 tensor")
    nb = (N + 127) // 128
    if tuple(block_mask.shape) not in ((nb, nb), (B, H, nb, nb)):
        raise ValueError(f"block_mask must be [{nb}, {nb}] or [{B}, {H}, {nb}, {nb}] for N = {N}")
    if not block_mask.is_cuda or block_mask.device != device:
        raise ValueError("block_mask must be on the CUDA device of q")
    return block_mask.data_ptr(), (0 if block_mask.dim() == 2 else nb * nb)


def fwd_blocksparse(q, k, v, block_mask, scale: float | None = None, causal: bool = False, window: int = -1,
                    out=None, lse=None):
    """fwd() restricted to the 128 x 128 blocks that `block_mask` switches on."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v)
    if out is not None:
        _same(out, q.shape, q, "out")
    if lse is not None:
        _check_lse(lse, (B, H, N), q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    mp, hs = _mask_args(block_mask, B, H, N, q.device)
    code = _on(q.device, lib().fa_fwd_blocksparse, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                                    B, H, Hkv, N, d, float(scale), int(bool(causal)), int(window), mp, hs,
                                    _dtype_code(q), _stream_ptr(q.device))
    _check(code, "fa_fwd_blocksparse")
    return o, l


def bwd_blocksparse(q, k, v, o, lse, do, block_mask, scale: float | None = None, causal: bool = False,
                    window: int = -1, workspace=None, grads=None):
    """bwd() of fwd_blocksparse()."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v, extra=_bwd_specs(q, k, o, do, grads))
    _check_lse(lse, (B, H, N), q)
    if workspace is not None:
        _check_workspace(workspace, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    code_t = _dtype_code(q)
    need = bwd_workspace_size(B, H, N, d, code_t)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    mp, hs = _mask_args(block_mask, B, H, N, q.device)
    code = _on(q.device, lib().fa_bwd_blocksparse, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                    lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(),
                                    ws.numel(), B, H, Hkv, N, d, float(scale), int(bool(causal)), int(window), mp, hs,
                                    code_t, _stream_ptr(q.device))
    _check(code, "fa_bwd_blocksparse")
    return dq, dk, dv


def _seqlens_ptr(seqlens, B):
    import torch
    if seqlens.dtype != torch.int32 or seqlens.numel() != B or not seqlens.is_cuda or not seqlens.is_contiguous():
        raise TypeError("seqlens must be a contiguous CUDA int32 tensor of B values")
    return seqlens.data_ptr()  # the caller's tensor: no temporary copy whose memory could be reused


def fwd_varlen(q, k, v, seqlens, scale: float | None = None, causal: bool = False, window: int = -1,
               out=None, lse=None):
    """fwd() where batch entry b holds seqlens[b] valid tokens (padded layout)."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v)
    if out is not None:
        _same(out, q.shape, q, "out")
    if lse is not None:
        _check_lse(lse, (B, H, N), q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    code = _on(q.device, lib().fa_fwd_varlen, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                               B, H, Hkv, N, d, float(scale), int(bool(causal)), int(window),
                               _seqlens_ptr(seqlens, B), _dtype_code(q), _stream_ptr(q.device))
    _check(code, "fa_fwd_varlen")
    return o, l


def bwd_varlen(q, k, v, o, lse, do, seqlens, scale: float | None = None, causal: bool = False, window: int = -1,
               workspace=None, grads=None):
    """bwd() of fwd_varlen()."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v, extra=_bwd_specs(q, k, o, do, grads))
    _check_lse(lse, (B, H, N), q)
    if workspace is not None:
        _check_workspace(workspace, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    code_t = _dtype_code(q)
    need = bwd_workspace_size(B, H, N, d, code_t)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    code = _on(q.device, lib().fa_bwd_varlen, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                               dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws.numel(),
                               B, H, Hkv, N, d, float(scale), int(bool(causal)), int(window),
                               _seqlens_ptr(seqlens, B), code_t, _stream_ptr(q.device))
    _check(code, "fa_bwd_varlen")
    return dq, dk, dv


class _Strides(ctypes.Structure):
    """fa_strides of include/fa.h: element strides of the batch, head and row axes."""
    _fields_ = [("batch", ctypes.c_longlong), ("head", ctypes.c_longlong), ("row", ctypes.c_longlong)]


def _strides_of(*tensors):
    arr = (_Strides * len(tensors))()
    for n, t in enumerate(tensors):
        if t.dim() != 4 or t.stride(3) != 1:
            raise ValueError("tensors must be 4-D [B, heads, N, d] views with a contiguous last axis")
        arr[n] = _Strides(t.stride(0), t.stride(1), t.stride(2))
    return arr


def fwd_strided(q, k, v, scale: float | None = None, causal: bool = False, window: int = -1, seqlens=None,
                out=None, lse=None):
    """fwd() on [B,H,N,d] / [B,Hkv,N,d] views of any layout with d contiguous
    (e.g. x.transpose(1, 2) of a [B,N,H,d] buffer).  O takes q's layout unless
    `out` is given; `seqlens` (optional) as in fwd_varlen()."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v, contiguous=False)
    if out is not None:
        _same(out, q.shape, q, "out", contiguous=False)
    if lse is not None:
        _check_lse(lse, (B, H, N), q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    st = _strides_of(q, k, v, o)
    sp = _seqlens_ptr(seqlens, B) if seqlens is not None else None
    code = _on(q.device, lib().fa_fwd_strided, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                                ctypes.addressof(st), B, H, Hkv, N, d, float(scale), int(bool(causal)),
                                int(window), sp, _dtype_code(q), _stream_ptr(q.device))
    _check(code, "fa_fwd_strided")
    return o, l


def bwd_strided(q, k, v, o, lse, do, scale: float | None = None, causal: bool = False, window: int = -1,
                seqlens=None, workspace=None, grads=None):
    """bwd() of fwd_strided(); dq, dk, dv take the layouts of q, k, v unless
    `grads` is given."""
    import torch
    B, H, Hkv, N, d = _check_qkv(q, k, v, contiguous=False, extra=_bwd_specs(q, k, o, do, grads))
    _check_lse(lse, (B, H, N), q)
    if workspace is not None:
        _check_workspace(workspace, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    code_t = _dtype_code(q)
    need = bwd_workspace_size(B, H, N, d, code_t)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    st = _strides_of(q, k, v, o, do, dq, dk, dv)
    sp = _seqlens_ptr(seqlens, B) if seqlens is not None else None
    code = _on(q.device, lib().fa_bwd_strided, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ctypes.addressof(st),
                                ws.data_ptr(), ws.numel(), B, H, Hkv, N, d, float(scale), int(bool(causal)),
                                int(window), sp, code_t, _stream_ptr(q.device))
    _check(code, "fa_bwd_strided")
    return dq, dk, dv


def _host_offsets(cu_seqlens):
    """ctypes int32 array of the B + 1 offsets (kept alive by the caller)."""
    vals = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    return (ctypes.c_int * len(vals))(*vals), len(vals) - 1


def _device_offsets(cu_seqlens, host, B, device, cu_seqlens_dev=None):
    """Device int32 copy of the offsets that the kernels read: cu_seqlens_dev
    when given, else the caller's tensor itself when it already is one
    (contiguous int32 on `device`), otherwise a new tensor made from the host
    values on the current stream (the calls run on that stream, after the copy)."""
    import torch
    t = cu_seqlens_dev if cu_seqlens_dev is not None else cu_seqlens
    if isinstance(t, torch.Tensor) and t.is_cuda:
        if t.device != device or t.dtype != torch.int32 or not t.is_contiguous() or t.numel() != B + 1:
            raise TypeError("device offsets must be a contiguous int32 tensor of B + 1 values on q's device")
        return t
    if cu_seqlens_dev is not None:
        raise TypeError("cu_seqlens_dev must be a CUDA int32 tensor")
    return torch.tensor([host[i] for i in range(B + 1)], dtype=torch.int32, device=device)


def fwd_packed(q, k, v, cu_seqlens, scale: float | None = None, causal: bool = False, window: int = -1,
               out=None, lse=None, cu_seqlens_dev=None):
    """O [T,H,d] and LSE (flat: sequence b's [H, len_b] block at H * cu[b]) for
    sequences packed along the token axis: q [T,H,d], k/v [T,Hkv,d], cu_seqlens
    the B + 1 offsets (list, CPU tensor, or int32 tensor on q's device, which
    is then read back to the host).  bf16 runs every sequence in one launch
    per kernel, reading a device copy of the offsets: cu_seqlens_dev (an int32
    tensor on q's device holding the same values) when given, else one made
    here."""
    import torch
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q, k, v must be 3-D [tokens, heads, head_dim]")
    T, H, d = q.shape
    Hkv = k.shape[1]
    cu, B = _host_offsets(cu_seqlens)
    if cu[B] != T:
        raise ValueError(f"cu_seqlens[-1] = {cu[B]} but q holds {T} tokens")
    _validate(q, (q, (T, H, d), "q", True), (k, (T, Hkv, d), "k", True), (v, (T, Hkv, d), "v", True))
    if out is not None:
        _same(out, q.shape, q, "out")
    if lse is not None:
        _check_lse(lse, (T * H,), q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty(T * H, dtype=torch.float32, device=q.device) if lse is None else lse
    cu_dev = _device_offsets(cu_seqlens, cu, B, q.device, cu_seqlens_dev)
    code = _on(q.device, lib().fa_fwd_packed, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(), cu,
               cu_dev.data_ptr(), B, H, Hkv, d, float(scale), int(bool(causal)), int(window), _dtype_code(q),
               _stream_ptr(q.device))
    _check(code, "fa_fwd_packed")
    return o, l


def bwd_packed(q, k, v, o, lse, do, cu_seqlens, scale: float | None = None, causal: bool = False, window: int = -1,
               workspace=None, grads=None, cu_seqlens_dev=None):
    """bwd() of fwd_packed()."""
    import torch
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q, k, v must be 3-D [tokens, heads, head_dim]")
    T, H, d = q.shape
    Hkv = k.shape[1]
    cu, B = _host_offsets(cu_seqlens)
    if cu[B] != T:
        raise ValueError(f"cu_seqlens[-1] = {cu[B]} but q holds {T} tokens")
    _validate(q, *[(t, sh, nm, True) for t, sh, nm in
                   [(q, (T, H, d), "q"), (k, (T, Hkv, d), "k"), (v, (T, Hkv, d), "v"),
                    *_bwd_specs(q, k, o, do, grads)]])
    _check_lse(lse, (T * H,), q)
    if workspace is not None:
        _check_workspace(workspace, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    code_t = _dtype_code(q)
    need = int(lib().fa_bwd_packed_workspace_size(cu, B, H, d, code_t))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    cu_dev = _device_offsets(cu_seqlens, cu, B, q.device, cu_seqlens_dev)
    code = _on(q.device, lib().fa_bwd_packed, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
               lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), cu, cu_dev.data_ptr(), ws.data_ptr(),
               ws.numel(), B, H, Hkv, d, float(scale), int(bool(causal)), int(window), code_t,
               _stream_ptr(q.device))
    _check(code, "fa_bwd_packed")
    return dq, dk, dv


def set_timing_events(start=None, stop=None):
    """Record torch.cuda.Event pair around the next calls' main kernel (None: off)."""
    lib().fa_set_timing_events(start.cuda_event if start is not None else None,
                               stop.cuda_event if stop is not None else None)


def device_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    import torch
    return int(lib().fa_last_device_status(torch.cuda.current_stream(device).cuda_stream))


def debug_set_wait_limit(ns: int = 0):
    """Test hook: limit (ns) of the kernels' waits on other roles; 0 restores the default."""
    _check(lib().fa_debug_set_wait_limit(int(ns)), "fa_debug_set_wait_limit")


def debug_set_stall(on: bool):
    """Test hook: while on, the sm_100a kernels never issue their first tile load."""
    _check(lib().fa_debug_set_stall(1 if on else 0), "fa_debug_set_stall")
