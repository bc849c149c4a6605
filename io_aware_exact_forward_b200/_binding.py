"""ctypes binding of libfa (include/fa.h).

Argument marshalling only: every step of the attention computation runs in
the CUDA kernels of libfa.so.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

STATUS = {
    0: "FA_OK",
    1: "FA_ERR_INVALID_ARG",
    2: "FA_ERR_UNSUPPORTED",
    3: "FA_ERR_ALIGNMENT",
    4: "FA_ERR_WORKSPACE",
    5: "FA_ERR_CUDA",
    6: "FA_ERR_TIMEOUT",
}

# Every symbol include/fa.h declares, with its ctypes signature.
_c_int, _c_float, _c_size, _vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p
SIGNATURES = {
    "fa_status_string": (ctypes.c_char_p, [_c_int]),
    "fa_version": (_c_int, []),
    "fa_forward": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 6 + [_c_float, _c_int, _vp]),
    "fa_forward_window": (_c_int, [_vp, _vp, _vp, _vp, _vp] + [_c_int] * 6 + [_c_float, _c_int, _vp]),
    "fa_forward_dropout": (_c_int, [_vp] * 5 + [_c_int] * 6 + [_c_float, _c_int, _c_float, ctypes.c_ulonglong,
                                                               ctypes.c_uint, _vp]),
    "fa_forward_fp8": (_c_int, [_vp] * 3 + [_c_float] * 3 + [_vp, _vp] + [_c_int] * 6 + [_c_float, _c_int, _vp]),
    "fa_backward_workspace_bytes": (_c_size, [_c_int] * 6),
    "fa_backward": (_c_int, [_vp] * 9 + [_vp, _c_size] + [_c_int] * 6 + [_c_float, _c_int, _vp]),
    "fa_backward_window": (_c_int, [_vp] * 9 + [_vp, _c_size] + [_c_int] * 6 + [_c_float, _c_int, _vp]),
    "fa_backward_deterministic": (_c_int, [_vp] * 9 + [_vp, _c_size] + [_c_int] * 6 + [_c_float, _c_int, _c_int,
                                                                                      _vp]),
    "fa_backward_dropout": (_c_int, [_vp] * 9 + [_vp, _c_size] + [_c_int] * 6 + [_c_float, _c_int, _c_float,
                                                                             ctypes.c_ulonglong, ctypes.c_uint, _vp]),
    "fa_backward_dkdv_dropout": (_c_int, [_vp] * 7 + [_c_size] + [_c_int] * 6 + [_c_float, _c_int, _c_float,
                                                                                ctypes.c_ulonglong, ctypes.c_uint,
                                                                                _vp]),
    "fa_backward_preprocess": (_c_int, [_vp] * 4 + [_c_size] + [_c_int] * 6 + [_vp]),
    "fa_backward_dkdv": (_c_int, [_vp] * 7 + [_c_size] + [_c_int] * 6 + [_c_float, _c_int, _vp]),
    "fa_backward_dkdv_window": (_c_int, [_vp] * 7 + [_c_size] + [_c_int] * 6 + [_c_float, _c_int, _vp]),
    "fa_backward_dq_finalize": (_c_int, [_vp] * 2 + [_c_size] + [_c_int] * 6 + [_vp]),
    "fa_decode_workspace_bytes": (_c_size, [_c_int] * 5),
    "fa_decode_splitkv": (_c_int, [_vp] * 6 + [_vp, _c_size] + [_c_int] * 5 + [_c_float, _c_int, _vp]),
    "fa_decode_splitkv_window": (_c_int, [_vp] * 6 + [_vp, _c_size] + [_c_int] * 5 + [_c_float, _c_int, _c_int,
                                                                                    _vp]),
    "fa_decode_splitkv_noalloc": (_c_int, [_vp] * 6 + [_c_int] * 5 + [_c_float, _c_int, _vp]),
    "fa_decode_splitkv_partial": (_c_int, [_vp] * 6 + [_vp, _c_size] + [_c_int] * 5 + [_c_float, _c_int, _vp]),
    "fa_decode_merge": (_c_int, [_vp, _c_size, _vp, _c_size, _vp, _vp] + [_c_int] * 4 + [_vp]),
    "fa_check": (_c_int, [_vp]),
    "fa_selftest_bounded_wait": (_c_int, [_c_int, _vp]),
    "fa_selftest_exp2_poly": (_c_int, [_vp, _vp, _c_int, _vp]),
}


class FAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfa.so (built in-tree by io_aware_exact_forward_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(
                f"libfa.so not found at {path}; build it with "
                "`python -m io_aware_exact_forward_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _stream_ptr(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _check_dev(name, t, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (libfa has no CPU path)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _raise(fn, st):
    if st != 0:
        raise FAError(fn, st)


def forward(q, k, v, scale=None, causal=False, out=None, lse=None, window=None):
    """O, LSE = attention(q, k, v).  q [B,Tq,Hq,d], k/v [B,Tk,Hkv,d] bf16 (CUDA).
    ``window`` (int >= 1) selects the sliding-window mask of fa_forward_window
    (which includes the causal one)."""
    lib = load_library()
    B, Tq, Hq, d = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_dev(n, t, torch.bfloat16, dev)
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=dev)
    _check_dev("out", out, torch.bfloat16, dev)
    _check_dev("lse", lse, torch.float32, dev)
    if window is None:
        st = lib.fa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Tq, Tk, d,
                            float(scale), int(bool(causal)), _stream_ptr(dev))
        _raise("fa_forward", st)
    else:
        st = lib.fa_forward_window(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Tq, Tk, d,
                                   float(scale), int(window), _stream_ptr(dev))
        _raise("fa_forward_window", st)
    return out, lse


def forward_dropout(q, k, v, p_drop, seed, offset=0, scale=None, causal=False, out=None, lse=None):
    """O, LSE of attention with dropout on P (fa_forward_dropout): each
    probability kept with probability round(256 (1 - p_drop)) / 256 by a
    Philox-4x32-10 mask regenerated from (seed, offset), the kept ones scaled
    up by the inverse.  bf16 tensors as in forward()."""
    lib = load_library()
    B, Tq, Hq, d = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_dev(n, t, torch.bfloat16, dev)
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=dev)
    _check_dev("out", out, torch.bfloat16, dev)
    _check_dev("lse", lse, torch.float32, dev)
    st = lib.fa_forward_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Tq, Tk, d,
                                float(scale), int(bool(causal)), float(p_drop), int(seed) & (2 ** 64 - 1),
                                int(offset) & 0xFFFFFFFF, _stream_ptr(dev))
    _raise("fa_forward_dropout", st)
    return out, lse


def forward_fp8(q, k, v, q_descale, k_descale, v_descale, scale=None, causal=False, out=None, lse=None):
    """O, LSE of attention on E4M3 inputs (fa_forward_fp8).  q [B,Tq,Hq,128],
    k/v [B,Tk,Hkv,128] torch.float8_e4m3fn (CUDA); the descale factors map
    codes to values.  O is bf16, LSE fp32 [B,Hq,Tq]."""
    lib = load_library()
    B, Tq, Hq, d = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_dev(n, t, torch.float8_e4m3fn, dev)
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty((B, Tq, Hq, d), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=dev)
    _check_dev("out", out, torch.bfloat16, dev)
    _check_dev("lse", lse, torch.float32, dev)
    st = lib.fa_forward_fp8(_ptr(q), _ptr(k), _ptr(v), float(q_descale), float(k_descale), float(v_descale),
                            _ptr(out), _ptr(lse), B, Hq, Hkv, Tq, Tk, d, float(scale), int(bool(causal)),
                            _stream_ptr(dev))
    _raise("fa_forward_fp8", st)
    return out, lse


def backward_workspace_bytes(B, Hq, Hkv, Tq, Tk, d) -> int:
    return int(load_library().fa_backward_workspace_bytes(B, Hq, Hkv, Tq, Tk, d))


def backward(q, k, v, o, lse, do, scale=None, causal=False, workspace=None, dq=None, dk=None, dv=None,
             window=None, deterministic=False):
    """dQ, dK, dV for L = sum(dO * O).  `workspace` (uint8 CUDA tensor) is
    allocated here when not given; ``window`` as in forward().
    ``deterministic``: fa_backward_deterministic (dQ the same bit for bit from
    run to run, at the cost of a second pass)."""
    lib = load_library()
    B, Tq, Hq, d = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _check_dev(n, t, torch.bfloat16, dev)
    _check_dev("lse", lse, torch.float32, dev)
    if scale is None:
        scale = d ** -0.5
    need = backward_workspace_bytes(B, Hq, Hkv, Tq, Tk, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
            _ptr(workspace), workspace.numel(), B, Hq, Hkv, Tq, Tk, d, float(scale))
    if deterministic:
        win = 0 if window is None else int(window)
        st = lib.fa_backward_deterministic(*args, int(bool(causal) or win > 0), win, _stream_ptr(dev))
        _raise("fa_backward_deterministic", st)
    elif window is None:
        st = lib.fa_backward(*args, int(bool(causal)), _stream_ptr(dev))
        _raise("fa_backward", st)
    else:
        st = lib.fa_backward_window(*args, int(window), _stream_ptr(dev))
        _raise("fa_backward_window", st)
    return dq, dk, dv


def backward_dropout(q, k, v, o, lse, do, p_drop, seed, offset=0, scale=None, causal=False, workspace=None,
                     dq=None, dk=None, dv=None):
    """dQ, dK, dV for forward_dropout with the same (p_drop, seed, offset):
    the kernel regenerates the forward's keep mask.  o and lse are the
    dropout forward's outputs."""
    lib = load_library()
    B, Tq, Hq, d = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _check_dev(n, t, torch.bfloat16, dev)
    _check_dev("lse", lse, torch.float32, dev)
    if scale is None:
        scale = d ** -0.5
    need = backward_workspace_bytes(B, Hq, Hkv, Tq, Tk, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    st = lib.fa_backward_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                                 _ptr(dv), _ptr(workspace), workspace.numel(), B, Hq, Hkv, Tq, Tk, d, float(scale),
                                 int(bool(causal)), float(p_drop), int(seed) & (2 ** 64 - 1),
                                 int(offset) & 0xFFFFFFFF, _stream_ptr(dev))
    _raise("fa_backward_dropout", st)
    return dq, dk, dv


def decode_workspace_bytes(B, Hq, Tk_max, d, chunk=256) -> int:
    return int(load_library().fa_decode_workspace_bytes(B, Hq, Tk_max, d, chunk))


def decode_splitkv(q, k_cache, v_cache, seqlens, scale=None, chunk=256, workspace=None, out=None, lse=None,
                   window=None):
    """Split-KV decode.  q [B,Hq,d], caches [B,Tk_max,Hkv,d] bf16, seqlens int32 [B] (CUDA).
    ``window`` (int >= 1) keeps only the last `window` keys of each sequence."""
    lib = load_library()
    B, Hq, d = q.shape
    Tk_max, Hkv = k_cache.shape[1], k_cache.shape[2]
    dev = q.device
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_dev(n, t, torch.bfloat16, dev)
    _check_dev("seqlens", seqlens, torch.int32, dev)
    if scale is None:
        scale = d ** -0.5
    need = decode_workspace_bytes(B, Hq, Tk_max, d, chunk)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev) if lse is None else lse
    args = (_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(out), _ptr(lse), _ptr(workspace),
            workspace.numel(), B, Hq, Hkv, Tk_max, d, float(scale), int(chunk))
    if window is None:
        st = lib.fa_decode_splitkv(*args, _stream_ptr(dev))
        _raise("fa_decode_splitkv", st)
    else:
        st = lib.fa_decode_splitkv_window(*args, int(window), _stream_ptr(dev))
        _raise("fa_decode_splitkv_window", st)
    return out, lse


def decode_splitkv_noalloc(q, k_cache, v_cache, seqlens, scale=None, chunk=256, out=None, lse=None):
    """Split-KV decode through fa_decode_splitkv_noalloc: the chunk partials
    live in the library's built-in 32 MiB device array instead of a caller
    workspace.  Calls that overlap on the GPU share that array and race."""
    lib = load_library()
    B, Hq, d = q.shape
    Tk_max, Hkv = k_cache.shape[1], k_cache.shape[2]
    dev = q.device
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_dev(n, t, torch.bfloat16, dev)
    _check_dev("seqlens", seqlens, torch.int32, dev)
    if scale is None:
        scale = d ** -0.5
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev) if lse is None else lse
    st = lib.fa_decode_splitkv_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(out), _ptr(lse),
                                       B, Hq, Hkv, Tk_max, d, float(scale), int(chunk), _stream_ptr(dev))
    _raise("fa_decode_splitkv_noalloc", st)
    return out, lse


def decode_splitkv_partial(q, k_cache, v_cache, seqlens, scale=None, chunk=256, workspace=None, out=None,
                           lse=None):
    """Split-KV decode of this device's share of the keys with O kept in
    fp32 (fa_decode_splitkv_partial), for a later decode_merge.  Shapes as in
    decode_splitkv; ``out`` is float32 [B,Hq,d] and may be a view into a
    larger packed buffer."""
    lib = load_library()
    B, Hq, d = q.shape
    Tk_max, Hkv = k_cache.shape[1], k_cache.shape[2]
    dev = q.device
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_dev(n, t, torch.bfloat16, dev)
    _check_dev("seqlens", seqlens, torch.int32, dev)
    if scale is None:
        scale = d ** -0.5
    need = decode_workspace_bytes(B, Hq, Tk_max, d, chunk)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev) if lse is None else lse
    _check_dev("out", out, torch.float32, dev)
    _check_dev("lse", lse, torch.float32, dev)
    st = lib.fa_decode_splitkv_partial(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(out), _ptr(lse),
                                       _ptr(workspace), workspace.numel(), B, Hq, Hkv, Tk_max, d, float(scale),
                                       int(chunk), _stream_ptr(dev))
    _raise("fa_decode_splitkv_partial", st)
    return out, lse


def decode_merge(o_parts, lse_parts, out=None, lse=None):
    """Merge R partial decodes by their log-sum-exp (fa_decode_merge).
    o_parts float32 [R,B,Hq,d] and lse_parts float32 [R,B,Hq]; each may have
    any stride along R (e.g. views into one packed all-gather buffer) but must
    be contiguous within a partial.  Returns O bf16 [B,Hq,d], LSE [B,Hq]."""
    lib = load_library()
    if o_parts.dim() != 4 or o_parts.shape[0] < 1:
        raise ValueError(f"o_parts must be [R >= 1, B, Hq, d], got {tuple(o_parts.shape)}")
    R, B, Hq, d = o_parts.shape
    dev = o_parts.device
    for n, t in (("o_parts", o_parts), ("lse_parts", lse_parts)):
        if t.device.type != "cuda" or t.device != dev:
            raise ValueError(f"{n} must be on {dev}")
        if t.dtype != torch.float32:
            raise TypeError(f"{n} must be float32")
        if not t[0].is_contiguous():
            raise ValueError(f"{n} must be contiguous within a partial")
    if tuple(lse_parts.shape) != (R, B, Hq):
        raise ValueError(f"lse_parts has shape {tuple(lse_parts.shape)}, expected {(R, B, Hq)}")
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev) if lse is None else lse
    _check_dev("out", out, torch.bfloat16, dev)
    _check_dev("lse", lse, torch.float32, dev)
    st = lib.fa_decode_merge(_ptr(o_parts), o_parts.stride(0), _ptr(lse_parts), lse_parts.stride(0), _ptr(out),
                             _ptr(lse), R, B, Hq, d, _stream_ptr(dev))
    _raise("fa_decode_merge", st)
    return out, lse


def check(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    return int(load_library().fa_check(_stream_ptr(dev)))


def selftest_bounded_wait(limit_us: int, device=None) -> int:
    dev = torch.device("cuda") if device is None else torch.device(device)
    return int(load_library().fa_selftest_bounded_wait(int(limit_us), _stream_ptr(dev)))
