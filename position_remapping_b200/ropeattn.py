"""Thin Python binding of the ropeattn C ABI (include/ropeattn.h).

Argument marshalling only: every step of the computation runs in the CUDA
library. PyTorch provides device memory and the current stream. Importing this
module loads libropeattn.so and raises if it is missing; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

from .inputs import MapParams

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libropeattn.so")

OK = 0
ERR_INVALID_ARG, ERR_UNSUPPORTED_DEVICE, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = -1, -2, -3, -4, -5

# every symbol include/ropeattn.h declares
EXPORTS = ("ropeattn_posmap", "ropeattn_cache_write", "ropeattn_prefill_workspace_size", "ropeattn_prefill",
           "ropeattn_prefill_prepare", "ropeattn_prefill_attend",
           "ropeattn_prefill_chunk_workspace_size", "ropeattn_prefill_chunk", "ropeattn_prefill_chunk_cache",
           "ropeattn_prefill_three_call_workspace_size", "ropeattn_prefill_three_call",
           "ropeattn_decode_workspace_size", "ropeattn_decode", "ropeattn_decode_cache", "ropeattn_decode_noalloc",
           "ropeattn_status",
           "ropeattn_wait_selftest", "ropeattn_decode_unfused_workspace_size", "ropeattn_decode_unfused",
           "ropeattn_prefill_backward_workspace_size", "ropeattn_prefill_backward",
           "ropeattn_last_error", "ropeattn_version")


class RopeAttnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"ropeattn error {code}: {msg}")
        self.code = code


class CParams(ctypes.Structure):
    """Mirror of ``ropeattn_params``."""
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("fixed_group", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
        ("interp", ctypes.c_double),
        ("seg1_len", ctypes.c_int64),
        ("term_start", ctypes.c_int64),
        ("window", ctypes.c_int64),
        ("w0", ctypes.c_int64),
        ("w_pretrained", ctypes.c_int64),
        ("softmax_scale", ctypes.c_float),
        ("pairing", ctypes.c_int32),
        ("reserved", ctypes.c_int32 * 2),
    ]


_CPARAMS_CACHE: dict = {}
_CPARAMS_LAST: list = [None, None]   # the last (MapParams object, struct): a decode loop passes the same object


def _cparams(p: MapParams) -> CParams:
    """The C parameter struct of `p` for the binding's own calls, which never
    modify it (cached: MapParams is frozen, and a decode step runs every
    token)."""
    if _CPARAMS_LAST[0] is p:
        return _CPARAMS_LAST[1]
    c = _CPARAMS_CACHE.get(p)
    if c is None:
        c = to_cparams(p)
        if len(_CPARAMS_CACHE) < 256:
            _CPARAMS_CACHE[p] = c
    _CPARAMS_LAST[0], _CPARAMS_LAST[1] = p, c
    return c


def to_cparams(p: MapParams) -> CParams:
    """A fresh C parameter struct of `p`."""
    c = CParams()
    c.kind = int(p.kind)
    c.fixed_group = int(p.fixed_group)
    c.rope_base = float(p.rope_base)
    c.interp = float(p.interp)
    c.seg1_len = int(p.seg1_len)
    c.term_start = int(p.term_start)
    c.window = int(p.window)
    c.w0 = int(p.w0)
    c.w_pretrained = int(p.w_pretrained)
    c.softmax_scale = float(p.softmax_scale)
    c.pairing = int(p.pairing)
    return c


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m position_remapping_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    P = ctypes.POINTER(CParams)
    lib.ropeattn_posmap.argtypes = [P, i64, vp, vp, ctypes.POINTER(i32), vp]
    lib.ropeattn_cache_write.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i32, i32, P, vp]
    lib.ropeattn_prefill_workspace_size.argtypes = [P, i64, i64, i32, i32, i32]
    lib.ropeattn_prefill_workspace_size.restype = sz
    lib.ropeattn_prefill.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, P, vp, sz, vp]
    lib.ropeattn_prefill_prepare.argtypes = [vp, i64, i64, i32, i32, i32, P, vp, sz, vp]
    lib.ropeattn_prefill_attend.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, P, vp, sz, vp]
    lib.ropeattn_prefill_chunk_workspace_size.argtypes = [P, i64, i64, i64, i32, i32, i32]
    lib.ropeattn_prefill_chunk_workspace_size.restype = sz
    lib.ropeattn_prefill_chunk.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, P, vp, sz, vp]
    lib.ropeattn_prefill_chunk_cache.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, i32, i32, P, vp, sz, vp]
    lib.ropeattn_prefill_chunk_cache.restype = ctypes.c_int
    lib.ropeattn_prefill_three_call_workspace_size.argtypes = [P, i64, i64, i32, i32, i32]
    lib.ropeattn_prefill_three_call_workspace_size.restype = sz
    lib.ropeattn_prefill_three_call.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, P, vp, sz, vp]
    lib.ropeattn_decode_workspace_size.argtypes = [i64, i64, i32, i32, i32]
    lib.ropeattn_decode_workspace_size.restype = sz
    lib.ropeattn_decode.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, P, vp, sz, vp]
    lib.ropeattn_decode_cache.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, P, vp, sz, vp]
    lib.ropeattn_decode_cache.restype = ctypes.c_int
    lib.ropeattn_decode_unfused_workspace_size.argtypes = [i64, i64, i32, i32, i32]
    lib.ropeattn_decode_unfused_workspace_size.restype = sz
    lib.ropeattn_decode_unfused.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, P, vp, sz, vp]
    lib.ropeattn_decode_unfused.restype = ctypes.c_int
    lib.ropeattn_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, P, vp]
    lib.ropeattn_decode_noalloc.restype = ctypes.c_int
    lib.ropeattn_prefill_backward_workspace_size.argtypes = [P, i64, i64, i32, i32, i32]
    lib.ropeattn_prefill_backward_workspace_size.restype = sz
    lib.ropeattn_prefill_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, P, vp, sz,
                                              vp]
    lib.ropeattn_prefill_backward.restype = ctypes.c_int
    lib.ropeattn_status.argtypes = []
    lib.ropeattn_wait_selftest.argtypes = [i64, vp, vp]
    lib.ropeattn_wait_selftest.restype = ctypes.c_int
    lib.ropeattn_last_error.argtypes = []
    lib.ropeattn_last_error.restype = ctypes.c_char_p
    lib.ropeattn_version.argtypes = []
    for name in ("ropeattn_posmap", "ropeattn_cache_write", "ropeattn_prefill", "ropeattn_prefill_chunk",
                 "ropeattn_prefill_three_call", "ropeattn_prefill_prepare", "ropeattn_prefill_attend",
                 "ropeattn_decode", "ropeattn_status", "ropeattn_version"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


lib = _load()


def _check(rc: int):
    if rc != OK:
        raise RopeAttnError(rc, lib.ropeattn_last_error().decode())


def _current_device() -> int:
    return torch.cuda.current_device()


def _device_of(t: torch.Tensor):
    idx = t.get_device()   # -1 for a CPU tensor
    if idx >= 0 and t.is_cuda:
        return "cuda", idx
    d = t.device
    return d.type, d.index


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    idx = getattr(stream, "device_index", None)
    if idx is None:
        dev = getattr(stream, "device", None)
        idx = None if dev is None else dev.index
    if idx is not None and idx != _current_device():
        raise ValueError(f"the stream belongs to cuda:{idx}, but the current device is cuda:{_current_device()}")
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()   # the argtypes declare void*


# The C ABI sees only pointers and sizes: the dtype, layout and device of
# every tensor are checked here, before the call.
def _need(t, name: str, dtype, shape=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if shape is not None and t.shape != shape:
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    _need_current_device(t, name)
    return t


def _need_current_device(t: torch.Tensor, name: str) -> None:
    # the library builds its TMA maps and launches on the current device, so
    # every tensor must live there (a pointer into another GPU's memory would
    # be read by a kernel on this one)
    kind, index = _device_of(t)
    if kind != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (got {t.device})")
    cur = _current_device()
    if index != cur:
        raise ValueError(f"{name} is on cuda:{index}, but the current device is cuda:{cur}")


def _need_ndim(t, name: str, dtype, ndim: int) -> torch.Tensor:
    if isinstance(t, torch.Tensor) and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions (got shape {tuple(t.shape)})")
    return _need(t, name, dtype)


def _need_workspace(ws: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if ws is None:
        return None
    if not isinstance(ws, torch.Tensor) or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    _need_current_device(ws, "workspace")
    return ws


def _check_prefill_args(q, k, v):
    _need_ndim(q, "q", torch.bfloat16, 4)
    _need_ndim(k, "k", torch.bfloat16, 4)
    B, S, _, D = q.shape
    if k.shape[0] != B or k.shape[1] != S or k.shape[3] != D:
        raise ValueError(f"k {tuple(k.shape)} does not match q {tuple(q.shape)} (B, S, D)")
    _need(v, "v", torch.bfloat16, k.shape)


def _check_cache_args(q, k_cache, v_cache):
    _need_ndim(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, k_cache.shape)
    if q.shape[0] != k_cache.shape[0] or q.shape[-1] != k_cache.shape[3]:
        raise ValueError(f"q {tuple(q.shape)} does not match the cache {tuple(k_cache.shape)} (B, D)")


def version() -> int:
    return lib.ropeattn_version()


def wait_selftest(limit_ns: int = 1_000_000, stream=None) -> int:
    """Runs the bounded-wait self-test; returns the device result (0: the
    wait gave up, as it must). Follow with status() to read the timeout."""
    res = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check(lib.ropeattn_wait_selftest(int(limit_ns), _ptr(res), _stream(stream)))
    return int(res.item())


def status() -> None:
    """Raises RopeAttnError(ERR_TIMEOUT) if a kernel gave up on a bounded wait."""
    _check(lib.ropeattn_status())


def posmap(params: MapParams, L: int, device="cuda", stream=None) -> Tuple[torch.Tensor, torch.Tensor, int]:
    cp = _cparams(params)
    loc = torch.empty(max(L, 1), dtype=torch.int32, device=device)
    rem = torch.empty(max(L, 1), dtype=torch.int32, device=device)
    G = ctypes.c_int32(0)
    _check(lib.ropeattn_posmap(ctypes.byref(cp), int(L), _ptr(loc), _ptr(rem), ctypes.byref(G), _stream(stream)))
    return loc[:L], rem[:L], int(G.value)


def cache_write(k: torch.Tensor, v: Optional[torch.Tensor], k_cache: torch.Tensor, v_cache: Optional[torch.Tensor],
                params: MapParams, start: int, stream=None) -> None:
    """Stores k [B,count,Hkv,D] rotated at positions start..start+count-1 (and
    v as is) into rows start.. of k_cache / v_cache [B,cache_len,Hkv,D]."""
    _need_ndim(k, "k", torch.bfloat16, 4)
    B, count, Hkv, D = k.shape
    _need_ndim(k_cache, "k_cache", torch.bfloat16, 4)
    if k_cache.shape[0] != B or k_cache.shape[2] != Hkv or k_cache.shape[3] != D:
        raise ValueError(f"k_cache {tuple(k_cache.shape)} does not match k {tuple(k.shape)} (B, Hkv, D)")
    if (v is None) != (v_cache is None):
        raise ValueError("v and v_cache must be both given or both None")
    if v is not None:
        _need(v, "v", torch.bfloat16, k.shape)
        _need(v_cache, "v_cache", torch.bfloat16, k_cache.shape)
    cache_len = k_cache.shape[1]
    cp = _cparams(params)
    _check(lib.ropeattn_cache_write(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), B, int(start), count, cache_len,
                                    Hkv, D, ctypes.byref(cp), _stream(stream)))


def prefill_workspace_size(params: MapParams, B, S, Hq, Hkv, D) -> int:
    cp = _cparams(params)
    return int(lib.ropeattn_prefill_workspace_size(ctypes.byref(cp), B, S, Hq, Hkv, D))


def prefill_chunk_workspace_size(params: MapParams, B, start, count, Hq, Hkv, D) -> int:
    cp = _cparams(params)
    return int(lib.ropeattn_prefill_chunk_workspace_size(ctypes.byref(cp), B, start, count, Hq, Hkv, D))


def decode_workspace_size(B, n, Hq, Hkv, D) -> int:
    return int(lib.ropeattn_decode_workspace_size(B, n, Hq, Hkv, D))


def _workspace(nbytes: int, device) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, params: MapParams,
            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None, stream=None):
    """q [B,S,Hq,D], k/v [B,S,Hkv,D] bf16 contiguous on one CUDA device.
    Returns (out [B,S,Hq,D] fp32, lse [B,Hq,S] fp32)."""
    _check_prefill_args(q, k, v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty((B, S, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, S, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq, S))
    _need_workspace(workspace)
    need = prefill_workspace_size(params, B, S, Hq, Hkv, D)
    if workspace is None:
        workspace = _workspace(need, q.device)
    cp = _cparams(params)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ropeattn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, S, Hq, Hkv, D,
                                ctypes.byref(cp), _ptr(workspace), ws_bytes, _stream(stream)))
    return out, lse


def prefill_backward_workspace_size(params: MapParams, B, S, Hq, Hkv, D) -> int:
    cp = _cparams(params)
    return int(lib.ropeattn_prefill_backward_workspace_size(ctypes.byref(cp), B, S, Hq, Hkv, D))


def prefill_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
                     dout: torch.Tensor, params: MapParams, dq: Optional[torch.Tensor] = None,
                     dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None):
    """Gradients of the prefill: q, k, v as for prefill, out/lse the forward's
    results, dout [B,S,Hq,D] bf16 the upstream gradient of out. Returns
    (dq [B,S,Hq,D], dk [B,S,Hkv,D], dv [B,S,Hkv,D]), fp32."""
    _check_prefill_args(q, k, v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _need(out, "out", torch.float32, (B, S, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq, S))
    _need(dout, "dout", torch.bfloat16, (B, S, Hq, D))
    if dq is None:
        dq = torch.empty((B, S, Hq, D), dtype=torch.float32, device=q.device)
    if dk is None:
        dk = torch.empty((B, S, Hkv, D), dtype=torch.float32, device=q.device)
    if dv is None:
        dv = torch.empty((B, S, Hkv, D), dtype=torch.float32, device=q.device)
    _need(dq, "dq", torch.float32, (B, S, Hq, D))
    _need(dk, "dk", torch.float32, (B, S, Hkv, D))
    _need(dv, "dv", torch.float32, (B, S, Hkv, D))
    _need_workspace(workspace)
    if workspace is None:
        workspace = _workspace(prefill_backward_workspace_size(params, B, S, Hq, Hkv, D), q.device)
    cp = _cparams(params)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ropeattn_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                                         _ptr(dk), _ptr(dv), B, S, Hq, Hkv, D, ctypes.byref(cp), _ptr(workspace),
                                         ws_bytes, _stream(stream)))
    return dq, dk, dv


def prefill_three_call(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, params: MapParams,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None):
    """Comparator: the literal three-call bifocal prefill with a separate
    merge kernel (same layouts as prefill)."""
    _check_prefill_args(q, k, v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty((B, S, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, S, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq, S))
    _need_workspace(workspace)
    cp = _cparams(params)
    if workspace is None:
        workspace = _workspace(int(lib.ropeattn_prefill_three_call_workspace_size(ctypes.byref(cp), B, S, Hq, Hkv, D)),
                               q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ropeattn_prefill_three_call(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, S, Hq, Hkv, D,
                                           ctypes.byref(cp), _ptr(workspace), ws_bytes, _stream(stream)))
    return out, lse


def prefill_prepare(k: torch.Tensor, Hq: int, params: MapParams, workspace: torch.Tensor, stream=None) -> None:
    """First half of prefill: rotated keys and query angle tables into ``workspace``."""
    _need_ndim(k, "k", torch.bfloat16, 4)
    _need_workspace(workspace)
    B, S, Hkv, D = k.shape
    cp = _cparams(params)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ropeattn_prefill_prepare(_ptr(k), B, S, Hq, Hkv, D, ctypes.byref(cp), _ptr(workspace), ws_bytes,
                                        _stream(stream)))


def prefill_attend(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, params: MapParams,
                   out: torch.Tensor, lse: torch.Tensor, workspace: Optional[torch.Tensor], stream=None) -> None:
    """Second half of prefill: attention on a workspace filled by prefill_prepare."""
    _check_prefill_args(q, k, v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _need(out, "out", torch.float32, (B, S, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq, S))
    _need_workspace(workspace)
    cp = _cparams(params)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ropeattn_prefill_attend(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, S, Hq, Hkv, D,
                                       ctypes.byref(cp), _ptr(workspace), ws_bytes, _stream(stream)))


def prefill_chunk(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, params: MapParams, start: int,
                  out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None):
    """q [B,count,Hq,D] (tokens start..start+count-1), caches [B,cache_len,Hkv,D]
    bf16 (cache_len >= start+count; the first start+count rows are used)
    holding every key rotated at its own position. Returns
    (out [B,count,Hq,D] fp32, lse [B,Hq,count] fp32)."""
    _need_ndim(q, "q", torch.bfloat16, 4)
    _check_cache_args(q, k_cache, v_cache)
    B, count, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    cache_len = k_cache.shape[1]
    if cache_len < start + count:
        raise ValueError(f"the cache holds {cache_len} rows; start + count = {start + count}")
    if out is None:
        out = torch.empty((B, count, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, count), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, count, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq, count))
    _need_workspace(workspace)
    cp = _cparams(params)
    if workspace is None:
        workspace = _workspace(prefill_chunk_workspace_size(params, B, int(start), count, Hq, Hkv, D), q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ropeattn_prefill_chunk_cache(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), B,
                                            int(start), count, cache_len, Hq, Hkv, D, ctypes.byref(cp),
                                            _ptr(workspace), ws_bytes, _stream(stream)))
    return out, lse


def decode_cache(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, n: int, params: MapParams,
                 out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None):
    """Decode over the first n rows of caches [B, cache_len, Hkv, D] with
    spare rows (q [B,Hq,D], the token at position n-1)."""
    _need_ndim(q, "q", torch.bfloat16, 3)
    _check_cache_args(q, k_cache, v_cache)
    B, Hq, D = q.shape
    cache_len, Hkv = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq))
    _need_workspace(workspace)
    if workspace is None:
        workspace = _workspace(decode_workspace_size(B, n, Hq, Hkv, D), q.device)
    cp = _cparams(params)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ropeattn_decode_cache(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), B, int(n), cache_len,
                                     Hq, Hkv, D, ctypes.byref(cp), _ptr(workspace), ws_bytes, _stream(stream)))
    return out, lse


def decode_unfused(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, params: MapParams,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None):
    """Comparator: decode with the correction rotation as a separate pass
    (same layouts as decode)."""
    _need_ndim(q, "q", torch.bfloat16, 3)
    _check_cache_args(q, k_cache, v_cache)
    B, Hq, D = q.shape
    n, Hkv = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq))
    _need_workspace(workspace)
    if workspace is None:
        workspace = _workspace(int(lib.ropeattn_decode_unfused_workspace_size(B, n, Hq, Hkv, D)), q.device)
    cp = _cparams(params)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ropeattn_decode_unfused(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), B, n, Hq, Hkv,
                                       D, ctypes.byref(cp), _ptr(workspace), ws_bytes, _stream(stream)))
    return out, lse


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, params: MapParams,
           out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None, stream=None):
    """q [B,Hq,D] (unrotated, position n-1), caches [B,n,Hkv,D] bf16.
    Returns (out [B,Hq,D] fp32, lse [B,Hq] fp32)."""
    _need_ndim(q, "q", torch.bfloat16, 3)
    _check_cache_args(q, k_cache, v_cache)
    B, Hq, D = q.shape
    n, Hkv = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq))
    _need_workspace(workspace)
    if workspace is None:
        workspace = _workspace(decode_workspace_size(B, n, Hq, Hkv, D), q.device)
    cp = _cparams(params)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ropeattn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), B, n, Hq, Hkv, D,
                               ctypes.byref(cp), _ptr(workspace), ws_bytes, _stream(stream)))
    return out, lse
