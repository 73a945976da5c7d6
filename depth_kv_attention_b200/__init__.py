"""Python binding of the MoDA C ABI (``libmoda.so``, header ``include/moda.h``).

Argument marshalling only: every function forwards torch CUDA tensors' device
pointers and the current CUDA stream to the C entry point of the same name.
All arithmetic runs in the library's CUDA kernels. There is no CPU fallback:
importing this package fails if the library has not been built
(``python depth_kv_attention_b200/csrc/build.py``).

Layouts (contiguous): q/out/dout [B,T,Hq,d]; k/v [B,T,Hkv,d];
kd/vd [B,T,Ld,Hkv,d]; lse [B,Hq,T] fp32.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "MODA_OK", "ModaError", "lib", "LIB_PATH", "moda_abi_version", "moda_status_string",
    "moda_fwd", "moda_fwd_sel", "moda_bwd", "moda_bwd_sel", "moda_bwd_workspace_bytes", "moda_bwd_noalloc", "moda_pack_depth",
    "moda_pack_depth_bytes", "moda_fwd_packed", "moda_depth_write", "moda_device_status",
    "moda_debug_set_wait_limit", "moda_debug_exp2_poly", "moda_fwd_from_host",
    "moda_fwd_host_staging_bytes", "moda_fwd_q8", "moda_depth_quantize_q8", "moda_depth_write_q8",
    "moda_depth_slot_layout", "depth_slot_view",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoda.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python depth_kv_attention_b200/csrc/build.py` "
        "(the MoDA path has no CPU fallback)")
lib = ctypes.CDLL(LIB_PATH)

MODA_OK = 0
_DTYPE = {torch.bfloat16: 0, torch.float32: 1}
_IMPL = {"auto": 0, "simt": 1, "tc": 2, "tc2": 3}
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def _sig(name, res, args):
    fn = getattr(lib, name)
    fn.restype = res
    fn.argtypes = args
    return fn


_DIMS = [_i] * 6  # B, T, Hq, Hkv, d, Ld
_c_abi_version = _sig("moda_abi_version", _i, [])
_c_status_string = _sig("moda_status_string", ctypes.c_char_p, [_i])
_c_fwd_ex = _sig("moda_fwd_ex", _i, [_vp] * 5 + _DIMS + [_i, _f, _vp, _vp, _vp, _i])
_c_fwd = _sig("moda_fwd", _i, [_vp] * 5 + _DIMS + [_i, _f, _vp, _vp, _vp])
_c_fwd_sel = _sig("moda_fwd_sel", _i, [_vp] * 6 + _DIMS + [_i, _f, _vp, _vp, _vp, _i])
_c_bwd_ws = _sig("moda_bwd_workspace_bytes", _sz, _DIMS + [_i])
_c_bwd_ex = _sig("moda_bwd_ex", _i, [_vp] * 8 + _DIMS + [_i, _f] + [_vp] * 5 + [_vp, _sz, _vp, _i])
_c_bwd = _sig("moda_bwd", _i, [_vp] * 8 + _DIMS + [_i, _f] + [_vp] * 5 + [_vp, _sz, _vp])
_c_bwd_sel = _sig("moda_bwd_sel", _i, [_vp] * 9 + _DIMS + [_i, _f] + [_vp] * 5 + [_vp, _sz, _vp, _i])
_c_pack_bytes = _sig("moda_pack_depth_bytes", _sz, [_i] * 5 + [_i])
_c_pack = _sig("moda_pack_depth", _i, [_vp, _vp] + [_i] * 5 + [_i, _vp, _vp])
_c_fwd_packed = _sig("moda_fwd_packed", _i, [_vp] * 4 + _DIMS + [_i, _f, _vp, _vp, _vp])
_c_depth_write = _sig("moda_depth_write", _i, [_vp, _vp] + [_i] * 6 + [_i, _vp, _vp, _vp])
_c_dev_status = _sig("moda_device_status", _i, [_vp])
_c_wait_limit = _sig("moda_debug_set_wait_limit", _i, [ctypes.c_uint32])
_c_exp2_poly = _sig("moda_debug_exp2_poly", _i, [_vp, _vp, _i, _vp])
_c_bwd_noalloc = _sig("moda_bwd_noalloc", _i, [_vp] * 8 + _DIMS + [_i, _f] + [_vp] * 5 + [_vp])
_c_host_bytes = _sig("moda_fwd_host_staging_bytes", _sz, _DIMS + [_i])
_c_slot_layout = _sig("moda_depth_slot_layout", _i, [_i] * 6 + [ctypes.POINTER(ctypes.c_longlong),
                                                                  ctypes.POINTER(ctypes.c_longlong)])
_c_fwd_q8 = _sig("moda_fwd_q8", _i, [_vp] * 7 + _DIMS + [_i, _f, _vp, _vp, _vp, _i])
_c_quant_q8 = _sig("moda_depth_quantize_q8", _i, [_vp, _vp] + [_i] * 5 + [_i] + [_vp] * 4 + [_vp])
_c_write_q8 = _sig("moda_depth_write_q8", _i, [_vp, _vp] + [_i] * 6 + [_i] + [_vp] * 4 + [_vp])
_c_fwd_host = _sig("moda_fwd_host", _i, [_vp] * 5 + _DIMS + [_i, _f, _vp, _vp, _vp, _sz, _vp])


class ModaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {moda_status_string(code)} ({code})")


def moda_abi_version() -> int:
    return _c_abi_version()


def moda_status_string(code: int) -> str:
    return _c_status_string(code).decode()


def _check(code: int, where: str) -> None:
    if code != MODA_OK:
        raise ModaError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dims(q, k, kd):
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    Ld = 0 if kd is None else kd.shape[2]
    return B, T, Hq, Hkv, d, Ld


def _check_tensors(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("MoDA tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("MoDA tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("MoDA tensors must be on one device")


def moda_fwd(q, k, v, kd=None, vd=None, scale: float | None = None, out=None, lse=None,
             impl: str = "auto", stream=None):
    """MoDA forward (``moda_fwd_ex``). Returns (out, lse)."""
    if kd is not None and kd.shape[2] == 0:
        kd = vd = None
    _check_tensors(q, k, v, kd, vd, out, lse)
    B, T, Hq, Hkv, d, Ld = _dims(q, k, kd)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    with torch.cuda.device(q.device):
        _check(_c_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(kd), _ptr(vd), B, T, Hq, Hkv, d, Ld,
                         _DTYPE[q.dtype], scale, _ptr(out), _ptr(lse), _stream(stream), _IMPL[impl]),
               "moda_fwd")
    return out, lse


def _check_sel(depth_sel, B, T):
    if depth_sel is None:
        return
    if depth_sel.dtype != torch.int64 or tuple(depth_sel.shape) != (B, T):
        raise ValueError("depth_sel must be an int64 [B, T] tensor of depth-slot bit masks")


def moda_fwd_sel(q, k, v, kd, vd, depth_sel, scale: float | None = None, out=None, lse=None,
                 impl: str = "auto", stream=None):
    """MoDA forward with per-token depth-slot selection (``moda_fwd_sel``).

    ``depth_sel``: int64 [B, T] bit masks (bit i set = the token's depth slot
    i takes part), or None for every slot. Returns (out, lse)."""
    _check_tensors(q, k, v, kd, vd, depth_sel, out, lse)
    B, T, Hq, Hkv, d, Ld = _dims(q, k, kd)
    _check_sel(depth_sel, B, T)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    with torch.cuda.device(q.device):
        _check(_c_fwd_sel(_ptr(q), _ptr(k), _ptr(v), _ptr(kd), _ptr(vd), _ptr(depth_sel), B, T, Hq,
                          Hkv, d, Ld, _DTYPE[q.dtype], scale, _ptr(out), _ptr(lse), _stream(stream),
                          _IMPL[impl]), "moda_fwd_sel")
    return out, lse


def moda_bwd_sel(q, k, v, kd, vd, depth_sel, out, lse, dout, scale: float | None = None,
                 grads=None, workspace=None, impl: str = "auto", stream=None):
    """Gradients of ``moda_fwd_sel`` (``moda_bwd_sel``), same ``depth_sel``.
    Returns (dq, dk, dv, dkd, dvd)."""
    _check_tensors(q, k, v, kd, vd, depth_sel, out, lse, dout)
    B, T, Hq, Hkv, d, Ld = _dims(q, k, kd)
    _check_sel(depth_sel, B, T)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 torch.empty_like(kd), torch.empty_like(vd))
    dq, dk, dv, dkd, dvd = grads
    need = moda_bwd_workspace_bytes(B, T, Hq, Hkv, d, Ld, q.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    with torch.cuda.device(q.device):
        _check(_c_bwd_sel(_ptr(q), _ptr(k), _ptr(v), _ptr(kd), _ptr(vd), _ptr(depth_sel), _ptr(out),
                          _ptr(lse), _ptr(dout), B, T, Hq, Hkv, d, Ld, _DTYPE[q.dtype], scale,
                          _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dkd), _ptr(dvd), _ptr(workspace),
                          workspace.numel(), _stream(stream), _IMPL[impl]), "moda_bwd_sel")
    return dq, dk, dv, dkd, dvd


def moda_bwd_workspace_bytes(B, T, Hq, Hkv, d, Ld, dtype) -> int:
    return _c_bwd_ws(B, T, Hq, Hkv, d, Ld, _DTYPE[dtype])


def moda_bwd(q, k, v, kd, vd, out, lse, dout, scale: float | None = None, grads=None,
             workspace=None, impl: str = "auto", stream=None):
    """MoDA backward (``moda_bwd_ex``). Returns (dq, dk, dv, dkd, dvd)."""
    if kd is not None and kd.shape[2] == 0:
        kd = vd = None
    _check_tensors(q, k, v, kd, vd, out, lse, dout)
    B, T, Hq, Hkv, d, Ld = _dims(q, k, kd)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 None if kd is None else torch.empty_like(kd),
                 None if vd is None else torch.empty_like(vd))
    dq, dk, dv, dkd, dvd = grads
    need = moda_bwd_workspace_bytes(B, T, Hq, Hkv, d, Ld, q.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    with torch.cuda.device(q.device):
        _check(_c_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(kd), _ptr(vd), _ptr(out), _ptr(lse),
                         _ptr(dout), B, T, Hq, Hkv, d, Ld, _DTYPE[q.dtype], scale, _ptr(dq),
                         _ptr(dk), _ptr(dv), _ptr(dkd), _ptr(dvd), _ptr(workspace),
                         workspace.numel(), _stream(stream), _IMPL[impl]), "moda_bwd")
    return dq, dk, dv, dkd, dvd


def moda_bwd_noalloc(q, k, v, kd, vd, out, lse, dout, scale: float | None = None, grads=None,
                     stream=None):
    """``moda_bwd_noalloc``: the backward without a workspace argument, for
    callers that cannot allocate device memory (the library's fixed scratch
    array holds the row statistics). Output tensors come from ``grads`` or
    are created here by torch (the C call itself allocates nothing).
    Returns (dq, dk, dv, dkd, dvd)."""
    if kd is not None and kd.shape[2] == 0:
        kd = vd = None
    _check_tensors(q, k, v, kd, vd, out, lse, dout)
    B, T, Hq, Hkv, d, Ld = _dims(q, k, kd)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 None if kd is None else torch.empty_like(kd),
                 None if vd is None else torch.empty_like(vd))
    dq, dk, dv, dkd, dvd = grads
    with torch.cuda.device(q.device):
        _check(_c_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(kd), _ptr(vd), _ptr(out), _ptr(lse),
                              _ptr(dout), B, T, Hq, Hkv, d, Ld, _DTYPE[q.dtype], scale, _ptr(dq),
                              _ptr(dk), _ptr(dv), _ptr(dkd), _ptr(dvd), _stream(stream)),
               "moda_bwd_noalloc")
    return dq, dk, dv, dkd, dvd


def moda_pack_depth_bytes(B, T, Hkv, d, Ld, dtype) -> int:
    return _c_pack_bytes(B, T, Hkv, d, Ld, _DTYPE[dtype])


def moda_pack_depth(kd, vd, packed=None, stream=None):
    """Repack kd, vd [B,T,Ld,Hkv,d] into [2,B,Hkv,T*Ld,d] (``moda_pack_depth``)."""
    _check_tensors(kd, vd, packed)
    B, T, Ld, Hkv, d = kd.shape
    n = moda_pack_depth_bytes(B, T, Hkv, d, Ld, kd.dtype)
    if packed is None:
        packed = torch.empty(n // kd.element_size(), device=kd.device, dtype=kd.dtype)
    with torch.cuda.device(kd.device):
        _check(_c_pack(_ptr(kd), _ptr(vd), B, T, Hkv, d, Ld, _DTYPE[kd.dtype], _ptr(packed),
                       _stream(stream)), "moda_pack_depth")
    return packed


def moda_fwd_packed(q, k, v, packed, Ld: int, scale: float | None = None, out=None, lse=None,
                    stream=None):
    """MoDA forward reading depth from ``moda_pack_depth``'s layout."""
    _check_tensors(q, k, v, packed, out, lse)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    with torch.cuda.device(q.device):
        _check(_c_fwd_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(packed) if Ld else None, B, T, Hq,
                             Hkv, d, Ld, _DTYPE[q.dtype], scale, _ptr(out), _ptr(lse),
                             _stream(stream)), "moda_fwd_packed")
    return out, lse


def moda_depth_write(k, v, kd, vd, slot: int, stream=None):
    """The write step (``moda_depth_write``): k, v [B,T,Hkv,d] into slot
    ``slot`` of the depth cache kd, vd [B,T,Ld,Hkv,d], in place. Returns (kd, vd)."""
    _check_tensors(k, v, kd, vd)
    B, T, Hkv, d = k.shape
    Ld = kd.shape[2]
    if tuple(v.shape) != (B, T, Hkv, d) or tuple(kd.shape) != (B, T, Ld, Hkv, d) or kd.shape != vd.shape:
        raise ValueError("moda_depth_write: k, v [B,T,Hkv,d] and kd, vd [B,T,Ld,Hkv,d] expected")
    if not (k.dtype == v.dtype == kd.dtype == vd.dtype):
        raise ValueError("moda_depth_write: one dtype expected")
    with torch.cuda.device(k.device):
        _check(_c_depth_write(_ptr(k), _ptr(v), B, T, Hkv, d, Ld, slot, _DTYPE[k.dtype], _ptr(kd),
                              _ptr(vd), _stream(stream)), "moda_depth_write")
    return kd, vd


def moda_depth_quantize_q8(kd, vd, out=None, stream=None):
    """8-bit depth cache of kd, vd [B,T,Ld,Hkv,d] (``moda_depth_quantize_q8``).
    Returns (kd8, vd8, kd_scale, vd_scale): int8 codes [B,T,Ld,Hkv,d] and fp32
    row scales [B,T,Ld,Hkv]; ``out`` may supply those four tensors."""
    _check_tensors(kd, vd)
    B, T, Ld, Hkv, d = kd.shape
    if out is None:
        out = (torch.empty(kd.shape, dtype=torch.int8, device=kd.device),
               torch.empty(kd.shape, dtype=torch.int8, device=kd.device),
               torch.empty(kd.shape[:-1], dtype=torch.float32, device=kd.device),
               torch.empty(kd.shape[:-1], dtype=torch.float32, device=kd.device))
    _check_tensors(*out)
    with torch.cuda.device(kd.device):
        _check(_c_quant_q8(_ptr(kd), _ptr(vd), B, T, Hkv, d, Ld, _DTYPE[kd.dtype], *(_ptr(t) for t in out),
                           _stream(stream)), "moda_depth_quantize_q8")
    return out


def moda_depth_write_q8(k, v, kd8, vd8, kd_scale, vd_scale, slot: int, stream=None):
    """The write step into an 8-bit depth cache (``moda_depth_write_q8``): k, v
    [B,T,Hkv,d] quantised into slot ``slot`` of kd8, vd8 and their scales, in
    place. Returns (kd8, vd8, kd_scale, vd_scale)."""
    _check_tensors(k, v, kd8, vd8, kd_scale, vd_scale)
    B, T, Hkv, d = k.shape
    Ld = kd8.shape[2]
    if kd8.dtype != torch.int8 or kd_scale.dtype != torch.float32 or tuple(kd8.shape) != (B, T, Ld, Hkv, d):
        raise ValueError("moda_depth_write_q8: int8 kd8 [B,T,Ld,Hkv,d] and fp32 scales [B,T,Ld,Hkv] expected")
    with torch.cuda.device(k.device):
        _check(_c_write_q8(_ptr(k), _ptr(v), B, T, Hkv, d, Ld, slot, _DTYPE[k.dtype], _ptr(kd8), _ptr(vd8),
                           _ptr(kd_scale), _ptr(vd_scale), _stream(stream)), "moda_depth_write_q8")
    return kd8, vd8, kd_scale, vd_scale


def moda_fwd_q8(q, k, v, kd8, vd8, kd_scale, vd_scale, scale: float | None = None, out=None, lse=None,
                impl: str = "auto", stream=None):
    """MoDA forward over an 8-bit depth cache (``moda_fwd_q8``). Returns (out, lse)."""
    if kd8 is not None and kd8.shape[2] == 0:
        kd8 = vd8 = kd_scale = vd_scale = None
    _check_tensors(q, k, v, kd8, vd8, kd_scale, vd_scale, out, lse)
    B, T, Hq, Hkv, d, Ld = _dims(q, k, kd8)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    with torch.cuda.device(q.device):
        _check(_c_fwd_q8(_ptr(q), _ptr(k), _ptr(v), _ptr(kd8), _ptr(vd8), _ptr(kd_scale), _ptr(vd_scale),
                         B, T, Hq, Hkv, d, Ld, _DTYPE[q.dtype], scale, _ptr(out), _ptr(lse),
                         _stream(stream), _IMPL[impl]), "moda_fwd_q8")
    return out, lse


def moda_depth_slot_layout(B, T, Hkv, d, Ld, slot):
    """(offset, strides) of depth slot ``slot`` inside a native cache
    [B,T,Ld,Hkv,d], in elements (``moda_depth_slot_layout``)."""
    off = ctypes.c_longlong()
    st = (ctypes.c_longlong * 4)()
    _check(_c_slot_layout(B, T, Hkv, d, Ld, slot, ctypes.byref(off), st), "moda_depth_slot_layout")
    return off.value, tuple(st)


def depth_slot_view(kd, slot: int):
    """Slot ``slot`` of a depth cache kd [B,T,Ld,Hkv,d] as a strided
    [B, T, Hkv, d] view (no copy), per ``moda_depth_slot_layout``: a producer
    that writes its K or V into this view (e.g. a projection GEMM with
    ``out=view.view(B*T, Hkv*d)``-style leading dimension Ld*Hkv*d) fills the
    cache in place."""
    B, T, Ld, Hkv, d = kd.shape
    off, st = moda_depth_slot_layout(B, T, Hkv, d, Ld, slot)
    return kd.as_strided((B, T, Hkv, d), st, kd.storage_offset() + off)


def moda_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return _c_dev_status(_stream(stream))


def moda_debug_set_wait_limit(spins: int) -> None:
    _check(_c_wait_limit(spins), "moda_debug_set_wait_limit")


def moda_debug_exp2_poly(x, y=None, stream=None):
    """Apply the forward kernel's FMA-pipe exp2 to a CUDA fp32 tensor."""
    _check_tensors(x, y)
    if y is None:
        y = torch.empty_like(x)
    with torch.cuda.device(x.device):
        _check(_c_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "moda_debug_exp2_poly")
    return y


def moda_fwd_host_staging_bytes(B, T, Hq, Hkv, d, Ld, dtype) -> int:
    return _c_host_bytes(B, T, Hq, Hkv, d, Ld, _DTYPE[dtype])


def moda_fwd_from_host(q, k, v, kd=None, vd=None, scale: float | None = None, device="cuda",
                       out_host=None, lse_host=None, staging=None, stream=None):
    """End-to-end forward from HOST tensors through ``moda_fwd_host``: the C
    call enqueues the host->device copies of the inputs into the device
    ``staging`` buffer, the forward and the device->host copies of out and
    lse; this function then waits for the stream.

    ``out_host`` / ``lse_host`` (pinned CPU tensors) are filled in place when
    given, else created (pinned). ``staging`` (a CUDA uint8 tensor of at
    least ``moda_fwd_host_staging_bytes`` bytes) is created when not given.
    Returns (out_host, lse_host)."""
    if kd is not None and kd.shape[2] == 0:
        kd = vd = None
    for t in (q, k, v, kd, vd, out_host, lse_host):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("moda_fwd_from_host takes contiguous host tensors")
    B, T, Hq, Hkv, d, Ld = _dims(q, k, kd)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = torch.device(device)
    need = moda_fwd_host_staging_bytes(B, T, Hq, Hkv, d, Ld, q.dtype)
    if staging is None:
        staging = torch.empty(need, dtype=torch.uint8, device=dev)
    if out_host is None:
        out_host = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if lse_host is None:
        lse_host = torch.empty((B, Hq, T), dtype=torch.float32, pin_memory=True)
    with torch.cuda.device(staging.device):
        st = _stream(stream)
        _check(_c_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(kd), _ptr(vd), B, T, Hq, Hkv, d, Ld,
                           _DTYPE[q.dtype], scale, _ptr(out_host), _ptr(lse_host), _ptr(staging),
                           staging.numel(), st), "moda_fwd_host")
        _check(_c_dev_status(st), "moda_fwd_host (stream)")
    return out_host, lse_host
