"""Python binding of libsage_b200.so (include/sage_b200.h).

Argument marshalling only: torch provides device memory and the current
stream, and every step of the computation runs in the library's CUDA
kernels.  There is no fallback: if the library cannot be loaded, every call
raises.

Functions keep the C names: ``sage_quantize_qkv`` (and ``_noalloc``),
``sage_attn_fwd_quantized``, ``sage_attn_fwd``, ``sage_attn_fwd_host``,
``sage_quantize_qkv_nvfp4``, ``sage_attn_fwd_nvfp4``,
``sage_attn_fwd_nvfp4_host``, ``sage_attn_fwd_varlen``, ``sage_lse_merge``,
``sage_lse_merge_finalize``, ``sage_debug_qk_int32``, ``sage_debug_pv_fp32``,
``sage_debug_wait_timeout``, ``sage_get_device_status``.  The device calls
take CUDA tensors on one GPU and run with that GPU current; the ``*_host``
calls take host tensors.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsage_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "sage_b200.h")

SAGE_OK, SAGE_ERR_INVALID_ARG, SAGE_ERR_UNSUPPORTED, SAGE_ERR_WORKSPACE, SAGE_ERR_CUDA, \
    SAGE_ERR_TIMEOUT = range(6)
SAGE_BF16, SAGE_FP16 = 0, 1

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p


class SageError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{msg}: status {status}")
        self.status = status


class SageTensor(ctypes.Structure):
    _fields_ = [("ptr", _vp), ("dtype", ctypes.c_int32), ("B", _i64), ("H", _i64), ("N", _i64),
                ("D", _i64), ("sb", _i64), ("sh", _i64), ("sn", _i64)]


class SageMask(ctypes.Structure):
    _fields_ = [("ptr", _vp), ("B", _i64), ("H", _i64), ("Nq", _i64), ("Nk", _i64),
                ("sb", _i64), ("sh", _i64), ("sq", _i64), ("kind", ctypes.c_int32)]


SAGE_MASK_BOOL, SAGE_MASK_FLOAT = 0, 1


class SageQkvI8F8(ctypes.Structure):
    _fields_ = [("q", _vp), ("q_scale", _vp), ("k", _vp), ("k_scale", _vp), ("k_mean", _vp),
                ("v", _vp), ("v_scale", _vp), ("q_dot_kmean", _vp),
                ("B", _i64), ("Hq", _i64), ("Hkv", _i64), ("Nq", _i64), ("Nk", _i64), ("D", _i64)]


class SageQkvNvfp4(ctypes.Structure):
    _fields_ = [("q", _vp), ("q_sf", _vp), ("k", _vp), ("k_sf", _vp), ("v_t", _vp), ("v_sf_t", _vp),
                ("qk_correction", _vp), ("q_mean", _vp), ("k_mean", _vp), ("q_dot_kmean", _vp),
                ("B", _i64), ("Hq", _i64), ("Hkv", _i64), ("Nq", _i64), ("Nk", _i64), ("D", _i64),
                ("unpadded_k_len", _i64), ("per_block_mean", ctypes.c_int32)]


_lib = None
_lib_lock = threading.Lock()


def lib():
    """Load libsage_b200.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lib_lock:
        if _lib is None:
            _lib = _load()
    return _lib


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m quantized_attention_05_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    sig = {
        "sage_status_str": (ctypes.c_char_p, [ctypes.c_int]),
        "sage_version": (ctypes.c_char_p, []),
        "sage_get_device_status": (ctypes.c_int, [_vp, P(ctypes.c_uint32)]),
        "sage_quantize_workspace_bytes": (ctypes.c_size_t, [_i64, _i64, _i64, _i64]),
        "sage_quantize_qkv": (ctypes.c_int, [P(SageTensor), P(SageTensor), P(SageTensor), ctypes.c_int,
                                             P(SageQkvI8F8), _vp, ctypes.c_size_t, _vp]),
        "sage_attn_quantized_workspace_bytes": (ctypes.c_size_t, [P(SageQkvI8F8), P(SageMask)]),
        "sage_attn_fwd_quantized": (ctypes.c_int, [P(SageQkvI8F8), ctypes.c_int, ctypes.c_float,
                                                   ctypes.c_int, P(SageMask), _vp, ctypes.c_int32,
                                                   _i64, _i64, _i64, _vp, _vp, ctypes.c_size_t, _vp]),
        "sage_attn_fwd_workspace_bytes": (ctypes.c_size_t, [_i64, _i64, _i64, _i64, _i64, _i64,
                                                            P(SageMask)]),
        "sage_attn_fwd": (ctypes.c_int, [P(SageTensor), P(SageTensor), P(SageTensor), ctypes.c_int,
                                         ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         P(SageMask), _vp, _i64, _i64, _i64, _vp, _vp,
                                         ctypes.c_size_t, _vp]),
        "sage_attn_fwd_host_workspace_bytes": (ctypes.c_size_t, [_i64, _i64, _i64, _i64, _i64, _i64,
                                                                 P(SageMask), _i64]),
        "sage_attn_fwd_host": (ctypes.c_int, [P(SageTensor), P(SageTensor), P(SageTensor), ctypes.c_int,
                                              ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              P(SageMask), _vp, _i64, _i64, _i64, _vp, _i64, _vp,
                                              ctypes.c_size_t, _vp]),
        "sage_attn_fwd_nvfp4_host_workspace_bytes": (ctypes.c_size_t, [_i64] * 7),
        "sage_attn_fwd_nvfp4_host": (ctypes.c_int, [P(SageTensor), P(SageTensor), P(SageTensor),
                                                    ctypes.c_float, ctypes.c_int, ctypes.c_int, _i64,
                                                    ctypes.c_int, _vp, _i64, _i64, _i64, _vp, _i64, _vp,
                                                    ctypes.c_size_t, _vp]),
        "sage_attn_fwd_varlen_workspace_bytes": (ctypes.c_size_t, [_i64] * 8 + [ctypes.c_int]),
        "sage_attn_fwd_varlen": (ctypes.c_int, [P(SageTensor), P(SageTensor), P(SageTensor), _vp, _vp,
                                                _i64, _i64, _i64, ctypes.c_int, ctypes.c_float,
                                                ctypes.c_int, ctypes.c_int, _vp, _i64, _i64, _vp,
                                                _vp, ctypes.c_size_t, _vp]),
        "sage_lse_merge": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int32, _i64, _i64, _i64, _vp,
                                          _i64, _i64, _i64, _i64, ctypes.c_int, _vp]),
        "sage_lse_merge_finalize": (ctypes.c_int, [_vp, _vp, ctypes.c_int32, _i64, _i64, _i64,
                                                   _i64, _i64, _i64, _i64, _vp]),
        "sage_debug_qk_int32": (ctypes.c_int, [P(SageQkvI8F8), _i64, _i64, _i64, _i64, _vp, _vp]),
        "sage_debug_pv_fp32": (ctypes.c_int, [P(SageQkvI8F8), _vp, _i64, _i64, _i64, _vp, _vp]),
        "sage_debug_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, _vp]),
        "sage_quantize_qkv_noalloc": (ctypes.c_int, [P(SageTensor), P(SageTensor), P(SageTensor),
                                                     ctypes.c_int, P(SageQkvI8F8), _vp]),
        "sage_quantize_nvfp4_workspace_bytes": (ctypes.c_size_t, [_i64] * 6),
        "sage_quantize_qkv_nvfp4": (ctypes.c_int, [P(SageTensor), P(SageTensor), P(SageTensor),
                                                   ctypes.c_int, _i64, P(SageQkvNvfp4), _vp,
                                                   ctypes.c_size_t, _vp]),
        "sage_attn_fwd_nvfp4": (ctypes.c_int, [P(SageQkvNvfp4), ctypes.c_float, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, _vp, ctypes.c_int32,
                                               _i64, _i64, _i64, _vp, _vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


def _check(status, what):
    if status != SAGE_OK:
        msg = lib().sage_status_str(status).decode()
        raise SageError(status, f"{what} failed ({msg})")


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return SAGE_BF16
    if t.dtype == torch.float16:
        return SAGE_FP16
    raise TypeError(f"q/k/v must be bf16 or fp16, got {t.dtype}")


def _cuda_device(*tensors):
    """The one CUDA device that all the given tensors (None entries skipped)
    live on.  The device calls take device pointers, so a host tensor, or
    tensors spread over several GPUs, is refused here, before any pointer
    reaches the library; the call then runs with that device current."""
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("expected CUDA tensors (the *_host calls take host memory)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on {dev} and {t.device}: all must be on one CUDA device")
    return dev


def _as_tensor(t: torch.Tensor, layout: str = "HND") -> SageTensor:
    """Describe a 4-D tensor.  layout "HND": logical (B, H, N, D);
    "NHD": logical (B, N, H, D).  Strides are passed as they are."""
    if t.dim() != 4:
        raise ValueError("expected a 4-D tensor")
    if layout == "NHD":
        t = t.transpose(1, 2)
    elif layout != "HND":
        raise ValueError(layout)
    if t.stride(3) != 1:
        raise ValueError("the channel dimension must be contiguous")
    B, H, N, D = t.shape
    sb, sh, sn, _ = t.stride()
    return SageTensor(t.data_ptr(), _dtype_code(t), B, H, N, D, sb, sh, sn)


def _as_mask(mask: Optional[torch.Tensor], B, Hq, Nq, Nk):
    if mask is None:
        return None
    if mask.dtype not in (torch.bool, torch.uint8, torch.float32):
        raise TypeError("mask must be bool/uint8 (nonzero = attend) or float32 (added to the scores)")
    kind = SAGE_MASK_FLOAT if mask.dtype == torch.float32 else SAGE_MASK_BOOL
    m = mask
    while m.dim() < 4:
        m = m.unsqueeze(0)
    m = m.expand(m.shape[0], m.shape[1], Nq, Nk) if (m.shape[2] == 1 or m.shape[3] == 1) else m
    if m.stride(3) != 1:
        m = m.contiguous()
    mb, mh = m.shape[0], m.shape[1]
    return SageMask(m.data_ptr(), mb, mh, Nq, Nk, m.stride(0) if mb > 1 else 0,
                    m.stride(1) if mh > 1 else 0, m.stride(2), kind), m


def pad128(n):
    return (n + 127) // 128 * 128


@dataclasses.dataclass
class QuantizedQKV:
    """Quantised Q/K/V (device tensors) with the layouts of sage_qkv_i8f8."""
    q: torch.Tensor            # int8  [B, Hq, Nq_pad, D]
    q_scale: torch.Tensor      # fp32  [B, Hq, Nq_pad/128]
    k: torch.Tensor            # int8  [B, Hkv, Nk_pad, D]
    k_scale: torch.Tensor      # fp32  [B, Hkv, Nk_pad/128]
    k_mean: torch.Tensor       # fp32  [B, Hkv, D]
    v: torch.Tensor            # uint8 (E4M3) [B, Hkv, Nk_pad, D]
    v_scale: torch.Tensor      # fp32  [B, Hkv, D]
    q_dot_kmean: Optional[torch.Tensor]  # fp32 [B, Hq, Nq]
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    D: int

    @classmethod
    def empty(cls, B, Hq, Hkv, Nq, Nk, D, device, with_qdk=True):
        Nqp, Nkp = pad128(Nq), pad128(Nk)
        kw = dict(device=device)
        return cls(torch.empty(B, Hq, Nqp, D, dtype=torch.int8, **kw),
                   torch.empty(B, Hq, Nqp // 128, dtype=torch.float32, **kw),
                   torch.empty(B, Hkv, Nkp, D, dtype=torch.int8, **kw),
                   torch.empty(B, Hkv, Nkp // 128, dtype=torch.float32, **kw),
                   torch.empty(B, Hkv, D, dtype=torch.float32, **kw),
                   torch.empty(B, Hkv, Nkp, D, dtype=torch.uint8, **kw),
                   torch.empty(B, Hkv, D, dtype=torch.float32, **kw),
                   torch.empty(B, Hq, Nq, dtype=torch.float32, **kw) if with_qdk else None,
                   B, Hq, Hkv, Nq, Nk, D)

    def tensors(self):
        return (self.q, self.q_scale, self.k, self.k_scale, self.k_mean, self.v, self.v_scale,
                self.q_dot_kmean)

    def struct(self) -> SageQkvI8F8:
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        return SageQkvI8F8(p(self.q), p(self.q_scale), p(self.k), p(self.k_scale), p(self.k_mean),
                           p(self.v), p(self.v_scale), p(self.q_dot_kmean),
                           self.B, self.Hq, self.Hkv, self.Nq, self.Nk, self.D)


def _ws(nbytes, device):
    # 256-byte aligned: torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def sage_quantize_qkv(q, k, v, smooth_k=True, layout="HND", with_qdk=True,
                      out: Optional[QuantizedQKV] = None, ws: Optional[torch.Tensor] = None):
    """smooth_k + per-block INT8 Q/K + per-channel FP8 V (sage_quantize_qkv)."""
    L = lib()
    dev = _cuda_device(q, k, v, ws, *(out.tensors() if out is not None else ()))
    tq, tk, tv = _as_tensor(q, layout), _as_tensor(k, layout), _as_tensor(v, layout)
    if out is None:
        out = QuantizedQKV.empty(tq.B, tq.H, tk.H, tq.N, tk.N, tq.D, q.device, with_qdk)
    nbytes = L.sage_quantize_workspace_bytes(tk.B, tk.H, tk.N, tk.D)
    if ws is None:
        ws = _ws(nbytes, q.device)
    s = out.struct()
    with torch.cuda.device(dev):
        _check(L.sage_quantize_qkv(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv),
                                   int(bool(smooth_k)), ctypes.byref(s), ws.data_ptr(), ws.numel(),
                                   _stream(dev)), "sage_quantize_qkv")
    return out


def sage_quantize_qkv_noalloc(q, k, v, smooth_k=True, layout="HND", with_qdk=True,
                              out: Optional[QuantizedQKV] = None):
    """sage_quantize_qkv without a caller workspace: the library's own fixed
    device scratch is used instead (for callers that cannot allocate)."""
    L = lib()
    dev = _cuda_device(q, k, v, *(out.tensors() if out is not None else ()))
    tq, tk, tv = _as_tensor(q, layout), _as_tensor(k, layout), _as_tensor(v, layout)
    if out is None:
        out = QuantizedQKV.empty(tq.B, tq.H, tk.H, tq.N, tk.N, tq.D, q.device, with_qdk)
    s = out.struct()
    with torch.cuda.device(dev):
        _check(L.sage_quantize_qkv_noalloc(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv),
                                           int(bool(smooth_k)), ctypes.byref(s), _stream(dev)),
               "sage_quantize_qkv_noalloc")
    return out


def sage_attn_fwd_quantized(qkv: QuantizedQKV, causal=False, sm_scale=None, return_lse=False,
                            mask=None, out=None, out_dtype=torch.bfloat16, lse=None, ws=None):
    """Fused INT8-QK / FP8-PV attention on quantised inputs."""
    L = lib()
    dev = _cuda_device(*qkv.tensors(), mask, out, lse if return_lse else None, ws)
    if out is None:
        out = torch.empty(qkv.B, qkv.Hq, qkv.Nq, qkv.D, dtype=out_dtype, device=dev)
    if return_lse and lse is None:
        lse = torch.empty(qkv.B, qkv.Hq, qkv.Nq, dtype=torch.float32, device=dev)
    mk = _as_mask(mask, qkv.B, qkv.Hq, qkv.Nq, qkv.Nk)
    mstruct = ctypes.byref(mk[0]) if mk else None
    s = qkv.struct()
    if ws is None:
        ws = _ws(L.sage_attn_quantized_workspace_bytes(ctypes.byref(s), mstruct), dev)
    sb, sh, sn, _ = out.stride()
    with torch.cuda.device(dev):
        _check(L.sage_attn_fwd_quantized(ctypes.byref(s), int(bool(causal)),
                                         float(sm_scale) if sm_scale else 0.0, int(bool(return_lse)),
                                         mstruct, out.data_ptr(), _dtype_code(out), sb, sh, sn,
                                         lse.data_ptr() if return_lse else None, ws.data_ptr(),
                                         ws.numel(), _stream(dev)), "sage_attn_fwd_quantized")
    return (out, lse) if return_lse else out


def sage_attn_fwd_workspace_bytes(B, Hq, Hkv, Nq, Nk, D, mask_shape=None):
    m = None
    if mask_shape is not None:
        m = SageMask(None, mask_shape[0], mask_shape[1], Nq, Nk, 0, 0, Nk)
    return lib().sage_attn_fwd_workspace_bytes(B, Hq, Hkv, Nq, Nk, D,
                                              ctypes.byref(m) if m else None)


def sage_attn_fwd(q, k, v, causal=False, sm_scale=None, num_kv_heads=None, return_lse=False,
                  smooth_k=True, mask=None, layout="HND", out=None, lse=None, ws=None):
    """The whole path on bf16/fp16 Q/K/V (sage_attn_fwd): quantise, then attend.

    Returns out (same shape/layout/dtype as q) and, with return_lse, lse
    [B, Hq, Nq] fp32."""
    L = lib()
    dev = _cuda_device(q, k, v, mask, out, lse if return_lse else None, ws)
    tq, tk, tv = _as_tensor(q, layout), _as_tensor(k, layout), _as_tensor(v, layout)
    if num_kv_heads is None:
        num_kv_heads = tk.H
    if out is None:
        out = torch.empty_like(q)
    to = _as_tensor(out, layout)
    if return_lse and lse is None:
        lse = torch.empty(tq.B, tq.H, tq.N, dtype=torch.float32, device=q.device)
    mk = _as_mask(mask, tq.B, tq.H, tq.N, tk.N)
    mstruct = ctypes.byref(mk[0]) if mk else None
    nbytes = L.sage_attn_fwd_workspace_bytes(tq.B, tq.H, tk.H, tq.N, tk.N, tq.D, mstruct)
    if ws is None or ws.numel() < nbytes:
        ws = _ws(nbytes, q.device)
    with torch.cuda.device(dev):
        _check(L.sage_attn_fwd(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv),
                               int(bool(causal)), float(sm_scale) if sm_scale else 0.0,
                               int(num_kv_heads), int(bool(return_lse)), int(bool(smooth_k)),
                               mstruct, to.ptr, to.sb, to.sh, to.sn,
                               lse.data_ptr() if return_lse else None, ws.data_ptr(), ws.numel(),
                               _stream(dev)), "sage_attn_fwd")
    return (out, lse) if return_lse else out


def sage_attn_fwd_host_workspace_bytes(B, Hq, Hkv, Nq, Nk, D, mask_shape=None, chunk_groups=0):
    """Device workspace bytes of sage_attn_fwd_host (mask_shape: the mask's
    leading (B, H) or None)."""
    m = None
    if mask_shape is not None:
        m = ctypes.byref(SageMask(None, mask_shape[0], mask_shape[1], Nq, Nk, 0, 0, Nk,
                                  SAGE_MASK_BOOL))
    return lib().sage_attn_fwd_host_workspace_bytes(B, Hq, Hkv, Nq, Nk, D, m, chunk_groups)


def sage_attn_fwd_host(q, k, v, causal=False, sm_scale=None, num_kv_heads=None, return_lse=False,
                       smooth_k=True, mask=None, layout="HND", out=None, lse=None, ws=None,
                       chunk_groups=0, device=None):
    """The whole path on bf16/fp16 Q/K/V held in host memory
    (sage_attn_fwd_host): the problem is streamed through the GPU in chunks of
    (batch entry, KV head) groups with the copies overlapped with the
    kernels.  q/k/v and out/lse are CPU tensors (page-locked for the
    overlap; out and lse are allocated page-locked when not given); mask, if
    any, is a CUDA tensor.  Work is enqueued on the current stream of
    `device` (default: the current device); synchronise it before reading
    out.  Returns out (q's shape, layout and dtype) and, with return_lse,
    lse [B, Hq, Nq] fp32."""
    L = lib()
    for t in (q, k, v):
        if t.is_cuda:
            raise ValueError("sage_attn_fwd_host takes host tensors (use sage_attn_fwd for CUDA tensors)")
    device = _host_call_device(device, mask, ws)
    tq, tk, tv = _as_tensor(q, layout), _as_tensor(k, layout), _as_tensor(v, layout)
    if num_kv_heads is None:
        num_kv_heads = tk.H
    out, to, lse = _host_outputs(q, tq, layout, out, lse, return_lse)
    mk = _as_mask(mask, tq.B, tq.H, tq.N, tk.N)
    mstruct = ctypes.byref(mk[0]) if mk else None
    nbytes = L.sage_attn_fwd_host_workspace_bytes(tq.B, tq.H, tk.H, tq.N, tk.N, tq.D, mstruct,
                                                  int(chunk_groups))
    if nbytes == 0 and tq.B * tq.N:                       # (no queries: nothing to size)
        raise SageError(SAGE_ERR_INVALID_ARG, "sage_attn_fwd_host: invalid sizes")
    if ws is None or ws.numel() < nbytes:
        ws = _ws(nbytes, device)
    with torch.cuda.device(device):
        _check(L.sage_attn_fwd_host(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv),
                                    int(bool(causal)), float(sm_scale) if sm_scale else 0.0,
                                    int(num_kv_heads), int(bool(return_lse)), int(bool(smooth_k)),
                                    mstruct, to.ptr, to.sb, to.sh, to.sn,
                                    lse.data_ptr() if return_lse else None, int(chunk_groups),
                                    ws.data_ptr(), ws.numel(), _stream(device)),
               "sage_attn_fwd_host")
    return (out, lse) if return_lse else out


def _host_call_device(device, *device_tensors):
    """The GPU a host-memory call runs on (``device``, default the current
    one), after checking that its device-side tensors (mask, workspace) are
    CUDA tensors on it."""
    device = torch.device("cuda" if device is None else device)
    if device.type != "cuda":
        raise ValueError(f"device must be a CUDA device, got {device}")
    if device.index is None:
        device = torch.device("cuda", torch.cuda.current_device())
    dev = _cuda_device(*device_tensors)
    if dev is not None and dev != device:
        raise ValueError(f"mask and ws must be CUDA tensors on {device}, got {dev}")
    return device


def _host_outputs(q, tq, layout, out, lse, return_lse):
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if out.is_cuda:
        raise ValueError("out must be a host tensor")
    to = _as_tensor(out, layout)
    if return_lse:
        if lse is None:
            lse = torch.empty(tq.B, tq.H, tq.N, dtype=torch.float32, pin_memory=True)
        if lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous() or \
                lse.numel() != tq.B * tq.H * tq.N:
            raise ValueError("lse must be a contiguous fp32 host tensor [B, Hq, Nq]")
    return out, to, lse


def sage_attn_fwd_nvfp4_host_workspace_bytes(B, Hq, Hkv, Nq, Nk, D, chunk_groups=0):
    """Device workspace bytes of sage_attn_fwd_nvfp4_host."""
    return lib().sage_attn_fwd_nvfp4_host_workspace_bytes(B, Hq, Hkv, Nq, Nk, D, chunk_groups)


def sage_attn_fwd_nvfp4_host(q, k, v, sm_scale=None, causal=False, per_block_mean=True,
                             unpadded_k_len=None, return_lse=False, layout="HND", out=None, lse=None,
                             ws=None, chunk_groups=0, device=None):
    """The NVFP4 path (quantise, then attend) on bf16/fp16 Q/K/V held in host
    memory (sage_attn_fwd_nvfp4_host), streamed through the GPU in chunks of
    (batch entry, KV head) groups with the copies overlapped with the kernels.
    Host tensors as for sage_attn_fwd_host; out has q's dtype.  Returns out
    and, with return_lse, lse [B, Hq, Nq] fp32."""
    L = lib()
    for t in (q, k, v):
        if t.is_cuda:
            raise ValueError("sage_attn_fwd_nvfp4_host takes host tensors")
    device = _host_call_device(device, ws)
    tq, tk, tv = _as_tensor(q, layout), _as_tensor(k, layout), _as_tensor(v, layout)
    out, to, lse = _host_outputs(q, tq, layout, out, lse, return_lse)
    nbytes = L.sage_attn_fwd_nvfp4_host_workspace_bytes(tq.B, tq.H, tk.H, tq.N, tk.N, tq.D,
                                                        int(chunk_groups))
    if nbytes == 0 and tq.B * tq.N:
        raise SageError(SAGE_ERR_INVALID_ARG, "sage_attn_fwd_nvfp4_host: invalid sizes")
    if ws is None or ws.numel() < nbytes:
        ws = _ws(nbytes, device)
    with torch.cuda.device(device):
        _check(L.sage_attn_fwd_nvfp4_host(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv),
                                          float(sm_scale) if sm_scale else 0.0, int(bool(causal)),
                                          int(bool(per_block_mean)),
                                          int(unpadded_k_len) if unpadded_k_len else 0,
                                          int(bool(return_lse)), to.ptr, to.sb, to.sh, to.sn,
                                          lse.data_ptr() if return_lse else None, int(chunk_groups),
                                          ws.data_ptr(), ws.numel(), _stream(device)),
               "sage_attn_fwd_nvfp4_host")
    return (out, lse) if return_lse else out


def _packed(t: torch.Tensor) -> SageTensor:
    """Describe a packed [total, H, D] tensor (B = 1)."""
    if t.dim() != 3:
        raise ValueError("expected a packed [total, H, D] tensor")
    sn, sh, sd = t.stride()
    if sd != 1:
        raise ValueError("the channel stride must be 1")
    return SageTensor(t.data_ptr(), _dtype_code(t), 1, t.shape[1], t.shape[0], t.shape[2],
                      0, sh, sn)


def sage_attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                         causal=False, sm_scale=None, smooth_k=True, return_lse=False,
                         out=None, lse=None, ws=None):
    """Variable-length attention on packed sequences (sage_attn_fwd_varlen).

    q: [total_q, Hq, D], k/v: [total_k, Hkv, D] (bf16/fp16, CUDA);
    cu_seqlens_q/k: int32 CUDA tensors [nseq + 1].  Returns out
    [total_q, Hq, D] and, with return_lse, lse (fp32, one [Hq, len_s] block
    per sequence, flat)."""
    L = lib()
    dev = _cuda_device(q, k, v, cu_seqlens_q, cu_seqlens_k, out, lse if return_lse else None, ws)
    tq, tk, tv = _packed(q), _packed(k), _packed(v)
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    nseq = cu_seqlens_q.numel() - 1
    if cu_seqlens_k.numel() != nseq + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k describe different numbers of sequences")
    cq, ck = cu_seqlens_q.contiguous(), cu_seqlens_k.contiguous()
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    sn, sh, sd = out.stride()
    if sd != 1:
        raise ValueError("out: the channel stride must be 1")
    if return_lse and lse is None:
        lse = torch.empty(q.shape[0] * q.shape[1], dtype=torch.float32, device=q.device)
    nbytes = L.sage_attn_fwd_varlen_workspace_bytes(nseq, tq.H, tk.H, tq.N, tk.N, int(max_seqlen_q),
                                                    int(max_seqlen_k), tq.D, int(bool(return_lse)))
    if ws is None or ws.numel() < nbytes:
        ws = _ws(nbytes, q.device)
    with torch.cuda.device(dev):
        _check(L.sage_attn_fwd_varlen(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv),
                                      cq.data_ptr(), ck.data_ptr(), nseq, int(max_seqlen_q),
                                      int(max_seqlen_k), int(bool(causal)),
                                      float(sm_scale) if sm_scale else 0.0, int(bool(smooth_k)),
                                      int(bool(return_lse)), out.data_ptr(), sn, sh,
                                      lse.data_ptr() if return_lse else None, ws.data_ptr(),
                                      ws.numel(), _stream(dev)), "sage_attn_fwd_varlen")
    return (out, lse) if return_lse else out


def sage_lse_merge(acc, acc_lse, part, part_lse, init=False):
    """Merge a partial attention result (part [B, H, N, D] bf16/fp16 in any
    layout with channel stride 1, part_lse [B, H, N]) into the running fp32
    (acc [B, H, N, D] contiguous, acc_lse [B, H, N]) in place."""
    dev = _cuda_device(acc, acc_lse, part, part_lse)
    B, H, N, D = part.shape
    sb, sh, sn, sd = part.stride()
    if sd != 1 or not acc.is_contiguous() or acc.dtype != torch.float32 or acc_lse.dtype != torch.float32:
        raise ValueError("acc must be contiguous fp32 and part must have channel stride 1")
    if part_lse.dtype != torch.float32 or not part_lse.is_contiguous() or not acc_lse.is_contiguous():
        raise ValueError("the LSE tensors must be contiguous fp32")
    with torch.cuda.device(dev):
        _check(lib().sage_lse_merge(acc.data_ptr(), acc_lse.data_ptr(), part.data_ptr(),
                                    _dtype_code(part), sb, sh, sn, part_lse.data_ptr(), B, H, N, D,
                                    int(bool(init)), _stream(dev)), "sage_lse_merge")


def sage_lse_merge_finalize(acc, out):
    """Write the merged fp32 result into ``out`` (bf16/fp16 [B, H, N, D])."""
    dev = _cuda_device(acc, out)
    B, H, N, D = out.shape
    sb, sh, sn, sd = out.stride()
    if sd != 1 or not acc.is_contiguous():
        raise ValueError("out must have channel stride 1 and acc be contiguous")
    with torch.cuda.device(dev):
        _check(lib().sage_lse_merge_finalize(acc.data_ptr(), out.data_ptr(), _dtype_code(out), sb, sh,
                                             sn, B, H, N, D, _stream(dev)), "sage_lse_merge_finalize")
    return out


def sage_debug_qk_int32(qkv: QuantizedQKV, b, h, qblk, kblk):
    dev = _cuda_device(*qkv.tensors())
    tile = torch.empty(128, 128, dtype=torch.int32, device=dev)
    s = qkv.struct()
    with torch.cuda.device(dev):
        _check(lib().sage_debug_qk_int32(ctypes.byref(s), b, h, qblk, kblk, tile.data_ptr(),
                                         _stream(dev)), "sage_debug_qk_int32")
    return tile


def sage_debug_pv_fp32(qkv: QuantizedQKV, p_e4m3: torch.Tensor, b, h_kv, kblk):
    dev = _cuda_device(*qkv.tensors(), p_e4m3)
    p = p_e4m3.contiguous().view(torch.uint8)
    acc = torch.empty(128, qkv.D, dtype=torch.float32, device=dev)
    s = qkv.struct()
    with torch.cuda.device(dev):
        _check(lib().sage_debug_pv_fp32(ctypes.byref(s), p.data_ptr(), b, h_kv, kblk, acc.data_ptr(),
                                        _stream(dev)), "sage_debug_pv_fp32")
    return acc


def sage_debug_wait_timeout(timeout_us=1000):
    _check(lib().sage_debug_wait_timeout(int(timeout_us), _stream()), "sage_debug_wait_timeout")


def sage_get_device_status():
    """(status, site): SAGE_OK or SAGE_ERR_TIMEOUT with the wait site."""
    site = ctypes.c_uint32(0)
    st = lib().sage_get_device_status(_stream(), ctypes.byref(site))
    return st, site.value


@dataclasses.dataclass
class QuantizedNvfp4:
    """NVFP4 quantised Q/K/V (device tensors) with the layouts of sage_qkv_nvfp4."""
    q: torch.Tensor              # u8 [B, Hq, Nq_pad, D/2]   packed E2M1
    q_sf: torch.Tensor           # u8 [B, Hq, Nq_pad, D/16]  E4M3
    k: torch.Tensor              # u8 [B, Hkv, Nk_pad, D/2]
    k_sf: torch.Tensor           # u8 [B, Hkv, Nk_pad, D/16]
    v_t: torch.Tensor            # u8 [B, Hkv, D, Nk_pad/2]
    v_sf_t: torch.Tensor         # u8 [B, Hkv, D, Nk_pad/16]
    qk_correction: torch.Tensor  # fp32 [B, Hq, Nq_pad/128, Nk_pad]
    q_mean: torch.Tensor         # fp32 [B, Hq, Nq_pad/128, D]
    k_mean: torch.Tensor         # fp32 [B, Hkv, D]
    q_dot_kmean: Optional[torch.Tensor]
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    D: int
    unpadded_k_len: int
    per_block_mean: bool

    @classmethod
    def empty(cls, B, Hq, Hkv, Nq, Nk, D, unpadded_k_len, per_block_mean, device, with_qdk=True):
        Nqp, Nkp = pad128(Nq), pad128(Nk)
        u8 = dict(dtype=torch.uint8, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        return cls(torch.empty(B, Hq, Nqp, D // 2, **u8), torch.empty(B, Hq, Nqp, D // 16, **u8),
                   torch.empty(B, Hkv, Nkp, D // 2, **u8), torch.empty(B, Hkv, Nkp, D // 16, **u8),
                   torch.empty(B, Hkv, D, Nkp // 2, **u8), torch.empty(B, Hkv, D, Nkp // 16, **u8),
                   torch.empty(B, Hq, Nqp // 128, Nkp, **f32), torch.empty(B, Hq, Nqp // 128, D, **f32),
                   torch.empty(B, Hkv, D, **f32),
                   torch.empty(B, Hq, Nq, **f32) if with_qdk else None,
                   B, Hq, Hkv, Nq, Nk, D, unpadded_k_len, bool(per_block_mean))

    def tensors(self):
        return (self.q, self.q_sf, self.k, self.k_sf, self.v_t, self.v_sf_t, self.qk_correction,
                self.q_mean, self.k_mean, self.q_dot_kmean)

    def struct(self) -> SageQkvNvfp4:
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        return SageQkvNvfp4(p(self.q), p(self.q_sf), p(self.k), p(self.k_sf), p(self.v_t),
                            p(self.v_sf_t), p(self.qk_correction), p(self.q_mean), p(self.k_mean),
                            p(self.q_dot_kmean), self.B, self.Hq, self.Hkv, self.Nq, self.Nk, self.D,
                            self.unpadded_k_len, int(self.per_block_mean))


def sage_quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=None, layout="HND",
                            with_qdk=True, out: Optional[QuantizedNvfp4] = None,
                            ws: Optional[torch.Tensor] = None):
    """NVFP4 quantisation (sage_quantize_qkv_nvfp4)."""
    L = lib()
    dev = _cuda_device(q, k, v, ws, *(out.tensors() if out is not None else ()))
    tq, tk, tv = _as_tensor(q, layout), _as_tensor(k, layout), _as_tensor(v, layout)
    ukl = tk.N if unpadded_k_len is None else int(unpadded_k_len)
    if out is None:
        out = QuantizedNvfp4.empty(tq.B, tq.H, tk.H, tq.N, tk.N, tq.D, ukl, per_block_mean,
                                   q.device, with_qdk)
    if ws is None:
        ws = _ws(L.sage_quantize_nvfp4_workspace_bytes(tq.B, tq.H, tk.H, tq.N, tk.N, tq.D), q.device)
    s = out.struct()
    with torch.cuda.device(dev):
        _check(L.sage_quantize_qkv_nvfp4(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv),
                                         int(bool(per_block_mean)), ukl, ctypes.byref(s),
                                         ws.data_ptr(), ws.numel(), _stream(dev)),
               "sage_quantize_qkv_nvfp4")
    return out


def sage_attn_fwd_nvfp4(qkv: QuantizedNvfp4, sm_scale=None, causal=False, per_block_mean=None,
                        return_lse=True, out=None, out_dtype=torch.bfloat16, lse=None):
    """NVFP4 attention on pre-quantised inputs (sage_attn_fwd_nvfp4)."""
    L = lib()
    dev = _cuda_device(*qkv.tensors(), out, lse if return_lse else None)
    pbm = qkv.per_block_mean if per_block_mean is None else bool(per_block_mean)
    if out is None:
        out = torch.empty(qkv.B, qkv.Hq, qkv.Nq, qkv.D, dtype=out_dtype, device=dev)
    if return_lse and lse is None:
        lse = torch.empty(qkv.B, qkv.Hq, qkv.Nq, dtype=torch.float32, device=dev)
    sb, sh, sn, _ = out.stride()
    s = qkv.struct()
    with torch.cuda.device(dev):
        _check(L.sage_attn_fwd_nvfp4(ctypes.byref(s), float(sm_scale) if sm_scale else 0.0,
                                     int(bool(causal)), int(pbm), int(bool(return_lse)),
                                     out.data_ptr(), _dtype_code(out), sb, sh, sn,
                                     lse.data_ptr() if return_lse else None, _stream(dev)),
               "sage_attn_fwd_nvfp4")
    return (out, lse) if return_lse else out
