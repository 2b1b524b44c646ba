"""Python binding of libsage2 (the B200 SageAttention2 forward pass).

Argument marshalling only: every step runs in the CUDA kernels of
``libsage2.so`` (built in-tree by ``python -m quantized_attention_04_b200.build``),
called through its C ABI (include/sage2.h).  Importing works without a GPU;
calling any compute entry point without the built library raises.

The functions keep the C names.  Tensors are torch CUDA tensors; outputs are
allocated with torch on the input's device and every call is enqueued on
torch's current stream of that device.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "sage2_smooth_quant_qk", "sage2_quant_v", "sage2_attn_fwd_quantized", "sage2_attn_fwd",
    "sage2_attn_fwd_noalloc", "sage2_attn_fwd_varlen", "sage2_attn_fwd_host", "sage2_debug_qk_s32", "sage2_workspace_bytes", "sage2_check_device_error",
    "sage2_status_string", "sage2_version", "sage2_layout_info", "attn", "Sage2Error", "lib", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsage2.so")
F16, BF16, F32 = 0, 1, 2
QK_INT4, QK_INT8, QK_INT4_PACKED = 0, 1, 2
_QKF = {4: QK_INT4, 8: QK_INT8}


def _fmt(qk_bits: int, packed: bool = False) -> int:
    """sage2_qk_format of (qk_bits, packed): packed is two INT4 values per byte."""
    if qk_bits not in _QKF:
        raise ValueError("qk_bits must be 4 or 8")
    if packed:
        if qk_bits != 4:
            raise ValueError("packed storage is for INT4 values (qk_bits=4)")
        return QK_INT4_PACKED
    return _QKF[qk_bits]
_DT = {torch.float16: F16, torch.bfloat16: BF16, torch.float32: F32}
STATUS = {0: "SAGE2_OK", 1: "SAGE2_ERR_INVALID_ARG", 2: "SAGE2_ERR_UNSUPPORTED",
          3: "SAGE2_ERR_MISALIGNED", 4: "SAGE2_ERR_CUDA", 5: "SAGE2_ERR_NO_MEM",
          6: "SAGE2_ERR_TIMEOUT", 7: "SAGE2_ERR_TOO_LARGE"}

_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SIGS = {
    "sage2_smooth_quant_qk": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "sage2_quant_v": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "sage2_attn_fwd_quantized": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sage2_attn_fwd": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sage2_attn_fwd_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sage2_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "sage2_debug_qk_s32": (_I, [_P, _P, _I, _I, _I, _I, _P, _P]),
    "sage2_smooth_quant_qk_ex": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _I, _P]),
    "sage2_quant_v_ex": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "sage2_attn_fwd_quantized_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                         _F, _I, _P]),
    "sage2_attn_fwd_ex": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "sage2_debug_qk_s32_ex": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "sage2_attn_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "sage2_check_device_error": (_I, [_P]),
    "sage2_debug_wait_timeout": (_I, [_P]),
    "sage2_attn_fwd_host": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "sage2_status_string": (ctypes.c_char_p, [_I]),
    "sage2_version": (_I, []),
    "sage2_layout_info": (_I, [_P]),
}


class _Layout(ctypes.Structure):
    _fields_ = [("version", _I), ("block_rows", _I), ("tile_keys", _I), ("int4_max", _I),
                ("int8_max", _I), ("p_scale", _F), ("v_scale_div", _F),
                ("packed_low_first", _I), ("key_perm", _I * 128), ("value_perm", _I * 128)]


class Sage2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} "
                         f"({lib().sage2_status_string(status).decode()})")


def lib() -> ctypes.CDLL:
    """The loaded libsage2.so; raises ImportError if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m quantized_attention_04_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(fn: str, status: int):
    if status != 0:
        raise Sage2Error(fn, status)


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dims(x: torch.Tensor):
    if x.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    if not x.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not x.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return x.shape


def n_pad(N: int) -> int:
    return (N + 127) // 128 * 128


def sage2_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().sage2_workspace_bytes(B, H, N, d))


def sage2_status_string(status: int) -> str:
    return lib().sage2_status_string(status).decode()


def sage2_version() -> int:
    return int(lib().sage2_version())


def sage2_layout_info() -> dict:
    """The library's layout constants (sage2_layout in include/sage2.h)."""
    lay = _Layout()
    _check("sage2_layout_info", lib().sage2_layout_info(ctypes.byref(lay)))
    d = {name: getattr(lay, name) for name, _ in _Layout._fields_}
    d["key_perm"] = list(lay.key_perm)
    d["value_perm"] = list(lay.value_perm)
    return d


def sage2_check_device_error(device=None) -> int:
    """Synchronize torch's current stream and return (and clear) the device
    error status (0 = OK, 6 = a bounded wait timed out)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    return int(lib().sage2_check_device_error(st))


def _qk_bits_of(t: torch.Tensor) -> int:
    """Payload format from the payload dtype: uint8 e4m3 codes (INT4), int8 (INT8)."""
    return 8 if t.dtype == torch.int8 else 4


def _format_of(pay: dict) -> int:
    """sage2_qk_format of a payload dict: int8 -> INT8; uint8 rows of d/2
    bytes (d from q_mean) -> packed INT4; uint8 rows of d bytes -> INT4 codes."""
    if pay["q_i4"].dtype == torch.int8:
        return QK_INT8
    return QK_INT4_PACKED if 2 * pay["q_i4"].shape[-1] == pay["q_mean"].shape[-1] else QK_INT4


QK_CAUSAL_CORR = 0x100


def sage2_smooth_quant_qk(q: torch.Tensor, k: torch.Tensor, out: dict | None = None,
                          qk_bits: int = 4, packed: bool = False,
                          causal_corr: bool = False) -> dict:
    """Smoothing + INT4 (qk_bits=4, the method) or INT8 (qk_bits=8, the variant)
    of Q and K and the Q-smoothing correction.  Returns the payload dict (q_i4,
    q_scale, q_mean, k_i4, k_scale, k_mean, qk_corr); q_i4/k_i4 are uint8 e4m3
    codes for INT4, int8 values for INT8, and with packed=True (INT4 only)
    uint8 [B,H,Np,d/2] bytes of two two's-complement nibbles (channel 2c in
    bits 3:0).  `out`, if given, is such a dict (from an earlier call with the
    same format) and is overwritten.  causal_corr writes qk_corr only where
    a causal attention reads it (key tile <= query block)."""
    fmt = _fmt(qk_bits, packed)
    B, H, N, d = _dims(q)
    if k.shape != q.shape or k.dtype != q.dtype:
        raise ValueError("q and k must have the same shape and dtype")
    _dims(k)
    Np = n_pad(N)
    NB = Np // 128
    dev = q.device
    if out is None:
        out = _qk_payloads(B, H, Np, NB, d, dev, qk_bits, packed)
    elif _format_of(out) != fmt:
        raise ValueError("out holds payloads of another format")
    st = lib().sage2_smooth_quant_qk_ex(
        _ptr(q), _ptr(k), _DT[q.dtype], B, H, N, d, _ptr(out["q_i4"]), _ptr(out["q_scale"]),
        _ptr(out["q_mean"]), _ptr(out["k_i4"]), _ptr(out["k_scale"]), _ptr(out["k_mean"]),
        _ptr(out["qk_corr"]), fmt | (QK_CAUSAL_CORR if causal_corr else 0), _stream(q))
    _check("sage2_smooth_quant_qk_ex", st)
    return out


def _qk_payloads(B, H, Np, NB, d, dev, qk_bits=4, packed=False) -> dict:
    ity = torch.uint8 if qk_bits == 4 else torch.int8   # e4m3 codes of INT4 values / INT8 values
    w = d // 2 if packed else d                          # bytes per payload row
    return dict(
        q_i4=torch.empty(B, H, Np, w, dtype=ity, device=dev),
        q_scale=torch.empty(B, H, Np, dtype=torch.float32, device=dev),
        q_mean=torch.empty(B, H, NB, d, dtype=torch.float32, device=dev),
        k_i4=torch.empty(B, H, Np, w, dtype=ity, device=dev),   # rows permuted per block
        k_scale=torch.empty(B, H, Np, dtype=torch.float32, device=dev),
        k_mean=torch.empty(B, H, d, dtype=torch.float32, device=dev),
        qk_corr=torch.empty(B, H, NB, Np, dtype=torch.float32, device=dev),
    )


def sage2_quant_v(v: torch.Tensor, out: tuple | None = None, smooth: bool = False):
    """FP8 e4m3 V per channel. Returns (v_fp8_t uint8 [B,H,d,Np], v_scale f32 [B,H,d]),
    and with smooth=True (V smoothing) also v_mean f32 [B,H,d]; `out`, if given,
    is such a tuple (from an earlier call) and is overwritten."""
    B, H, N, d = _dims(v)
    Np = n_pad(N)
    if out is None:
        vt = torch.empty(B, H, d, Np, dtype=torch.uint8, device=v.device)
        vs = torch.empty(B, H, d, dtype=torch.float32, device=v.device)
        vm = torch.empty(B, H, d, dtype=torch.float32, device=v.device) if smooth else None
    else:
        vt, vs = out[0], out[1]
        vm = out[2] if smooth else None
    st = lib().sage2_quant_v_ex(_ptr(v), _DT[v.dtype], B, H, N, d, _ptr(vt), _ptr(vs), _ptr(vm),
                                _stream(v))
    _check("sage2_quant_v_ex", st)
    return (vt, vs, vm) if smooth else (vt, vs)


def sage2_attn_fwd_quantized(pay: dict, v_fp8_t: torch.Tensor, v_scale: torch.Tensor, N: int,
                             causal: bool, sm_scale: float, out_dtype=torch.float32,
                             out: torch.Tensor | None = None,
                             v_mean: torch.Tensor | None = None) -> torch.Tensor:
    """The attention kernel alone, over payloads from sage2_smooth_quant_qk /
    sage2_quant_v (or any tensors in those layouts).  The payload format (INT4
    codes, packed INT4 or INT8) follows the q_i4 dtype and row width; v_mean
    is the token mean of a smoothed V."""
    B, H, Np = pay["q_i4"].shape[:3]
    d = pay["q_mean"].shape[-1]
    if out is None:
        out = torch.empty(B, H, N, d, dtype=out_dtype, device=pay["q_i4"].device)
    st = lib().sage2_attn_fwd_quantized_ex(
        _ptr(pay["q_i4"]), _ptr(pay["q_scale"]), _ptr(pay["k_i4"]), _ptr(pay["k_scale"]),
        _ptr(pay["qk_corr"]), _ptr(v_fp8_t), _ptr(v_scale), _ptr(v_mean), _ptr(out),
        _DT[out.dtype], B, H, N, d, int(bool(causal)), float(sm_scale),
        _format_of(pay), _stream(out))
    _check("sage2_attn_fwd_quantized_ex", st)
    return out


def sage2_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                   sm_scale: float | None = None, out_dtype=None,
                   out: torch.Tensor | None = None, qk_bits: int = 4,
                   smooth_v: bool = False, packed: bool = False) -> torch.Tensor:
    """Full forward pass (quantization + correction + attention) on q's stream.
    qk_bits 4 is the method (INT4 Q/K); 8 is the INT8 variant.  smooth_v turns
    on V smoothing; packed stores the INT4 payloads two per byte."""
    fmt = _fmt(qk_bits, packed)
    B, H, N, d = _dims(q)
    for t in (k, v):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k and v must have the same shape and dtype")
        _dims(t)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(B, H, N, d, dtype=out_dtype or q.dtype, device=q.device)
    st = lib().sage2_attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, _DT[q.dtype],
                                 _DT[out.dtype], int(bool(causal)), float(sm_scale),
                                 fmt, int(bool(smooth_v)), _stream(q))
    _check("sage2_attn_fwd_ex", st)
    return out


attn = sage2_attn_fwd


def sage2_attn_fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens,
                          causal: bool = False, sm_scale: float | None = None, out_dtype=None,
                          out: torch.Tensor | None = None, qk_bits: int = 4,
                          smooth_v: bool = False, packed: bool = False) -> torch.Tensor:
    """Packed variable-length sequences: q, k, v head-major [H, T, d] CUDA
    tensors, cu_seqlens the S+1 token offsets (host ints).  Each sequence is
    attended within itself; returns o [H, T, d].  packed stores the INT4
    payloads two per byte."""
    fmt = _fmt(qk_bits, packed)
    for t in (q, k, v):
        if t.dim() != 3 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous CUDA tensors [H, T, d]")
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k and v must have the same shape and dtype")
    H, T, d = q.shape
    cu = [int(c) for c in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    arr = (ctypes.c_int * len(cu))(*cu)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(H, T, d, dtype=out_dtype or q.dtype, device=q.device)
    st = lib().sage2_attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), arr, len(cu) - 1, H, T,
                                     d, _DT[q.dtype], _DT[out.dtype], int(bool(causal)),
                                     float(sm_scale), fmt, int(bool(smooth_v)),
                                     _stream(q))
    _check("sage2_attn_fwd_varlen", st)
    return out


def sage2_attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                           sm_scale: float | None = None, out_dtype=None,
                           out: torch.Tensor | None = None) -> torch.Tensor:
    """sage2_attn_fwd without any device allocation by the library: the scratch
    is the library's fixed 64 MiB device array (see include/sage2.h)."""
    B, H, N, d = _dims(q)
    for t in (k, v):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k and v must have the same shape and dtype")
        _dims(t)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(B, H, N, d, dtype=out_dtype or q.dtype, device=q.device)
    st = lib().sage2_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d,
                                      _DT[q.dtype], _DT[out.dtype], int(bool(causal)),
                                      float(sm_scale), _stream(q))
    _check("sage2_attn_fwd_noalloc", st)
    return out


def sage2_debug_qk_s32(q_i4: torch.Tensor, k_i4: torch.Tensor, N: int) -> torch.Tensor:
    """Raw int32 tiles of q_i4 . k_i4^T through the attention kernel's tensor
    path: the FP8 path for uint8 e4m3 codes of INT4 values, the 8-bit integer
    path for int8 values (the INT8 variant)."""
    B, H, Np, d = q_i4.shape
    if k_i4.dtype != q_i4.dtype:
        raise ValueError("q_i4 and k_i4 must have the same payload format")
    s = torch.empty(B, H, Np, Np, dtype=torch.int32, device=q_i4.device)
    st = lib().sage2_debug_qk_s32_ex(_ptr(q_i4), _ptr(k_i4), B, H, N, d,
                                     _QKF[_qk_bits_of(q_i4)], _ptr(s), _stream(q_i4))
    _check("sage2_debug_qk_s32_ex", st)
    return s


def sage2_debug_wait_timeout(device=None) -> None:
    """Failure-detection test entry: a kernel whose bounded wait runs out
    (see include/sage2.h).  sage2_check_device_error() then reports 6."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    _check("sage2_debug_wait_timeout", lib().sage2_debug_wait_timeout(st))


def sage2_attn_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                        causal: bool = False, sm_scale: float | None = None, qk_bits: int = 4,
                        smooth_v: bool = False, device=None, packed: bool = False) -> torch.Tensor:
    """The forward pass over HOST tensors [B,H,N,d] (pinned for overlap): chunks of
    heads are copied in, run and copied back on library streams joined into the
    current stream of `device`; `out` (host) is complete once that stream is."""
    fmt = _fmt(qk_bits, packed)
    for t in (q, k, v, out):
        if t.dim() != 4 or t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v, out must be contiguous host tensors [B, H, N, d]")
    for t in (k, v):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k and v must have the same shape and dtype")
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    B, H, N, d = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    status = lib().sage2_attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d,
                                       _DT[q.dtype], _DT[out.dtype], int(bool(causal)),
                                       float(sm_scale), fmt, int(bool(smooth_v)), st)
    _check("sage2_attn_fwd_host", status)
    return out
