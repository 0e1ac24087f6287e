"""Python binding of the C ABI in ``include/attn.h`` (ctypes).

Argument marshalling only: every step of the attention forward runs in the
CUDA kernels of ``libattn.so``.  PyTorch supplies device memory and streams.
There is no fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn.so")
_lock = threading.Lock()
_lib = None

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_MISALIGNED = 3
ATTN_ERR_LAUNCH = 4
ATTN_ERR_DEVICE_TIMEOUT = 5
ATTN_ERR_CUDA = 6
ATTN_ERR_RANGE = 7

ATTN_DIRECT_P_AFFINE = 0
ATTN_DIRECT_P_EXP2 = 1
CLASSIFIERS = {"affine": ATTN_DIRECT_P_AFFINE, "exp2": ATTN_DIRECT_P_EXP2}
ATTN_FP4_MMA_AUTO = 0
ATTN_FP4_MMA_F16 = 1
ATTN_FP4_MMA_BLOCK_SCALED = 2
FP4_MMA = {"auto": ATTN_FP4_MMA_AUTO, "f16": ATTN_FP4_MMA_F16,
           "block_scaled": ATTN_FP4_MMA_BLOCK_SCALED}

EXPORTED = ("attn_fwd", "attn_fwd_ex", "attn_fwd_fp8", "attn_fwd_default_options",
            "attn_fp4_default_options", "attn_fwd_fp4_workspace_size", "attn_fwd_fp4", "attn_bwd",
            "attn_bwd_ex", "attn_bwd_workspace_size", "attn_bwd_noalloc", "attn_get_device_status",
            "attn_status_string", "attn_last_error_detail", "attn_abi_version")


class AttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class FwdOptions(ctypes.Structure):
    """Mirror of attn_fwd_options_t."""
    _fields_ = [("rescale_threshold", ctypes.c_float), ("exp2_mode", ctypes.c_int),
                ("wait_timeout_us", ctypes.c_int), ("debug_withhold_kv", ctypes.c_int),
                ("softcap", ctypes.c_float), ("reserved0", ctypes.c_int),
                ("alibi_slopes", ctypes.c_void_p), ("reserved", ctypes.c_int * 4)]


class BwdOptions(ctypes.Structure):
    """Mirror of attn_bwd_options_t."""
    _fields_ = [("softcap", ctypes.c_float), ("reserved0", ctypes.c_int),
                ("alibi_slopes", ctypes.c_void_p), ("reserved", ctypes.c_int * 4)]


class Fp4Options(ctypes.Structure):
    """Mirror of attn_fp4_options_t."""
    _fields_ = [("rescale_threshold", ctypes.c_float), ("classifier", ctypes.c_int),
                ("wait_timeout_us", ctypes.c_int), ("mma", ctypes.c_int),
                ("reserved", ctypes.c_int * 4)]


_FWD_ARGS = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 + [ctypes.c_float] + \
            [ctypes.c_int] * 3 + [ctypes.c_void_p, ctypes.c_int]


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libattn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is not built; run `python -m tiled_attention_blackwell_b200.build`")
            L = ctypes.CDLL(_LIB_PATH)
            L.attn_fwd.restype = ctypes.c_int
            L.attn_fwd.argtypes = _FWD_ARGS + [ctypes.c_void_p]
            L.attn_fwd_ex.restype = ctypes.c_int
            L.attn_fwd_ex.argtypes = _FWD_ARGS + [ctypes.POINTER(FwdOptions), ctypes.c_void_p]
            L.attn_fwd_fp8.restype = ctypes.c_int
            L.attn_fwd_fp8.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_float] * 3 + \
                [ctypes.c_void_p] * 2 + [ctypes.c_int] * 6 + [ctypes.c_float] + \
                [ctypes.c_int] * 3 + [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(FwdOptions),
                                      ctypes.c_void_p]
            L.attn_fp4_default_options.restype = None
            L.attn_fp4_default_options.argtypes = [ctypes.POINTER(Fp4Options)]
            L.attn_fwd_fp4_workspace_size.restype = ctypes.c_size_t
            L.attn_fwd_fp4_workspace_size.argtypes = [ctypes.c_int] * 6
            L.attn_fwd_fp4.restype = ctypes.c_int
            L.attn_fwd_fp4.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float] * 3 + \
                [ctypes.c_void_p] * 2 + [ctypes.c_int] * 6 + [ctypes.c_float] + \
                [ctypes.c_int] * 3 + [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                      ctypes.c_size_t, ctypes.POINTER(Fp4Options),
                                      ctypes.c_void_p]
            L.attn_fwd_default_options.restype = None
            L.attn_fwd_default_options.argtypes = [ctypes.POINTER(FwdOptions)]
            L.attn_get_device_status.restype = ctypes.c_int
            L.attn_get_device_status.argtypes = [ctypes.c_void_p]
            L.attn_status_string.restype = ctypes.c_char_p
            L.attn_status_string.argtypes = [ctypes.c_int]
            L.attn_last_error_detail.restype = ctypes.c_char_p
            L.attn_last_error_detail.argtypes = []
            L.attn_abi_version.restype = ctypes.c_int
            L.attn_bwd_workspace_size.restype = ctypes.c_size_t
            L.attn_bwd_workspace_size.argtypes = [ctypes.c_int] * 6
            L.attn_bwd.restype = ctypes.c_int
            L.attn_bwd.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 6 + \
                [ctypes.c_float] + [ctypes.c_int] * 3 + [ctypes.c_void_p, ctypes.c_int,
                                                         ctypes.c_void_p, ctypes.c_size_t,
                                                         ctypes.c_void_p]
            L.attn_bwd_ex.restype = ctypes.c_int
            L.attn_bwd_ex.argtypes = L.attn_bwd.argtypes[:-1] + [ctypes.POINTER(BwdOptions),
                                                                 ctypes.c_void_p]
            L.attn_bwd_noalloc.restype = ctypes.c_int
            L.attn_bwd_noalloc.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 6 + \
                [ctypes.c_float] + [ctypes.c_int] * 3 + [ctypes.c_void_p, ctypes.c_int,
                                                         ctypes.c_void_p]
            _lib = L
    return _lib


def _check(status: int, what: str):
    if status != ATTN_OK:
        L = lib()
        raise AttnError(status, f"{what}: {L.attn_status_string(status).decode()}"
                                f" ({L.attn_last_error_detail().decode()})")


def default_options(**overrides) -> FwdOptions:
    opts = FwdOptions()
    lib().attn_fwd_default_options(ctypes.byref(opts))
    for k, v in overrides.items():
        setattr(opts, k, v)
    return opts


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _slopes(alibi_slopes, Hq, device, stream):
    """ALiBi slopes as a contiguous CUDA fp32 [Hq] tensor that stays valid
    until the kernel that reads it has run on `stream`."""
    if alibi_slopes is None:
        return None
    if not torch.is_tensor(alibi_slopes) or not alibi_slopes.is_cuda:
        alibi_slopes = torch.as_tensor(alibi_slopes, dtype=torch.float32).to(device)
        if stream is not None:
            alibi_slopes.record_stream(stream)
    if alibi_slopes.dtype != torch.float32 or not alibi_slopes.is_contiguous() \
            or alibi_slopes.numel() != Hq:
        raise TypeError("alibi_slopes must be a contiguous fp32 tensor of Hq entries")
    return alibi_slopes


def attn_fwd(q, k, v, o, lse, *, scale, causal=False, window=None, doc_offsets=None,
             options=None, stream=None, softcap=None, alibi_slopes=None):
    """Enqueue the forward on `stream` (default: torch's current stream).

    q, o: bf16 CUDA [B,Sq,Hq,D]; k, v: bf16 CUDA [B,Sk,Hkv,D]; lse: fp32 CUDA
    [B,Hq,Sq]; doc_offsets: int32 CUDA [num_docs+1] or None.  All contiguous.
    softcap (> 0) and alibi_slopes (fp32 [Hq]) select the score modifiers;
    they override the same fields of `options`.
    """
    for name, t, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16),
                        ("v", v, torch.bfloat16), ("o", o, torch.bfloat16),
                        ("lse", lse, torch.float32)):
        if t.dtype != dt or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA {dt} tensor")
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    if doc_offsets is not None:
        if doc_offsets.dtype != torch.int32 or not doc_offsets.is_cuda:
            raise TypeError("doc_offsets must be a CUDA int32 tensor")
        docs_ptr, nd = _ptr(doc_offsets), doc_offsets.numel() - 1
    else:
        docs_ptr, nd = None, 0
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Sk, D,
            float(scale), int(bool(causal)), wl, wr, docs_ptr, nd]
    L = lib()
    slopes = _slopes(alibi_slopes, Hq, q.device, stream)
    if softcap is not None or slopes is not None:
        if options is None:
            options = default_options()
        else:
            options = FwdOptions.from_buffer_copy(options)
        if softcap is not None:
            options.softcap = float(softcap)
        if slopes is not None:
            options.alibi_slopes = slopes.data_ptr()
    if options is None:
        st = L.attn_fwd(*args, _stream_handle(stream))
    else:
        st = L.attn_fwd_ex(*args, ctypes.byref(options), _stream_handle(stream))
    _check(st, "attn_fwd")


def attention(q, k, v, *, scale=None, causal=False, window=None, doc_offsets=None,
              options=None, stream=None, softcap=None, alibi_slopes=None):
    """Allocate O and LSE with torch and run the forward.  Returns (O, LSE)."""
    B, Sq, Hq, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if doc_offsets is not None and not torch.is_tensor(doc_offsets):
        doc_offsets = torch.as_tensor(doc_offsets, dtype=torch.int32)
    if doc_offsets is not None and not doc_offsets.is_cuda:
        doc_offsets = doc_offsets.to(q.device)
    attn_fwd(q, k, v, o, lse, scale=scale, causal=causal, window=window,
             doc_offsets=doc_offsets, options=options, stream=stream, softcap=softcap,
             alibi_slopes=alibi_slopes)
    return o, lse


def attn_fwd_fp8(q, k, v, o, lse, *, q_descale, k_descale, v_descale, scale, causal=False,
                 window=None, doc_offsets=None, options=None, stream=None):
    """Enqueue the fp8 forward: q, k, v contiguous CUDA tensors of e4m3 codes
    (torch.float8_e4m3fn or uint8) standing for descale * code; o bf16, lse
    fp32 as in attn_fwd."""
    fp8_types = (torch.float8_e4m3fn, torch.uint8)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype not in fp8_types or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA float8_e4m3fn tensor")
    for name, t, dt in (("o", o, torch.bfloat16), ("lse", lse, torch.float32)):
        if t.dtype != dt or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA {dt} tensor")
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    if doc_offsets is not None:
        if doc_offsets.dtype != torch.int32 or not doc_offsets.is_cuda:
            raise TypeError("doc_offsets must be a CUDA int32 tensor")
        docs_ptr, nd = _ptr(doc_offsets), doc_offsets.numel() - 1
    else:
        docs_ptr, nd = None, 0
    st = lib().attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), float(q_descale), float(k_descale),
                            float(v_descale), _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Sk, D,
                            float(scale), int(bool(causal)), wl, wr, docs_ptr, nd,
                            None if options is None else ctypes.byref(options),
                            _stream_handle(stream))
    _check(st, "attn_fwd_fp8")


def attention_fp8(q, k, v, *, q_descale, k_descale, v_descale, scale=None, causal=False,
                  window=None, doc_offsets=None, options=None, stream=None):
    """Allocate O (bf16) and LSE with torch and run the fp8 forward."""
    B, Sq, Hq, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = torch.empty((B, Sq, Hq, D), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if doc_offsets is not None and not torch.is_tensor(doc_offsets):
        doc_offsets = torch.as_tensor(doc_offsets, dtype=torch.int32)
    if doc_offsets is not None and not doc_offsets.is_cuda:
        doc_offsets = doc_offsets.to(q.device)
    attn_fwd_fp8(q, k, v, o, lse, q_descale=q_descale, k_descale=k_descale,
                 v_descale=v_descale, scale=scale, causal=causal, window=window,
                 doc_offsets=doc_offsets, options=options, stream=stream)
    return o, lse


def fp4_options(**overrides) -> Fp4Options:
    opts = Fp4Options()
    lib().attn_fp4_default_options(ctypes.byref(opts))
    for k, v in overrides.items():
        setattr(opts, k, v)
    return opts


def fp4_workspace_size(B, Hq, Hkv, Sq, Sk, D) -> int:
    """Bytes of device workspace attn_fwd_fp4 needs."""
    return int(lib().attn_fwd_fp4_workspace_size(B, Hq, Hkv, Sq, Sk, D))


def attn_fwd_fp4(q_codes, q_scales, q_global, k_codes, k_scales, k_global, v_codes, v_scales,
                 v_global, o, lse, workspace, *, scale, causal=False, window=None,
                 doc_offsets=None, classifier="affine", mma=None, options=None, stream=None):
    """Enqueue the FP4 Direct-P forward.

    q_codes uint8 CUDA [B,Sq,Hq,D/2], q_scales uint8 [B,Sq,Hq,D/16] (e4m3
    bytes), likewise k_*; v_codes [B,Sk,Hkv,D/2], v_scales uint8
    [B,ceil(Sk/32),Hkv,D] (UE8M0 bytes); o bf16 [B,Sq,Hq,D]; lse fp32
    [B,Hq,Sq]; workspace uint8 CUDA of fp4_workspace_size() bytes.  All
    contiguous.  classifier: "affine" or "exp2" (overrides `options`); mma:
    None (keep `options`), "auto", "f16" or "block_scaled" (which tensor-core
    products run, see attn_fp4_options_t).
    """
    B, Sq, Hq, Dh = q_codes.shape
    _, Sk, Hkv, _ = k_codes.shape
    D = 2 * Dh
    shapes = (("q_codes", q_codes, (B, Sq, Hq, Dh)), ("q_scales", q_scales, (B, Sq, Hq, D // 16)),
              ("k_codes", k_codes, (B, Sk, Hkv, Dh)), ("k_scales", k_scales, (B, Sk, Hkv, D // 16)),
              ("v_codes", v_codes, (B, Sk, Hkv, Dh)),
              ("v_scales", v_scales, (B, (Sk + 31) // 32, Hkv, D)))
    for name, t, shape in shapes:
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or not t.is_cuda \
                or not t.is_contiguous() or tuple(t.shape) != shape:
            raise TypeError(f"{name} must be a contiguous CUDA uint8 tensor of shape {shape}")
    for name, t, dt in (("o", o, torch.bfloat16), ("lse", lse, torch.float32),
                        ("workspace", workspace, torch.uint8)):
        if t.dtype != dt or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA {dt} tensor")
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    if doc_offsets is not None:
        if doc_offsets.dtype != torch.int32 or not doc_offsets.is_cuda:
            raise TypeError("doc_offsets must be a CUDA int32 tensor")
        docs_ptr, nd = _ptr(doc_offsets), doc_offsets.numel() - 1
    else:
        docs_ptr, nd = None, 0
    options = fp4_options() if options is None else Fp4Options.from_buffer_copy(options)
    options.classifier = CLASSIFIERS[classifier]
    if mma is not None:
        options.mma = FP4_MMA[mma]
    st = lib().attn_fwd_fp4(_ptr(q_codes), _ptr(q_scales), float(q_global), _ptr(k_codes),
                            _ptr(k_scales), float(k_global), _ptr(v_codes), _ptr(v_scales),
                            float(v_global), _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Sk, D,
                            float(scale), int(bool(causal)), wl, wr, docs_ptr, nd,
                            _ptr(workspace), workspace.numel(), ctypes.byref(options),
                            _stream_handle(stream))
    _check(st, "attn_fwd_fp4")


def attention_fp4(q_codes, q_scales, q_global, k_codes, k_scales, k_global, v_codes, v_scales,
                  v_global, *, scale=None, causal=False, window=None, doc_offsets=None,
                  classifier="affine", mma=None, options=None, stream=None, workspace=None):
    """Allocate O, LSE (and the workspace unless given) with torch and run the
    FP4 Direct-P forward.  Returns (O, LSE)."""
    B, Sq, Hq, Dh = q_codes.shape
    _, Sk, Hkv, _ = k_codes.shape
    D = 2 * Dh
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dev = q_codes.device
    o = torch.empty((B, Sq, Hq, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(fp4_workspace_size(B, Hq, Hkv, Sq, Sk, D), dtype=torch.uint8,
                                device=dev)
    if doc_offsets is not None and not torch.is_tensor(doc_offsets):
        doc_offsets = torch.as_tensor(doc_offsets, dtype=torch.int32)
    if doc_offsets is not None and not doc_offsets.is_cuda:
        doc_offsets = doc_offsets.to(dev)
    attn_fwd_fp4(q_codes, q_scales, q_global, k_codes, k_scales, k_global, v_codes, v_scales,
                 v_global, o, lse, workspace, scale=scale, causal=causal, window=window,
                 doc_offsets=doc_offsets, classifier=classifier, mma=mma, options=options,
                 stream=stream)
    return o, lse


def _check_bwd_tensors(q, k, v, o, lse, dout, dq, dk, dv):
    """Dtype, device and layout of every tensor the backward kernels touch:
    a wrong dtype would make a kernel read or write past a buffer's end."""
    for name, t, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16),
                        ("v", v, torch.bfloat16), ("o", o, torch.bfloat16),
                        ("lse", lse, torch.float32), ("dout", dout, torch.bfloat16),
                        ("dq", dq, torch.float32), ("dk", dk, torch.bfloat16),
                        ("dv", dv, torch.bfloat16)):
        if not torch.is_tensor(t) or t.dtype != dt or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA {dt} tensor")
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    for name, t, shape in (("k", k, (B, Sk, Hkv, D)), ("v", v, (B, Sk, Hkv, D)),
                           ("o", o, (B, Sq, Hq, D)), ("dout", dout, (B, Sq, Hq, D)),
                           ("dq", dq, (B, Sq, Hq, D)), ("dk", dk, (B, Sk, Hkv, D)),
                           ("dv", dv, (B, Sk, Hkv, D)), ("lse", lse, (B, Hq, Sq))):
        if tuple(t.shape) != shape:
            raise TypeError(f"{name} must have shape {shape}, got {tuple(t.shape)}")


def _docs_arg(doc_offsets):
    """(pointer, num_docs) of a CUDA int32 doc_offsets tensor, or (None, 0).
    Anything else raises: the kernels read the offsets on the device."""
    if doc_offsets is None:
        return None, 0
    if not torch.is_tensor(doc_offsets) or doc_offsets.dtype != torch.int32 \
            or not doc_offsets.is_cuda or not doc_offsets.is_contiguous():
        raise TypeError("doc_offsets must be a contiguous CUDA int32 tensor")
    return _ptr(doc_offsets), doc_offsets.numel() - 1


def bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D) -> int:
    """Bytes of device workspace attn_bwd needs."""
    return int(lib().attn_bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D))


def attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, *, scale, causal=False, window=None,
             doc_offsets=None, stream=None, softcap=None, alibi_slopes=None):
    """Enqueue the backward on `stream`.  dq fp32 [B,Sq,Hq,D]; dk, dv bf16
    [B,Sk,Hkv,D]; workspace a CUDA uint8 tensor of at least
    bwd_workspace_size() bytes.  softcap / alibi_slopes must match the
    forward that produced o and lse."""
    _check_bwd_tensors(q, k, v, o, lse, dout, dq, dk, dv)
    if not torch.is_tensor(workspace) or not workspace.is_cuda or not workspace.is_contiguous():
        raise TypeError("workspace must be a contiguous CUDA tensor")
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    docs_ptr, nd = _docs_arg(doc_offsets)
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
            _ptr(dv), B, Hq, Hkv, Sq, Sk, D, float(scale), int(bool(causal)), wl, wr,
            docs_ptr, nd, _ptr(workspace), workspace.numel() * workspace.element_size()]
    slopes = _slopes(alibi_slopes, Hq, q.device, stream)
    if softcap is None and slopes is None:
        st = lib().attn_bwd(*args, _stream_handle(stream))
    else:
        opts = BwdOptions()
        opts.softcap = float(softcap or 0.0)
        opts.alibi_slopes = None if slopes is None else slopes.data_ptr()
        st = lib().attn_bwd_ex(*args, ctypes.byref(opts), _stream_handle(stream))
    _check(st, "attn_bwd")


def attention_backward(q, k, v, o, lse, dout, *, scale=None, causal=False, window=None,
                       doc_offsets=None, stream=None, softcap=None, alibi_slopes=None):
    """Allocate dQ (fp32), dK, dV (bf16) and the workspace with torch and run
    the backward.  Returns (dQ, dK, dV)."""
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    ws = torch.empty(bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D), dtype=torch.uint8,
                     device=q.device)
    if doc_offsets is not None and not torch.is_tensor(doc_offsets):
        doc_offsets = torch.as_tensor(doc_offsets, dtype=torch.int32)
    if doc_offsets is not None and not doc_offsets.is_cuda:
        doc_offsets = doc_offsets.to(q.device)
    attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, ws, scale=scale, causal=causal, window=window,
             doc_offsets=doc_offsets, stream=stream, softcap=softcap, alibi_slopes=alibi_slopes)
    return dq, dk, dv


def attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, *, scale, causal=False, window=None,
                     doc_offsets=None, stream=None):
    """attn_bwd for callers that cannot allocate device memory: the library
    uses its own fixed scratch (B*Hq*Sq <= 1048576 rows) instead of a
    workspace.  Calls that may run on the GPU at the same time must be
    ordered by the caller (they share that scratch).  Tensor checks are those
    of attn_bwd; doc_offsets must already be a CUDA int32 tensor (this entry
    point never copies or allocates)."""
    _check_bwd_tensors(q, k, v, o, lse, dout, dq, dk, dv)
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    docs_ptr, nd = _docs_arg(doc_offsets)
    st = lib().attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, Sq, Sk, D,
                                float(scale), int(bool(causal)), wl, wr, docs_ptr, nd,
                                _stream_handle(stream))
    _check(st, "attn_bwd_noalloc")


def device_status(stream=None) -> int:
    """Synchronise `stream`, then read and clear the device status word."""
    return lib().attn_get_device_status(_stream_handle(stream))


def check_device_status(stream=None):
    _check(device_status(stream), "device status")
