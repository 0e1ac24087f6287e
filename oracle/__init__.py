"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA path and the CUDA path
never imports it.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP); this module
only compiles it with gcc, loads it with ctypes and marshals arrays.  See the
header of ``attn_oracle.c`` for what is computed, the passages it follows and
the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so (gcc, -fopenmp)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            dims = [ctypes.c_int] * 6 + [ctypes.c_double] + [ctypes.c_int] * 3 + \
                   [ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_void_p]
            for name in ("oracle_attn_fwd_bf16", "oracle_attn_fwd_f64"):
                fn = getattr(lib, name)
                fn.restype = ctypes.c_int
                fn.argtypes = [ctypes.c_void_p] * 5 + dims + [ctypes.c_void_p, ctypes.c_int64]
            for name in ("oracle_attn_bwd_bf16", "oracle_attn_bwd_f64"):
                fn = getattr(lib, name)
                fn.restype = ctypes.c_int
                fn.argtypes = [ctypes.c_void_p] * 9 + dims
            lib.oracle_attn_fwd_e4m3.restype = ctypes.c_int
            lib.oracle_attn_fwd_e4m3.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_double] * 3 + \
                [ctypes.c_void_p] * 2 + dims[:-2] + [ctypes.c_void_p, ctypes.c_int64]
            lib.oracle_attn_fwd_fp4.restype = ctypes.c_int
            lib.oracle_attn_fwd_fp4.argtypes = \
                ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_double] * 3 + [ctypes.c_void_p] * 2
                 + dims[:-2] + [ctypes.c_int, ctypes.c_void_p, ctypes.c_int64])
            lib.oracle_direct_p_row.restype = ctypes.c_int
            lib.oracle_direct_p_row.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                                ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_void_p, ctypes.c_void_p]
            for name in ("oracle_e2m1_to_double", "oracle_ue8m0_to_double"):
                getattr(lib, name).restype = ctypes.c_double
                getattr(lib, name).argtypes = [ctypes.c_int]
            lib.oracle_e2m1_round.restype = ctypes.c_double
            lib.oracle_e2m1_round.argtypes = [ctypes.c_double]
            lib.oracle_e4m3_to_double.restype = ctypes.c_double
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_int]
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_num_threads())


def _as_input(x):
    """Return (contiguous array, is_bf16).  bf16 torch tensors are passed as
    their raw 16-bit patterns (converted exactly to double inside C); float64
    numpy arrays / tensors are passed as doubles."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), True
            return x.to(torch.float64).numpy(), False
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, True
    return np.ascontiguousarray(x, dtype=np.float64), False


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _mask_args(causal, window, doc_offsets):
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    if doc_offsets is None:
        return int(bool(causal)), wl, wr, None, 0
    offs = np.ascontiguousarray(np.asarray(doc_offsets, dtype=np.int32))
    return int(bool(causal)), wl, wr, offs, int(offs.size - 1)


def _mods(softcap, alibi_slopes, Hq):
    if alibi_slopes is None:
        return float(softcap or 0.0), None
    sl = np.ascontiguousarray(np.asarray(alibi_slopes, dtype=np.float64).reshape(-1))
    if sl.size != Hq:
        raise ValueError("alibi_slopes must have one entry per query head")
    return float(softcap or 0.0), sl


def _shapes(q, k):
    B, Sq, Hq, D = q.shape
    Bk, Sk, Hkv, Dk = k.shape
    if Bk != B or Dk != D:
        raise ValueError("q/k shape mismatch")
    return B, Hq, Hkv, Sq, Sk, D


def attn_fwd(q, k, v, *, scale, causal=False, window=None, doc_offsets=None,
             rows=None, softcap=0.0, alibi_slopes=None):
    """Exact attention forward in fp64.

    q: [B,Sq,Hq,D], k/v: [B,Sk,Hkv,D] (bf16 torch tensors or float64 arrays).
    rows: optional int array [n,3] of (b, hq, i); then only those rows are
    computed and O is [n, D], LSE is [n].  Otherwise O is [B,Sq,Hq,D] and
    LSE is [B,Hq,Sq].  Returns float64 numpy arrays (O, LSE).
    """
    lib = _load()
    (qa, qb), (ka, kb), (va, vb) = _as_input(q), _as_input(k), _as_input(v)
    if not (qb == kb == vb):
        raise TypeError("q, k, v must all be bf16 or all float64")
    B, Hq, Hkv, Sq, Sk, D = _shapes(qa, ka)
    causal_i, wl, wr, offs, nd = _mask_args(causal, window, doc_offsets)
    cap, slopes = _mods(softcap, alibi_slopes, Hq)
    if rows is None:
        o = np.zeros((B, Sq, Hq, D), dtype=np.float64)
        lse = np.zeros((B, Hq, Sq), dtype=np.float64)
        rows_a, n = None, 0
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n = rows_a.shape[0]
        o = np.zeros((n, D), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
    fn = lib.oracle_attn_fwd_bf16 if qb else lib.oracle_attn_fwd_f64
    rc = fn(_ptr(qa), _ptr(ka), _ptr(va), _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Sk, D,
            float(scale), causal_i, wl, wr, _ptr(offs), nd, cap, _ptr(slopes), _ptr(rows_a), n)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd failed with code {rc}")
    return o, lse


def e4m3_to_float(code: int) -> float:
    """The value of one fp8 e4m3 code (0..255), decoded by the oracle."""
    return float(_load().oracle_e4m3_to_double(int(code)))


def _as_codes(x):
    """fp8 e4m3 codes as a contiguous uint8 array (from a torch float8_e4m3fn
    or uint8 tensor, or a numpy uint8 array)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype != torch.uint8:
                x = x.view(torch.uint8)
            return x.numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint8:
        raise TypeError("fp8 inputs must be e4m3 codes (uint8)")
    return x


def attn_fwd_fp8(q, k, v, *, q_descale, k_descale, v_descale, scale, causal=False,
                 window=None, doc_offsets=None, rows=None):
    """Exact attention in fp64 of fp8 e4m3 inputs: Q = q_descale * decode(q),
    likewise K and V.  Shapes and return values as attn_fwd."""
    lib = _load()
    qa, ka, va = _as_codes(q), _as_codes(k), _as_codes(v)
    B, Hq, Hkv, Sq, Sk, D = _shapes(qa, ka)
    causal_i, wl, wr, offs, nd = _mask_args(causal, window, doc_offsets)
    if rows is None:
        o = np.zeros((B, Sq, Hq, D), dtype=np.float64)
        lse = np.zeros((B, Hq, Sq), dtype=np.float64)
        rows_a, n = None, 0
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n = rows_a.shape[0]
        o = np.zeros((n, D), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
    rc = lib.oracle_attn_fwd_e4m3(_ptr(qa), _ptr(ka), _ptr(va), float(q_descale),
                                  float(k_descale), float(v_descale), _ptr(o), _ptr(lse),
                                  B, Hq, Hkv, Sq, Sk, D, float(scale), causal_i, wl, wr,
                                  _ptr(offs), nd, _ptr(rows_a), n)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_e4m3 failed with code {rc}")
    return o, lse


_CLASSIFIERS = {"affine": 1, "exp2": 2}


def e2m1_to_float(code: int) -> float:
    """The value of one 4-bit E2M1 code (0..15, bit 3 = sign)."""
    return float(_load().oracle_e2m1_to_double(int(code)))


def ue8m0_to_float(u: int) -> float:
    """The value of one UE8M0 scale byte: 2^(u - 127), NaN for 255."""
    return float(_load().oracle_ue8m0_to_double(int(u)))


def e2m1_round(x: float) -> float:
    """x >= 0 rounded to the nearest E2M1 magnitude (ties to the even code),
    saturating at 6."""
    return float(_load().oracle_e2m1_round(float(x)))


def direct_p_row(y, v, *, allow=None, classifier="affine"):
    """Direct-P output and LSE of one row from its log2 scores y [n] and
    value rows v [n, D] (allow: optional bool mask [n])."""
    lib = _load()
    y = np.ascontiguousarray(np.asarray(y, dtype=np.float64).reshape(-1))
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    n, D = v.shape
    if y.size != n:
        raise ValueError("y and v disagree on the number of keys")
    a = np.ones(n, dtype=np.uint8) if allow is None else \
        np.ascontiguousarray(np.asarray(allow, dtype=bool).astype(np.uint8))
    o = np.zeros(D)
    lse = np.zeros(1)
    rc = lib.oracle_direct_p_row(_ptr(y), _ptr(a), n, _ptr(v), D, _CLASSIFIERS[classifier],
                                 _ptr(o), _ptr(lse))
    if rc != 0:
        raise RuntimeError(f"oracle_direct_p_row failed with code {rc}")
    return o, float(lse[0])


def attn_fwd_fp4(q_codes, q_scales, q_global, k_codes, k_scales, k_global, v_codes,
                 v_scales, v_global, *, scale, causal=False, window=None, doc_offsets=None,
                 classifier="affine", rows=None):
    """Direct-P forward in fp64 of NVFP4 Q/K and MXFP4 V.

    q_codes [B,Sq,Hq,D/2], q_scales [B,Sq,Hq,D/16] (e4m3 bytes), likewise K;
    v_codes [B,Sk,Hkv,D/2], v_scales [B,ceil(Sk/32),Hkv,D] (UE8M0 bytes); all
    uint8.  classifier: "affine" or "exp2".  Shapes of the results as
    attn_fwd."""
    lib = _load()
    qc, qs, kc, ks, vc, vs = (_as_codes(t) for t in (q_codes, q_scales, k_codes, k_scales,
                                                     v_codes, v_scales))
    B, Sq, Hq, Dh = qc.shape
    Sk, Hkv = kc.shape[1], kc.shape[2]
    D = 2 * Dh
    if kc.shape != (B, Sk, Hkv, Dh) or vc.shape != kc.shape:
        raise ValueError("code tensors disagree in shape")
    if qs.shape != (B, Sq, Hq, D // 16) or ks.shape != (B, Sk, Hkv, D // 16):
        raise ValueError("NVFP4 scales must be [B, S, H, D/16]")
    if vs.shape != (B, (Sk + 31) // 32, Hkv, D):
        raise ValueError("MXFP4 scales of V must be [B, ceil(Sk/32), Hkv, D]")
    causal_i, wl, wr, offs, nd = _mask_args(causal, window, doc_offsets)
    if rows is None:
        o = np.zeros((B, Sq, Hq, D), dtype=np.float64)
        lse = np.zeros((B, Hq, Sq), dtype=np.float64)
        rows_a, n = None, 0
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n = rows_a.shape[0]
        o = np.zeros((n, D), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
    rc = lib.oracle_attn_fwd_fp4(_ptr(qc), _ptr(qs), float(q_global), _ptr(kc), _ptr(ks),
                                 float(k_global), _ptr(vc), _ptr(vs), float(v_global),
                                 _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Sk, D, float(scale),
                                 causal_i, wl, wr, _ptr(offs), nd, _CLASSIFIERS[classifier],
                                 _ptr(rows_a), n)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_fp4 failed with code {rc}")
    return o, lse


def attn_bwd(q, k, v, dout, *, scale, causal=False, window=None, doc_offsets=None,
             softcap=0.0, alibi_slopes=None):
    """Exact attention backward of L = sum(O * dO) in fp64.

    Returns (dQ, dK, dV, O, LSE) as float64 numpy arrays; dK/dV are summed
    over the query heads that share a key/value head.
    """
    lib = _load()
    ins = [_as_input(t) for t in (q, k, v, dout)]
    if len({b for _, b in ins}) != 1:
        raise TypeError("q, k, v, dout must all be bf16 or all float64")
    (qa, bf), (ka, _), (va, _), (da, _) = ins
    B, Hq, Hkv, Sq, Sk, D = _shapes(qa, ka)
    causal_i, wl, wr, offs, nd = _mask_args(causal, window, doc_offsets)
    cap, slopes = _mods(softcap, alibi_slopes, Hq)
    dq = np.zeros((B, Sq, Hq, D))
    dk = np.zeros((B, Sk, Hkv, D))
    dv = np.zeros((B, Sk, Hkv, D))
    o = np.zeros((B, Sq, Hq, D))
    lse = np.zeros((B, Hq, Sq))
    fn = lib.oracle_attn_bwd_bf16 if bf else lib.oracle_attn_bwd_f64
    rc = fn(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), _ptr(dq), _ptr(dk), _ptr(dv),
            _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Sk, D, float(scale), causal_i, wl, wr,
            _ptr(offs), nd, cap, _ptr(slopes))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd failed with code {rc}")
    return dq, dk, dv, o, lse
