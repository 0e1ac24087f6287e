"""Seeded synthetic inputs for the attention benchmarks and parity tests.

This module only draws random numbers and lays out shapes; it contains none
of the attention arithmetic.  It is the one piece shared by the CUDA-path
tests and the oracle tests, so both sides see bit-identical bf16 inputs.

Recipe (all on the CPU, deterministic):
  * a ``torch.Generator`` seeded with the config's seed draws fp32 normals in
    the order Q, K, V (then dO for the backward), each rounded to bf16 at the
    end;
  * the outlier config multiplies a random 1% of the K rows (each
    (b, token, kv-head) row chosen independently, drawn after V) by 8 in fp32
    before rounding, which forces running-max jumps;
  * document lengths are drawn with ``numpy.random.default_rng(seed)`` as
    integers uniform in [512, 4096] (inclusive) until they cover the
    sequence; the last document is clipped to what is left;
  * fp8 workloads draw the same fp32 tensors and quantise each one to e4m3
    with one per-tensor factor, descale = max|x| / 448 (torch's
    round-to-nearest conversion of x / descale);
  * fp4 workloads draw the same fp32 tensors and encode Q and K as NVFP4
    (E2M1 codes, one e4m3 scale per 16 elements of a row, one fp32 factor
    per tensor) and V as MXFP4 (E2M1 codes, one power-of-two scale per 32
    keys of each (batch, head, d) column, the OCP rule 2^(floor(log2 amax)
    - 2)).  Codes are the nearest E2M1 magnitude (ties to the even code,
    saturating at 6).  With ``pow2_scales`` the NVFP4 block scales are the
    power of two 2^ceil(log2(amax / 6)) and K's per-tensor factor is chosen
    so that scale * q_global * k_global * log2(e) is a power of two: every
    score is then an exact dyadic number, so the fp32 dot products of the
    kernel and the fp64 ones of the oracle agree bit for bit and the
    quantised decisions on them can be compared exactly.  Otherwise the
    NVFP4 scales are e4m3(amax / (6 g)) with g = max|x| / (6 * 448).
No public dataset or benchmark suite stands behind these shapes; the pages
measure on none that could be used here, so synthetic inputs of the named
shapes stand in.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    S: int
    D: int
    causal: bool
    seed: int
    qk_std: float = 1.0
    k_outlier_frac: float = 0.0
    k_outlier_mult: float = 8.0
    doc_lengths: Optional[tuple] = None  # (lo, hi) inclusive, or None
    backward: bool = False
    window: tuple = (-1, -1)
    dtype: str = "bf16"  # "bf16", "fp8" (e4m3 Q, K, V) or "fp4" (NVFP4 Q/K, MXFP4 V)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def describe(self) -> str:
        mask = "causal" if self.causal else "non-causal"
        if self.doc_lengths:
            mask = f"document-causal, docs U[{self.doc_lengths[0]},{self.doc_lengths[1]}]"
        return (f"B={self.B} Hq={self.Hq} Hkv={self.Hkv} Sq=Sk={self.S} D={self.D} "
                f"{mask} {self.dtype}" + (" backward" if self.backward else " forward"))


# The five workloads: tiny oracle case, outlier-K non-causal, the causal
# S=8192 headline, GQA with document masking, and the causal backward.
WORKLOADS = {
    "tiny_d64": Workload("tiny_d64", 1, 2, 2, 256, 64, False, seed=1),
    "outlier_s4096": Workload("outlier_s4096", 4, 16, 16, 4096, 128, False, seed=2,
                              qk_std=1.5, k_outlier_frac=0.01),
    "causal_s8192": Workload("causal_s8192", 2, 16, 16, 8192, 128, True, seed=3),
    "gqa_doc_s16384": Workload("gqa_doc_s16384", 1, 32, 8, 16384, 128, True, seed=4,
                               doc_lengths=(512, 4096)),
    "causal_bwd_s4096": Workload("causal_bwd_s4096", 2, 16, 16, 4096, 128, True, seed=5,
                                 backward=True),
    # Causal sliding window of 4096 keys (window_left 4095) over S = 16384.
    "window_s16384": Workload("window_s16384", 1, 16, 16, 16384, 128, True, seed=6,
                              window=(4095, 0)),
    # The headline shape with e4m3 inputs (the low-precision forward).
    "causal_s8192_fp8": Workload("causal_s8192_fp8", 2, 16, 16, 8192, 128, True, seed=3,
                                 dtype="fp8"),
    # The headline shape in FP4 (NVFP4 Q/K with power-of-two block scales,
    # MXFP4 V), for the Direct-P forward.
    "causal_s8192_fp4": Workload("causal_s8192_fp4", 2, 16, 16, 8192, 128, True, seed=3,
                                 dtype="fp4"),
    # The shape of the FP4 page's peak Direct-P figure ("Hardware-Aware FP4
    # FlashAttention-4", "Rendimiento de Inferencia Forward": S32768/H24,
    # D = 128, inference, so no mask), in FP4 and in bf16 for the ratio.
    "full_s32768_h24_fp4": Workload("full_s32768_h24_fp4", 1, 24, 24, 32768, 128, False, seed=8,
                                    dtype="fp4"),
    "full_s32768_h24": Workload("full_s32768_h24", 1, 24, 24, 32768, 128, False, seed=8),
}

HEADLINE = "causal_s8192"


def draw_doc_offsets(S: int, seed: int, lo: int = 512, hi: int = 4096) -> np.ndarray:
    """Document boundaries: int32 [num_docs + 1], offsets[0] = 0, offsets[-1] = S."""
    rng = np.random.default_rng(seed)
    lengths = []
    total = 0
    while total < S:
        n = int(rng.integers(lo, hi, endpoint=True))
        n = min(n, S - total)
        lengths.append(n)
        total += n
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def make_tensors(B, Hq, Hkv, Sq, Sk, D, seed, *, qk_std=1.0, k_outlier_frac=0.0,
                 k_outlier_mult=8.0, with_dout=False, v_std=1.0):
    """bf16 CPU tensors q [B,Sq,Hq,D], k/v [B,Sk,Hkv,D] (and dout like q)."""
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn((B, Sq, Hq, D), generator=g, dtype=torch.float32) * qk_std
    k = torch.randn((B, Sk, Hkv, D), generator=g, dtype=torch.float32) * qk_std
    v = torch.randn((B, Sk, Hkv, D), generator=g, dtype=torch.float32) * v_std
    if k_outlier_frac > 0.0:
        sel = torch.rand((B, Sk, Hkv), generator=g) < k_outlier_frac
        k = torch.where(sel[..., None], k * k_outlier_mult, k)
    out = {"q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16), "v": v.to(torch.bfloat16)}
    if with_dout:
        out["dout"] = torch.randn((B, Sq, Hq, D), generator=g,
                                  dtype=torch.float32).to(torch.bfloat16)
    return out


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor e4m3 codes (torch.float8_e4m3fn) and the descale factor
    with x ~= descale * codes."""
    amax = float(x.abs().max())
    descale = amax / 448.0 if amax > 0 else 1.0
    return (x.float() / descale).to(torch.float8_e4m3fn), descale


def make_tensors_fp8(B, Hq, Hkv, Sq, Sk, D, seed, *, qk_std=1.0, v_std=1.0):
    """e4m3 CPU tensors q8/k8/v8 and their descale factors (fp32 draws in
    the order Q, K, V, as make_tensors)."""
    g = torch.Generator().manual_seed(int(seed))
    out = {}
    for name, shape, std in (("q", (B, Sq, Hq, D), qk_std), ("k", (B, Sk, Hkv, D), qk_std),
                             ("v", (B, Sk, Hkv, D), v_std)):
        codes, descale = quantize_e4m3(torch.randn(shape, generator=g, dtype=torch.float32) * std)
        out[name] = codes
        out[name + "_descale"] = descale
    return out


_E2M1_MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    """4-bit E2M1 codes of x (bit 3 = sign): the nearest of the magnitudes
    0, 0.5, 1, 1.5, 2, 3, 4, 6, ties to the even code, saturating at 6."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    idx = np.searchsorted(_E2M1_MIDPOINTS, a, side="left")
    tie = (idx < 7) & (a == _E2M1_MIDPOINTS[np.minimum(idx, 6)])
    idx = idx + (tie & (idx % 2 == 1))
    return (idx | np.where(np.signbit(x) & (idx > 0), 8, 0)).astype(np.uint8)


def _pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., D] 4-bit codes -> [..., D/2] bytes, element 2j in the low nibble."""
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def quantize_nvfp4(x: torch.Tensor, *, pow2_scales: bool, global_scale=None):
    """NVFP4 encoding of x [..., D] along its last dimension: (codes uint8
    [..., D/2], e4m3 scale bytes uint8 [..., D/16], per-tensor factor g) with
    x ~= g * scale * e2m1(code)."""
    xf = x.double().numpy()
    if global_scale is None:
        amax = float(np.abs(xf).max())
        global_scale = 1.0 if pow2_scales else (amax / (6.0 * 448.0) if amax > 0 else 1.0)
    blocks = xf.reshape(*xf.shape[:-1], -1, 16) / global_scale
    bmax = np.abs(blocks).max(axis=-1)
    if pow2_scales:
        e = np.ceil(np.log2(np.where(bmax > 0, bmax / 6.0, 1.0)))
        scale = np.exp2(np.clip(e, -9, 8))
    else:
        scale = torch.from_numpy(np.where(bmax > 0, bmax / 6.0, 1.0)).float() \
            .to(torch.float8_e4m3fn).float().double().numpy()
    scale_bytes = torch.from_numpy(scale).float().to(torch.float8_e4m3fn).view(torch.uint8)
    codes = e2m1_encode(blocks / scale[..., None]).reshape(xf.shape)
    return (torch.from_numpy(_pack_nibbles(codes)), scale_bytes.reshape(*xf.shape[:-1], -1),
            float(global_scale))


def quantize_mxfp4_keys(x: torch.Tensor):
    """MXFP4 encoding of V [B, S, H, D] with one UE8M0 scale per 32 keys of
    each (b, h, d) column: (codes uint8 [B, S, H, D/2], scale bytes uint8
    [B, ceil(S/32), H, D])."""
    xf = x.double().numpy()
    B, S, H, D = xf.shape
    nblk = (S + 31) // 32
    pad = np.zeros((B, nblk * 32, H, D))
    pad[:, :S] = xf
    blocks = pad.reshape(B, nblk, 32, H, D)
    amax = np.abs(blocks).max(axis=2)
    e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2, 0)
    e = np.clip(e, -127, 127)
    codes = e2m1_encode(blocks / np.exp2(e)[:, :, None]).reshape(B, nblk * 32, H, D)[:, :S]
    return (torch.from_numpy(_pack_nibbles(codes)),
            torch.from_numpy((e + 127).astype(np.uint8)))


def fp4_k_global(scale: float) -> float:
    """K's per-tensor factor that makes scale * k_global * log2(e) (with
    q_global = 1) the power of two just below scale * log2(e)."""
    c = scale * 1.4426950408889634
    return 2.0 ** math.floor(math.log2(c)) / c


def make_tensors_fp4(B, Hq, Hkv, Sq, Sk, D, seed, *, scale=None, pow2_scales=True,
                     qk_std=1.0, v_std=1.0):
    """NVFP4 Q/K and MXFP4 V (CPU uint8 tensors and per-tensor factors) from
    the fp32 draws of make_tensors (order Q, K, V)."""
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn((B, Sq, Hq, D), generator=g, dtype=torch.float32) * qk_std
    k = torch.randn((B, Sk, Hkv, D), generator=g, dtype=torch.float32) * qk_std
    v = torch.randn((B, Sk, Hkv, D), generator=g, dtype=torch.float32) * v_std
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = {}
    out["q_codes"], out["q_scales"], out["q_global"] = quantize_nvfp4(
        q, pow2_scales=pow2_scales, global_scale=1.0 if pow2_scales else None)
    kg = fp4_k_global(scale) if pow2_scales else None
    out["k_codes"], out["k_scales"], out["k_global"] = quantize_nvfp4(
        k, pow2_scales=pow2_scales, global_scale=kg)
    out["v_codes"], out["v_scales"] = quantize_mxfp4_keys(v)
    out["v_global"] = 1.0
    return out


def make_inputs(w: Workload):
    """All inputs of a named workload (CPU tensors) plus its mask arguments."""
    if w.dtype == "fp8":
        t = make_tensors_fp8(w.B, w.Hq, w.Hkv, w.S, w.S, w.D, w.seed, qk_std=w.qk_std)
    elif w.dtype == "fp4":
        t = make_tensors_fp4(w.B, w.Hq, w.Hkv, w.S, w.S, w.D, w.seed, qk_std=w.qk_std)
    else:
        t = make_tensors(w.B, w.Hq, w.Hkv, w.S, w.S, w.D, w.seed, qk_std=w.qk_std,
                         k_outlier_frac=w.k_outlier_frac, k_outlier_mult=w.k_outlier_mult,
                         with_dout=w.backward)
    t["doc_offsets"] = (draw_doc_offsets(w.S, w.seed, *w.doc_lengths)
                        if w.doc_lengths else None)
    t["causal"] = w.causal
    t["window"] = w.window
    t["scale"] = w.scale
    return t


def window_keys_per_row(Sq, Sk, window, causal):
    """Keys each query row may see under a sliding window (bottom-right
    aligned, as the masks): int64 [Sq]."""
    i = np.arange(Sq, dtype=np.int64) + (Sk - Sq)
    wl, wr = window
    lo = np.maximum(i - wl, 0) if wl >= 0 else np.zeros_like(i)
    hi = i if causal else np.full_like(i, Sk - 1)
    if wr >= 0:
        hi = np.minimum(hi, i + wr)
    hi = np.minimum(hi, Sk - 1)
    return np.maximum(hi - lo + 1, 0)


def useful_flops(B, Hq, Sq, Sk, D, *, causal=False, doc_offsets=None, window=None):
    """Forward FLOPs by the useful-work convention: 4*D per (row, key) pair,
    counting a causal mask as half of the square (per document when a
    document mask is given); a sliding window counts its allowed pairs
    exactly.  Used only for reporting throughput."""
    if window is not None and tuple(window) != (-1, -1):
        return 4.0 * B * Hq * D * float(window_keys_per_row(Sq, Sk, window, causal).sum())
    if doc_offsets is not None:
        lengths = np.diff(np.asarray(doc_offsets, dtype=np.int64))
        pairs = float(np.sum(lengths.astype(np.float64) ** 2)) / 2.0
        return 4.0 * B * Hq * D * pairs
    f = 4.0 * B * Hq * Sq * Sk * D
    return f / 2.0 if causal else f
