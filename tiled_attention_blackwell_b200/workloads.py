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
    round-to-nearest conversion of x / descale).
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
    dtype: str = "bf16"  # "bf16" or "fp8" (e4m3 Q, K, V with per-tensor factors)

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


def make_inputs(w: Workload):
    """All inputs of a named workload (CPU tensors) plus its mask arguments."""
    if w.dtype == "fp8":
        t = make_tensors_fp8(w.B, w.Hq, w.Hkv, w.S, w.S, w.D, w.seed, qk_std=w.qk_std)
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
