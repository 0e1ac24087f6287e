"""How often the forward's running-maximum rescale is skipped.

    python -m tiled_attention_blackwell_b200.rescale_stats --config causal_s8192 [--tau 8]

Runs one forward of a named workload through the rescale-statistics build of
the library (libattn_count.so: the same kernels compiled with per-row
counters) and prints one JSON line.  For every query row and every key block
after the row's first one, the kernel counts whether the rescale threshold
lets the block rescale the row's output accumulator; the same forward at
threshold 0 (a rescale whenever a block raises the running maximum, the
plain online softmax) gives the count the threshold is measured against.
It also counts the O corrections executed per warp (a warp rescales its 32
rows of O in tensor memory when any of them needs it).
"""
from __future__ import annotations

import argparse
import contextlib
import ctypes
import json
import os
import sys

import torch

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from tiled_attention_blackwell_b200 import attn, build  # noqa: E402
from tiled_attention_blackwell_b200.workloads import WORKLOADS, make_inputs  # noqa: E402


@contextlib.contextmanager
def counting_library():
    """The binding's argument marshalling pointed at the counting build for
    the duration (the product library is put back afterwards).  Yields a
    function that sets or clears the device counter buffer."""
    path = build.build_count()
    L = ctypes.CDLL(path)
    L.attn_count_set_buffer.restype = None
    L.attn_count_set_buffer.argtypes = [ctypes.c_void_p]
    with attn._lock:
        saved = attn._LIB_PATH, attn._lib
        attn._LIB_PATH, attn._lib = path, None
    try:
        yield lambda counts: L.attn_count_set_buffer(
            None if counts is None else ctypes.c_void_p(counts.data_ptr()))
    finally:
        with attn._lock:
            attn._LIB_PATH, attn._lib = saved


def _count(w, t, tau: float):
    q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
    docs = None if t["doc_offsets"] is None else \
        torch.as_tensor(t["doc_offsets"], dtype=torch.int32, device="cuda")
    window = None if tuple(w.window) == (-1, -1) else w.window
    counts = torch.zeros(4, dtype=torch.int64, device="cuda")
    with counting_library() as set_counts:
        set_counts(counts)
        attn.attention(q, k, v, scale=w.scale, causal=w.causal, window=window, doc_offsets=docs,
                       options=attn.default_options(rescale_threshold=tau))
        torch.cuda.synchronize()
        set_counts(None)
        attn.check_device_status()
    return [int(x) for x in counts.cpu()]


def rescale_stats(config: str, tau: float) -> dict:
    """Rescales of O at threshold `tau` against those without a threshold
    (every raise of a row's running maximum), per row and per warp."""
    w = WORKLOADS[config]
    if w.backward or w.dtype != "bf16":
        raise SystemExit("rescale statistics are taken on the bf16 forward workloads")
    t = make_inputs(w)
    blocks, _, taken, warp_corr = _count(w, t, tau)
    _, _, taken0, warp_corr0 = _count(w, t, 0.0)
    warp_blocks = blocks // 32  # a warp's 32 rows share their key blocks
    return {"workload": config, "rescale_threshold": tau,
            "row_blocks_after_first": blocks,
            "rescales_without_threshold": taken0, "rescales": taken,
            "skipped_fraction": round(1.0 - taken / taken0, 4) if taken0 else None,
            "warp_corrections_without_threshold": warp_corr0, "warp_corrections": warp_corr,
            "warp_skipped_fraction": round(1.0 - warp_corr / warp_corr0, 4) if warp_corr0 else None,
            "rescale_rate_per_row_block": round(taken / blocks, 5) if blocks else None,
            "warp_correction_rate": round(warp_corr / warp_blocks, 5) if warp_blocks else None}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--config", default="causal_s8192", choices=sorted(WORKLOADS))
    ap.add_argument("--tau", type=float, default=8.0)
    args = ap.parse_args(argv)
    print(json.dumps(rescale_stats(args.config, args.tau)), flush=True)


if __name__ == "__main__":
    main()
