#!/usr/bin/env python
"""Attention-forward benchmark on B200: TFLOP/s and % of BF16 tensor peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one forward pass (O and LSE) over one batch of the named workload
(default: the causal S=8192 one), inputs resident in HBM.  Prints ONE JSON
line on rank 0.  For N > 1 (launched under torchrun) every rank runs an
independent replica of the same workload on its own GPU: the path needs no
exchange between GPUs, so there is no collective on the data path ("replicas
only"); ranks synchronise only to start and stop the clock, and the time is
the max over ranks.

`--impl reference` times the fp64 CPU oracle (the only reference this
method has) on a bounded sample of rows of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import re
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tiled_attention_blackwell_b200.workloads import (HEADLINE, WORKLOADS,  # noqa: E402
                                                      make_inputs, useful_flops,
                                                      window_keys_per_row)

METRIC = "attention fwd TFLOP/s and % of B200 BF16 tensor peak (S=8192 causal, D=128)"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["tiled_attention_blackwell_b200/csrc/fwd_kernel.cuh",
                  "tiled_attention_blackwell_b200/csrc/fwd_persistent.cuh",
                  "tiled_attention_blackwell_b200/csrc/bwd_kernel.cuh",
                  "tiled_attention_blackwell_b200/csrc/common.cuh",
                  "tiled_attention_blackwell_b200/csrc/ptx.cuh",
                  "tiled_attention_blackwell_b200/csrc/exp2_poly.cuh",
                  "tiled_attention_blackwell_b200/csrc/fp4_dequant.cuh",
                  "tiled_attention_blackwell_b200/csrc/fp4_prepare.cuh",
                  "tiled_attention_blackwell_b200/csrc/fwd_fp4_kernel.cuh",
                  "tiled_attention_blackwell_b200/csrc/attn_api.cu"]
FP4_INPUTS = ("q_codes", "q_scales", "k_codes", "k_scales", "v_codes", "v_scales")


# ------------------------------------------------------------------ helpers

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing leg (faster local iteration)")
    ap.add_argument("--exp2-mode", type=int, default=None)
    ap.add_argument("--rescale-threshold", type=float, default=None)
    ap.add_argument("--softcap", type=float, default=None,
                    help="time with the soft-capping score modifier (cap value)")
    ap.add_argument("--alibi", action="store_true",
                    help="time with ALiBi slopes 2^(-8(h+1)/Hq)")
    ap.add_argument("--classifier", default="affine", choices=["affine", "exp2"],
                    help="Direct-P code classifier of the fp4 workloads")
    ap.add_argument("--fp4-mma", default="block_scaled", choices=["block_scaled", "f16"],
                    help="tensor-core products of the fp4 workloads: block-scaled FP4 "
                         "(default) or f16 operands after a widening pass")
    ap.add_argument("--sustained-seconds", type=float, default=2.0,
                    help="length of the back-to-back run of the 'sustained' record (0: skip)")
    ap.add_argument("--no-rescale-stats", action="store_true",
                    help="skip the rescale statistics (a separate process on the counting build)")
    return ap.parse_args(argv)


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace collapsed, so that
    editing a comment does not invalidate a profile of the same code."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def _profile_fields(name: str):
    try:
        text = open(os.path.join(ROOT, "profiles", name)).read()
    except OSError:
        return {}
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    return fields


def profiled_traffic(config: str):
    """DRAM bytes per launch from the committed ncu summaries of this
    workload, if they were taken on the current kernel sources; else None."""
    for name, key in ((f"fwd_{config}_ncu.md", "dram_bytes_per_launch"),
                      ("fwd_all_workloads_ncu.md", f"dram_bytes_per_launch[{config}]")):
        fields = _profile_fields(name)
        if fields.get("kernel_sources_sha256") != kernel_source_hash() or key not in fields:
            continue
        try:
            return int(fields[key])
        except ValueError:
            return None
    return None


def allowed_keys_per_row(w, doc_offsets):
    """Number of keys each query row may see (for FLOP accounting of a row
    sample): causal -> i + 1, document-causal -> i - doc_start + 1, sliding
    window -> the window's width clipped at the sequence ends."""
    if tuple(w.window) != (-1, -1):
        return window_keys_per_row(w.S, w.S, w.window, w.causal)
    i = np.arange(w.S, dtype=np.int64)
    if doc_offsets is not None:
        starts = np.repeat(doc_offsets[:-1], np.diff(doc_offsets)).astype(np.int64)
        return (i - starts + 1) if w.causal else np.repeat(np.diff(doc_offsets), np.diff(doc_offsets))
    return (i + 1) if w.causal else np.full(w.S, w.S, dtype=np.int64)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = torch.cuda.get_device_properties(device_index).uuid
            uuid = str(uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                mask = get(self.h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------- distributed

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return rank, world, local


def init_process_group(world: int, local: int, backend: str = "nccl"):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120), **kw)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------- CPU oracle leg

def oracle_sample(w, inputs, n_rows: int, seed: int = 0):
    """Time the oracle on `n_rows` random rows of the workload.  Returns
    (seconds, useful FLOPs, threads)."""
    import oracle  # test infrastructure: only this leg of the benchmark loads it
    rng = np.random.default_rng(seed)
    rows = np.stack([rng.integers(0, w.B, n_rows), rng.integers(0, w.Hq, n_rows),
                     rng.integers(0, w.S, n_rows)], axis=1).astype(np.int64)
    keys = allowed_keys_per_row(w, inputs["doc_offsets"])
    flops = float((4.0 * w.D * keys[rows[:, 2]]).sum())
    window = None if w.window == (-1, -1) else w.window
    t0 = time.perf_counter()
    if w.dtype == "fp8":
        oracle.attn_fwd_fp8(inputs["q"], inputs["k"], inputs["v"],
                            q_descale=inputs["q_descale"], k_descale=inputs["k_descale"],
                            v_descale=inputs["v_descale"], scale=w.scale, causal=w.causal,
                            window=window, doc_offsets=inputs["doc_offsets"], rows=rows)
    elif w.dtype == "fp4":
        oracle.attn_fwd_fp4(*[inputs[n] for n in ("q_codes", "q_scales", "q_global", "k_codes",
                                                  "k_scales", "k_global", "v_codes", "v_scales",
                                                  "v_global")],
                            scale=w.scale, causal=w.causal, window=window,
                            doc_offsets=inputs["doc_offsets"], rows=rows,
                            classifier=inputs.get("classifier", "affine"))
    else:
        oracle.attn_fwd(inputs["q"], inputs["k"], inputs["v"], scale=w.scale, causal=w.causal,
                        window=window, doc_offsets=inputs["doc_offsets"], rows=rows)
    return time.perf_counter() - t0, flops, oracle.num_threads()


def oracle_bwd_sample(w, inputs, n_kv: int):
    """Time the oracle backward on batch 0's first n_kv key/value heads (and
    their query heads): a smaller problem of the same shape per head.
    Returns (seconds, useful FLOPs by the 2.5x-forward convention, threads)."""
    import oracle  # test infrastructure: only this leg of the benchmark loads it
    g = w.Hq // w.Hkv
    q = inputs["q"][:1, :, :n_kv * g].contiguous()
    dout = inputs["dout"][:1, :, :n_kv * g].contiguous()
    k = inputs["k"][:1, :, :n_kv].contiguous()
    v = inputs["v"][:1, :, :n_kv].contiguous()
    window = None if w.window == (-1, -1) else w.window
    flops = 2.5 * useful_flops(1, n_kv * g, w.S, w.S, w.D, causal=w.causal,
                               doc_offsets=inputs["doc_offsets"], window=w.window)
    t0 = time.perf_counter()
    oracle.attn_bwd(q, k, v, dout, scale=w.scale, causal=w.causal, window=window,
                    doc_offsets=inputs["doc_offsets"])
    return time.perf_counter() - t0, flops, oracle.num_threads()


def kv_heads_for_seconds(w, inputs, seconds: float) -> int:
    """Number of key/value heads of batch 0 the oracle backward covers in
    about `seconds` (at least one, at most all of batch 0's)."""
    t1, _, _ = oracle_bwd_sample(w, inputs, 1)
    return int(min(max(1, seconds // max(t1, 1e-3)), w.Hkv))


def rescale_stats(config: str, tau):
    """How often the threshold skips the running-maximum rescale on this
    workload: forwards at the run's threshold and at 0 through the counting
    build of the library, in a process of its own (it loads that library
    instead of the product's)."""
    import subprocess
    cmd = [sys.executable, "-m", "tiled_attention_blackwell_b200.rescale_stats", "--config",
           config, "--tau", str(8.0 if tau is None else float(tau))]
    try:
        out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300,
                             check=True).stdout
        return [json.loads(line) for line in out.splitlines() if line.startswith("{")][-1]
    except (subprocess.SubprocessError, ValueError, IndexError) as e:
        return {"unavailable": str(e).splitlines()[0][:200]}


def metric_for(w, softcap=None, alibi=False, classifier="affine") -> str:
    mods = "".join([f", softcap {softcap:g}" if softcap is not None else "",
                    ", ALiBi" if alibi else ""])
    if w.dtype == "fp4":
        # f16 operands on the tensor cores: the same dense peak as bf16
        return (f"attention fwd TFLOP/s and % of B200 BF16/F16 tensor peak ({w.describe()}, "
                f"Direct-P {classifier} classifier)")
    if w.backward:
        return f"attention bwd TFLOP/s and % of B200 BF16 tensor peak ({w.describe()}{mods})"
    if w.dtype == "fp8":
        return f"attention fwd TFLOP/s and % of B200 FP8 tensor peak ({w.describe()})"
    if w.name != HEADLINE or alibi or softcap is not None:
        return f"attention fwd TFLOP/s and % of B200 BF16 tensor peak ({w.describe()}{mods})"
    return METRIC


def rows_for_seconds(w, inputs, seconds: float) -> int:
    """Calibrate the row count so the oracle runs for about `seconds`.  Each
    call has a fixed cost (converting the inputs) besides the per-row work, so
    two sample sizes give both terms."""
    n1, n2 = 200, 1200
    t1, _, _ = oracle_sample(w, inputs, n1, seed=123)
    t2, _, _ = oracle_sample(w, inputs, n2, seed=124)
    per_row = max((t2 - t1) / (n2 - n1), 1e-7)
    fixed = max(t1 - n1 * per_row, 0.0)
    return max(100, int(max(seconds - fixed, 0.0) / per_row))


def workload_config(w, doc_offsets):
    cfg = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Sq": w.S, "Sk": w.S,
           "D": w.D, "mask": ("document-causal" if doc_offsets is not None else
                              ("causal" if w.causal else "none")),
           "scale": w.scale}
    if doc_offsets is not None:
        cfg["num_docs"] = int(len(doc_offsets) - 1)
    if tuple(w.window) != (-1, -1):
        cfg["mask"] = "causal sliding window" if w.causal else "sliding window"
        cfg["window"] = list(w.window)
    # bytes per Q/K/V element (fp4: half a byte of code plus the block
    # scales, 1/16 byte for NVFP4 Q/K and 1/32 for MXFP4 V); O is bf16
    nq, nkv = w.B * w.S * w.Hq * w.D, w.B * w.S * w.Hkv * w.D
    if w.dtype == "fp4":
        in_bytes = nq * (0.5 + 1 / 16) + nkv * (0.5 + 1 / 16) + nkv * (0.5 + 1 / 32)
    else:
        in_bytes = (1 if w.dtype == "fp8" else 2) * (nq + 2 * nkv)
    io_bytes = int(in_bytes + 2 * nq + 4 * w.B * w.Hq * w.S)
    cfg["io_bytes"] = io_bytes
    cfg["l2"] = (f"inputs+outputs {io_bytes / 2**20:.0f} MiB > L2 126 MiB; no flush"
                 if io_bytes > L2_BYTES else "L2 flushed between steps")
    return cfg


# ---------------------------------------------------------------- our arm

def run_ours(args):
    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    init_process_group(world, local)
    device = torch.device("cuda", local)
    from tiled_attention_blackwell_b200 import attn

    w = WORKLOADS[args.config]
    inp = make_inputs(w)
    docs_np = inp["doc_offsets"]
    flops = useful_flops(w.B, w.Hq, w.S, w.S, w.D, causal=w.causal, doc_offsets=docs_np,
                         window=w.window)
    cfg = workload_config(w, docs_np)
    cfg["parallelism"] = f"replicas x{world}" if world > 1 else "single GPU"

    fp8, fp4 = w.dtype == "fp8", w.dtype == "fp4"
    host = {n: inp[n].pin_memory() for n in (FP4_INPUTS if fp4 else ("q", "k", "v"))}
    dev = {n: host[n].to(device) for n in host}
    docs = None if docs_np is None else torch.as_tensor(docs_np, dtype=torch.int32, device=device)
    o = torch.empty((w.B, w.S, w.Hq, w.D), dtype=torch.bfloat16, device=device)
    ws4 = None
    if fp4:
        ws4 = torch.empty(attn.fp4_workspace_size(w.B, w.Hq, w.Hkv, w.S, w.S, w.D),
                          dtype=torch.uint8, device=device)
        cfg["classifier"] = args.classifier
        cfg["formats"] = "NVFP4 Q/K (power-of-two e4m3 block scales), MXFP4 V and P"
        cfg["products"] = args.fp4_mma
    lse = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device=device)
    window = None if w.window == (-1, -1) else w.window
    slopes = None
    if args.alibi:
        slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / w.Hq) for h in range(w.Hq)],
                              dtype=torch.float32, device=device)
        cfg["alibi"] = "slopes 2^(-8(h+1)/Hq)"
    if w.backward:
        # Backward workload: O and LSE come from one forward (with the same
        # score modifiers) before timing; a step is one attn_bwd (the dQ
        # kernel, which also forms the D_i row terms, then the dK/dV kernel).
        flops *= 2.5
        attn.attn_fwd(dev["q"], dev["k"], dev["v"], o, lse, scale=w.scale, causal=w.causal,
                      window=window, doc_offsets=docs, softcap=args.softcap,
                      alibi_slopes=slopes)
        host.update(o=o.cpu().pin_memory(), lse=lse.cpu().pin_memory(),
                    dout=inp["dout"].pin_memory())
        dev.update(o=o, lse=lse, dout=host["dout"].to(device))
        g_dq = torch.empty(o.shape, dtype=torch.float32, device=device)
        g_dk = torch.empty_like(dev["k"])
        g_dv = torch.empty_like(dev["v"])
        ws = torch.empty(attn.bwd_workspace_size(w.B, w.Hq, w.Hkv, w.S, w.S, w.D),
                         dtype=torch.uint8, device=device)
        outputs = [g_dq, g_dk, g_dv]
    else:
        outputs = [o, lse]
    flush = None if cfg["io_bytes"] > L2_BYTES else torch.empty(2 * L2_BYTES, dtype=torch.uint8,
                                                                 device=device)
    opts = None
    if args.softcap is not None:
        cfg["softcap"] = args.softcap
    if (args.exp2_mode is not None or args.rescale_threshold is not None
            or slopes is not None or args.softcap is not None):
        kw = {}
        if args.exp2_mode is not None:
            kw["exp2_mode"] = args.exp2_mode
        if args.rescale_threshold is not None:
            kw["rescale_threshold"] = args.rescale_threshold
        if args.softcap is not None:
            kw["softcap"] = args.softcap
        if slopes is not None:
            kw["alibi_slopes"] = slopes.data_ptr()
        opts = attn.default_options(**kw)
    stream = torch.cuda.current_stream(device)

    def run(d, outs, s):
        """One step of the path on stream s: inputs d, outputs outs."""
        if w.backward:
            attn.attn_bwd(d["q"], d["k"], d["v"], d["o"], d["lse"], d["dout"], outs[0], outs[1],
                          outs[2], ws, scale=w.scale, causal=w.causal, window=window,
                          doc_offsets=docs, stream=s, softcap=args.softcap, alibi_slopes=slopes)
        elif fp4:
            attn.attn_fwd_fp4(d["q_codes"], d["q_scales"], inp["q_global"], d["k_codes"],
                              d["k_scales"], inp["k_global"], d["v_codes"], d["v_scales"],
                              inp["v_global"], outs[0], outs[1], ws4, scale=w.scale,
                              causal=w.causal, window=window, doc_offsets=docs,
                              classifier=args.classifier, mma=args.fp4_mma, stream=s)
        elif fp8:
            attn.attn_fwd_fp8(d["q"], d["k"], d["v"], outs[0], outs[1],
                              q_descale=inp["q_descale"], k_descale=inp["k_descale"],
                              v_descale=inp["v_descale"], scale=w.scale, causal=w.causal,
                              window=window, doc_offsets=docs, options=opts, stream=s)
        else:
            attn.attn_fwd(d["q"], d["k"], d["v"], outs[0], outs[1], scale=w.scale,
                          causal=w.causal, window=window, doc_offsets=docs, options=opts,
                          stream=s)

    def step():
        run(dev, outputs, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    attn.check_device_status(stream)

    # ---- device-resident timing: K steps, per-launch events on the launch stream
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(device)
    with sampler:
        t_begin.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(device)
    barrier(world)
    attn.check_device_status(stream)
    burst_clocks = sampler.summary()
    total_ms = t_begin.elapsed_time(t_end)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    if flush is not None:
        # The L2 flush between steps is not part of the work: time the K
        # steps as the sum of their own event intervals.
        total_ms = float(sum(launch_ms))
        cfg["timed"] = "sum of the per-step event intervals (L2 flush excluded)"
    total_ms_max = max_over_ranks(total_ms, world, device)
    ms_per_step = total_ms_max / args.steps
    value = flops * args.steps * world / (total_ms_max / 1e3) / 1e12
    launch_avg_ms = float(np.mean(launch_ms))

    # ---- end to end through the C ABI: pinned host inputs in, results out.
    # Every step copies its inputs from pinned host memory and its results
    # back; with two sets of device buffers and three streams the copies of
    # neighbouring steps overlap a step's kernels (inputs of step i+1 and
    # results of step i-1 move while step i computes), as a serving loop
    # would run it.
    out_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outputs]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outputs)
    slots = [(dev, outputs),
             ({n: torch.empty_like(t) for n, t in dev.items()},
              [torch.empty_like(t) for t in outputs])]
    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in", "cmp", "out")}

    def e2e_steps(n):
        for i in range(n):
            k = i % 2
            d, outs = slots[k]
            if i >= 2:
                s_in.wait_event(ev["cmp"][k])    # step i-2 has read these inputs
                s_cmp.wait_event(ev["out"][k])   # and its results have left
            with torch.cuda.stream(s_in):
                for name in host:
                    d[name].copy_(host[name], non_blocking=True)
            ev["in"][k].record(s_in)
            s_cmp.wait_event(ev["in"][k])
            run(d, outs, s_cmp)
            ev["cmp"][k].record(s_cmp)
            s_out.wait_event(ev["cmp"][k])
            with torch.cuda.stream(s_out):
                for hst, dvc in zip(out_host, outs):
                    hst.copy_(dvc, non_blocking=True)
            ev["out"][k].record(s_out)

    torch.cuda.synchronize(device)
    e2e_steps(min(args.warmup, 3))
    torch.cuda.synchronize(device)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_cmp.wait_event(e0)
    s_out.wait_event(e0)
    e2e_steps(args.steps)
    s_out.wait_event(ev["cmp"][(args.steps - 1) % 2])
    e1.record(s_out)
    torch.cuda.synchronize(device)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    e2e_value = flops * args.steps * world / (e2e_ms / 1e3) / 1e12

    # ---- sustained: the same step back to back for a few seconds, so the
    # clock settles where the power limit puts it; its own clock samples.
    sustained = None
    if args.sustained_seconds > 0:
        n_sus = max(1, int(math.ceil(args.sustained_seconds * 1e3 / max(launch_avg_ms, 1e-3))))
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sus_sampler = ClockSampler(local, period_s=0.01)
        torch.cuda.synchronize(device)
        with sus_sampler:
            s0.record(stream)
            for _ in range(n_sus):
                if flush is not None:
                    flush.zero_()
                step()
            s1.record(stream)
            torch.cuda.synchronize(device)
        attn.check_device_status(stream)
        sus_ms = s0.elapsed_time(s1)
        sustained = {"launches": n_sus, "seconds": round(sus_ms / 1e3, 3),
                     "value": round(flops * n_sus / (sus_ms / 1e3) / 1e12, 2), "unit": UNIT,
                     "clocks": sus_sampler.summary()}
        if flush is not None:
            sustained["note"] = "includes the L2 flush between steps"

    peaks, peak_kind = read_peaks()
    achieved = flops / (launch_avg_ms / 1e3) / 1e12
    # fp8 and block-scaled fp4 contractions: the measured bf16 peak times the
    # nominal dense fp8 / bf16 (4.5 / 2.25) or fp4 / bf16 (9 / 2.25) ratio.
    fp4_bs = fp4 and args.fp4_mma == "block_scaled"
    peak_mult = 2.0 if fp8 else (4.0 if fp4_bs else 1.0)
    peak = float(peaks["bf16_tflops"]) * peak_mult
    metric = metric_for(w, args.softcap, slopes is not None, args.classifier)
    result = {
        "metric": metric, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("fp8e4m3" if fp8 else
                  ("fp4e2m1 (NVFP4 Q/K, MXFP4 P/V) on block-scaled FP4 tensor cores" if fp4_bs
                   else "fp4e2m1 (NVFP4/MXFP4) on f16 tensor operands") if fp4 else "bf16"),
        "data": "synthetic", "config": cfg,
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": profiled_traffic(w.name),
                     "peak_source": (f"{peak_kind} bf16 burst (MEASURED_PEAKS.json)"
                                     if peak_kind == "measured" else "fallback 1590 TFLOP/s")
                     + (" x 2 (nominal fp8/bf16 dense ratio)" if fp8 else "")
                     + (" x 4 (nominal fp4/bf16 dense ratio)" if fp4_bs else ""),
                     "frac_of_sustained": round(achieved / (peak_mult * float(
                         peaks.get("bf16_tflops_sustained", peak))), 4),
                     "flops_per_launch": flops, "launch_ms": round(launch_avg_ms, 4),
                     "cycles_per_launch": (round(launch_avg_ms * 1e-3 * burst_clocks["sm_mhz"] * 1e6)
                                           if burst_clocks["sm_mhz"] else None),
                     "kernel": "attn_bwd (dQ kernel with the D_i row terms, then dK/dV kernel)"
                     if w.backward else
                     (("attn_fwd_fp4 (fp4_prepare_kernel + attn_fwd_fp4bs_kernel, timed together)"
                       if fp4_bs else
                       "attn_fwd_fp4 (fp4_dequant_kernel + attn_fwd_kernel, timed together)")
                      if fp4 else "attn_fwd_kernel")},
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "pipelining": "two buffer sets, copy-in / compute / copy-out streams"},
        "gpu_launches": args.steps * (2 if w.backward or fp4 else 1),
        "clocks": burst_clocks,
    }
    if sustained is not None:
        sus_peak = peak_mult * float(peaks.get("bf16_tflops_sustained", peak))
        sustained["frac_of_sustained_peak"] = round(sustained["value"] / sus_peak, 4)
        sustained["peak"] = sus_peak
        result["sustained"] = sustained
    if (rank == 0 and world == 1 and not args.no_rescale_stats and not w.backward
            and w.dtype == "bf16" and slopes is None and args.softcap is None):
        result["rescale_stats"] = rescale_stats(w.name, args.rescale_threshold)
    inp["classifier"] = args.classifier
    if (rank == 0 and world == 1 and not args.no_cpu_baseline
            and slopes is None and args.softcap is None):
        if w.backward:
            n_kv = kv_heads_for_seconds(w, inp, 15.0)
            dt, fl, cores = oracle_bwd_sample(w, inp, n_kv)
            sample = (f"backward of batch 0's first {n_kv} key/value heads of {w.name}, "
                      f"fp64, {dt:.1f} s")
        else:
            n_rows = rows_for_seconds(w, inp, 15.0)
            dt, fl, cores = oracle_sample(w, inp, n_rows)
            sample = f"{n_rows} random (b, head, row) rows of {w.name}, fp64, {dt:.1f} s"
        result["cpu_baseline"] = {"value": round(fl / dt / 1e12, 6), "unit": UNIT,
                                  "cores": cores, "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.config]
    inp = make_inputs(w)
    inp["classifier"] = args.classifier
    cfg = workload_config(w, inp["doc_offsets"])
    cfg["parallelism"] = "CPU oracle, rank 0 only"
    if w.dtype == "fp4":
        cfg["classifier"] = args.classifier
    # each step: ~2 s of oracle work, so steps + warmup end within minutes
    if w.backward:
        n_kv = kv_heads_for_seconds(w, inp, 2.0)
        sample_fn = lambda i: oracle_bwd_sample(w, inp, n_kv)  # noqa: E731
        sample = f"backward of batch 0's first {n_kv} key/value heads of {w.name} per step, fp64"
    else:
        n_rows = rows_for_seconds(w, inp, 2.0)
        sample_fn = lambda i: oracle_sample(w, inp, n_rows, seed=i)  # noqa: E731
        sample = f"{n_rows} random (b, head, row) rows of {w.name} per step, fp64"
    for i in range(args.warmup):
        sample_fn(1000 + i)
    times, fl_total, cores = [], 0.0, 1
    for i in range(args.steps):
        dt, fl, cores = sample_fn(i)
        times.append(dt)
        fl_total += fl
    total = sum(times)
    value = fl_total / total / 1e12
    result = {
        "impl": "reference", "metric": metric_for(w, classifier=args.classifier),
        "value": round(value, 6), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": cfg,
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores,
                         "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
