"""Host-side logic of bench.py on the CPU: FLOP accounting, the reduction
of timings over ranks (world size 2 on gloo), and the reference arm's
rank handling.  The path needs no data exchange between GPUs (replicas
only); ranks meet only to start and stop the clock."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from tiled_attention_blackwell_b200.workloads import WORKLOADS, Workload, useful_flops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        ms = [12.5, 17.0][rank]
        out[rank] = (bench.max_over_ranks(ms, world, dev), bench.sum_over_ranks(ms, world, dev))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_and_sum_over_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1] == (17.0, 29.5)


def test_single_rank_reductions_are_identity():
    dev = torch.device("cpu")
    assert bench.max_over_ranks(3.0, 1, dev) == 3.0
    assert bench.sum_over_ranks(3.0, 1, dev) == 3.0


@pytest.mark.parametrize("name", ["causal_s8192", "gqa_doc_s16384", "outlier_s4096",
                                  "tiny_d64", "window_s16384"])
def test_row_key_counts_match_dense_mask(name):
    """The per-row key counts used for the CPU sample's FLOPs equal the
    allowed-set sizes of the mask, on a shrunken copy of the workload."""
    w0 = WORKLOADS[name]
    S = 1000
    window = (255, 0) if tuple(w0.window) != (-1, -1) else (-1, -1)
    w = Workload(name, 1, 1, 1, S, w0.D, w0.causal, w0.seed, doc_lengths=w0.doc_lengths,
                 window=window)
    docs = None
    if w.doc_lengths:
        docs = np.array([0, 130, 131, 600, 1000], dtype=np.int32)
    keys = bench.allowed_keys_per_row(w, docs)
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    allowed = np.ones((S, S), dtype=bool)
    if w.causal:
        allowed &= j <= i
    if docs is not None:
        ids = np.repeat(np.arange(len(docs) - 1), np.diff(docs))
        allowed &= ids[:, None] == ids[None, :]
    if window != (-1, -1):
        allowed &= j >= i - window[0]
    np.testing.assert_array_equal(keys, allowed.sum(axis=1))
    if window != (-1, -1):
        assert useful_flops(1, 1, S, S, w.D, causal=True, window=window) == \
            4.0 * w.D * allowed.sum()
    # and the whole-workload convention: causal = half of the square
    elif docs is None:
        full = useful_flops(1, 1, S, S, w.D, causal=w.causal)
        expect = 4.0 * w.D * (S * S / 2 if w.causal else S * S)
        assert full == expect


def test_reference_arm_other_ranks_exit_silently():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--config", "tiny_d64"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line():
    import json
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--config", "tiny_d64"], cwd=ROOT,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["higher_is_better"] is True


def test_profiled_traffic_is_tied_to_the_kernel_sources(monkeypatch):
    """The roofline's traffic comes from the committed ncu summary only while
    the kernel sources hash to the value recorded there."""
    real = bench.kernel_source_hash()
    fields = bench._profile_fields("fwd_causal_s8192_ncu.md")
    if fields.get("kernel_sources_sha256") == real:
        assert bench.profiled_traffic("causal_s8192") == int(fields["dram_bytes_per_launch"])
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0000000000000000")
    assert bench.profiled_traffic("causal_s8192") is None
    assert bench.profiled_traffic("causal_s8192_fp8") is None


def test_metric_names_per_workload():
    assert bench.metric_for(WORKLOADS["causal_s8192"]) == bench.METRIC
    assert "bwd" in bench.metric_for(WORKLOADS["causal_bwd_s4096"])
    assert "FP8" in bench.metric_for(WORKLOADS["causal_s8192_fp8"])
    assert "softcap 30" in bench.metric_for(WORKLOADS["causal_s8192"], softcap=30.0)
    assert "ALiBi" in bench.metric_for(WORKLOADS["causal_s8192"], alibi=True)
    m = bench.metric_for(WORKLOADS["causal_s8192_fp4"], classifier="exp2")
    assert "Direct-P exp2" in m and "fp4" in m


def test_fp4_io_bytes_count_codes_and_scales():
    w = WORKLOADS["causal_s8192_fp4"]
    cfg = bench.workload_config(w, None)
    n = w.B * w.S * w.Hq * w.D
    # Q, K: half a byte of code + one e4m3 byte per 16; V: + one UE8M0 byte
    # per 32; O bf16; LSE fp32
    assert cfg["io_bytes"] == int(2 * n * (0.5 + 1 / 16) + n * (0.5 + 1 / 32) + 2 * n
                                  + 4 * w.B * w.Hq * w.S)


def test_fp4_oracle_sample_runs():
    from tiled_attention_blackwell_b200.workloads import make_inputs
    w = Workload("fp4_small", 1, 2, 2, 96, 64, True, seed=9, dtype="fp4")
    inp = make_inputs(w)
    for classifier in ("affine", "exp2"):
        inp["classifier"] = classifier
        dt, fl, cores = bench.oracle_sample(w, inp, 20)
        assert dt > 0 and fl > 0 and cores >= 1


def test_oracle_backward_sample_counts_the_sliced_problem():
    """The CPU backward sample runs batch 0's first n key/value heads; its
    FLOPs are the 2.5x-forward count of exactly that slice."""
    from tiled_attention_blackwell_b200.workloads import make_inputs
    w = Workload("bwd_small", 2, 4, 2, 160, 64, True, seed=7, backward=True)
    inp = make_inputs(w)
    dt, fl, cores = bench.oracle_bwd_sample(w, inp, 1)
    assert dt > 0 and cores >= 1
    assert fl == 2.5 * useful_flops(1, 2, 160, 160, 64, causal=True)
    n = bench.kv_heads_for_seconds(w, inp, 1e-9)
    assert n == 1
    assert bench.kv_heads_for_seconds(w, inp, 1e9) == w.Hkv
