"""GPU parity of the fp8 (e4m3) forward against the fp64 oracle.

The oracle computes exact attention of the dequantized inputs
(descale * code); the fp8 path rounds P to e4m3 before the PV product, so the
tolerance comes from that rounding:
  * e4m3 keeps 3 mantissa bits: round-to-nearest changes a normal-range
    weight by at most 2^-4 of itself, so O moves by at most 2^-4 * max|V|;
    weights below e4m3's normal range (P < 2^-6 after the 2^(8 - tau) scale)
    move by at most 2^-10 each against a row sum of at least 2^(8 - tau), which
    adds N_keys * 2^(tau - 18) * max|V|; bf16 output rounding adds 2^-8 |O|;
  * as a whole-tensor check, cosine similarity >= 0.995 (a relative error of
    at most 0.1, i.e. the 2^-4 weight bound with room for the subnormal tail
    and the output rounding; the pages report about 0.990 for their FP8 path
    on Gaussian softmax tests);
  * LSE does not see the rounding of P (the row sum is taken from the
    unrounded values): |LSE error| <= 1e-3 as for bf16.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_blackwell_b200 import attn, build
from tiled_attention_blackwell_b200.workloads import WORKLOADS, make_inputs, make_tensors_fp8

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LSE_TOL = 1e-3
COS_MIN = 0.995


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    attn.lib()
    yield
    assert attn.device_status() == attn.ATTN_OK


def dequant(t, name):
    return t[name].to(torch.float64).numpy() * t[name + "_descale"]


def check(o, lse, o_ref, lse_ref, vmax, n_keys, tau, what):
    assert np.isfinite(o).all(), f"{what}: non-finite O"
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: -inf rows differ"
    bound = (2.0 ** -4 + n_keys * 2.0 ** (tau - 18)) * vmax + 2.0 ** -8 * np.abs(o_ref).max()
    err = np.abs(o - o_ref)
    assert err.max() <= bound, f"{what}: O max-abs {err.max():.3e} > {bound:.3e}"
    cos = float((o * o_ref).sum() / (np.linalg.norm(o) * np.linalg.norm(o_ref) + 1e-300))
    assert cos >= COS_MIN, f"{what}: cosine similarity {cos:.5f}"
    lse_err = np.abs(np.where(empty, 0.0, lse) - np.where(empty, 0.0, lse_ref))
    assert lse_err.max() <= LSE_TOL, f"{what}: LSE abs {lse_err.max():.3e}"
    return cos


def run_case(B, Hq, Hkv, Sq, Sk, seed, *, causal=False, window=None, doc_offsets=None,
             tau=8.0, exp2_mode=1, qk_std=1.0):
    D = 128
    t = make_tensors_fp8(B, Hq, Hkv, Sq, Sk, D, seed, qk_std=qk_std)
    scale = 1.0 / math.sqrt(D)
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    docs = None if doc_offsets is None else torch.as_tensor(doc_offsets, dtype=torch.int32,
                                                             device=DEV)
    opts = attn.default_options(rescale_threshold=tau, exp2_mode=exp2_mode)
    o, lse = attn.attention_fp8(q, k, v, q_descale=t["q_descale"], k_descale=t["k_descale"],
                                v_descale=t["v_descale"], scale=scale, causal=causal,
                                window=window, doc_offsets=docs, options=opts)
    torch.cuda.synchronize()
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    o_ref, lse_ref = oracle.attn_fwd_fp8(t["q"], t["k"], t["v"], q_descale=t["q_descale"],
                                         k_descale=t["k_descale"], v_descale=t["v_descale"],
                                         scale=scale, causal=causal, window=window,
                                         doc_offsets=doc_offsets)
    vmax = float(np.abs(dequant(t, "v")).max())
    return check(o, lse, o_ref, lse_ref, vmax, Sk, tau,
                 f"fp8 B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} causal={causal} tau={tau}")


@pytest.mark.parametrize("S", [1, 5, 127, 128, 129, 257, 700])
@pytest.mark.parametrize("causal", [False, True])
def test_shapes_and_ragged_tails(S, causal):
    run_case(2, 2, 2, S, S, seed=500 + S, causal=causal)


@pytest.mark.parametrize("heads", [(4, 1), (4, 2), (8, 8)])
def test_grouped_heads(heads):
    run_case(1, heads[0], heads[1], 520, 520, seed=501, causal=True)


@pytest.mark.parametrize("tau", [0.0, 4.0, 8.0])
@pytest.mark.parametrize("exp2_mode", [0, 1, 2])
def test_rescale_threshold_and_exp2_split(tau, exp2_mode):
    run_case(1, 2, 2, 1000, 1000, seed=502, causal=True, tau=tau, exp2_mode=exp2_mode,
             qk_std=1.5)


@pytest.mark.parametrize("window", [(37, 50), (100, 0), (-1, 90)])
def test_sliding_window(window):
    run_case(1, 2, 2, 900, 900, seed=503, window=window)


def test_document_mask_and_unequal_lengths():
    run_case(1, 4, 2, 700, 700, seed=504, causal=True, doc_offsets=[0, 1, 130, 400, 700])
    run_case(1, 2, 2, 300, 1000, seed=505, causal=True)
    run_case(1, 2, 2, 1000, 300, seed=506, causal=True)


def test_full_size_workload_sampled():
    """The benchmark's fp8 workload at full size in the benchmark's launch
    configuration: sampled rows against the oracle, finite results everywhere."""
    w = WORKLOADS["causal_s8192_fp8"]
    t = make_inputs(w)
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    o, lse = attn.attention_fp8(q, k, v, q_descale=t["q_descale"], k_descale=t["k_descale"],
                                v_descale=t["v_descale"], scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    rng = np.random.default_rng(w.seed)
    fixed = [0, 1, 127, 128, 255, 256, w.S // 2, w.S - 129, w.S - 1]
    rows = [(b, h, i) for b in range(w.B) for h in (0, w.Hq - 1) for i in fixed]
    rows += [(int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.S)))
             for _ in range(150)]
    rows = np.array(rows, dtype=np.int64)
    o_ref, lse_ref = oracle.attn_fwd_fp8(t["q"], t["k"], t["v"], q_descale=t["q_descale"],
                                         k_descale=t["k_descale"], v_descale=t["v_descale"],
                                         scale=w.scale, causal=w.causal, rows=rows)
    o_s = o[rows[:, 0], rows[:, 2], rows[:, 1]]
    lse_s = lse[rows[:, 0], rows[:, 1], rows[:, 2]]
    vmax = float(np.abs(t["v"].to(torch.float64).numpy()).max() * t["v_descale"])
    check(o_s, lse_s, o_ref, lse_ref, vmax, w.S, 8.0, "causal_s8192_fp8 sampled")


def test_fp8_and_bf16_paths_agree_on_e4m3_representable_inputs():
    """Inputs that are exactly e4m3 values (descale 1) give the bf16 path the
    same numbers; the two outputs differ only by the rounding of P."""
    t = make_tensors_fp8(1, 2, 2, 400, 400, 128, seed=507)
    q8, k8, v8 = (t[n].to(DEV) for n in ("q", "k", "v"))
    o8, l8 = attn.attention_fp8(q8, k8, v8, q_descale=1.0, k_descale=1.0, v_descale=1.0,
                                scale=0.01, causal=True)
    ob, lb = attn.attention(q8.to(torch.bfloat16), k8.to(torch.bfloat16), v8.to(torch.bfloat16),
                            scale=0.01, causal=True)
    torch.cuda.synchronize()
    assert torch.allclose(l8, lb, atol=1e-3)
    vmax = float(v8.float().abs().max())
    assert float((o8.float() - ob.float()).abs().max()) <= 2.0 ** -3 * vmax
