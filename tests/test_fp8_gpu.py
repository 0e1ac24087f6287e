"""GPU parity of the fp8 (e4m3) forward against the fp64 oracle.

The oracle computes exact attention of the dequantized inputs
(descale * code); the fp8 path rounds P to e4m3 before the PV product and
keeps the row sum l from the unrounded values, so O_kernel - O_ref =
sum_j (p~_j - p_j) v_j / l.  The tolerance is derived per output element
from each row's exact probabilities P_ij = exp(s_ij - LSE_i) (s from the
dequantized inputs, LSE from the oracle):
  * e4m3 keeps 3 mantissa bits, so rounding moves a weight in its normal
    range by at most 2^-4 of itself: 2^-4 P_ij |v_jd|;
  * the kernel scales P by 2^(8 - tau) relative to its running maximum m
    (never above the row maximum M, at most tau below it); a key whose
    weight is at least 2^(tau-14) of the row maximum's is certainly in the
    normal range.  Below the normal range the rounding error is at most half
    a subnormal step, 2^-10, in the block's units, i.e. at most
    2^(tau-18) / sum_j exp(s_ij - M_i) in probability units (and never more
    than the probability itself);
  * 2^-10 P_ij |v_jd| more for the kernel's exponentials (the cubic's
    7.5e-5 relative error) and fp32 score rounding, 2^-8 |O_ref| for the bf16
    output and 1e-6 max|V| for fp32 accumulation;
  * as a whole-tensor check, cosine similarity >= 0.995 (the pages report
    about 0.990 for their FP8 path on Gaussian softmax tests);
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


def allowed_keys(i, Sq, Sk, causal, window, doc_offsets):
    """Bool [Sk]: the keys row i may see (bottom-right aligned causal,
    window bounds, same document)."""
    j = np.arange(Sk)
    diag = i + Sk - Sq
    ok = np.ones(Sk, dtype=bool)
    if causal:
        ok &= j <= diag
    if window is not None:
        wl, wr = window
        if wl >= 0:
            ok &= j >= diag - wl
        if wr >= 0:
            ok &= j <= diag + wr
    if doc_offsets is not None:
        offs = np.asarray(doc_offsets)
        d = np.searchsorted(offs, i, side="right") - 1
        ok &= (j >= offs[d]) & (j < offs[d + 1])
    return ok


def row_bounds(t, rows, lse_ref, o_ref, scale, tau, causal=False, window=None,
               doc_offsets=None):
    """Per-element bound [n, D] on |O_kernel - O_ref| for the given rows
    (b, hq, i), from each row's exact probabilities."""
    q, k, v = dequant(t, "q"), dequant(t, "k"), dequant(t, "v")
    Sq, Hq = q.shape[1], q.shape[2]
    Sk, Hkv = k.shape[1], k.shape[2]
    vmax = np.abs(v).max()
    out = np.zeros((len(rows), q.shape[3]))
    for r, (b, h, i) in enumerate(rows):
        hk = h // (Hq // Hkv)
        ok = allowed_keys(i, Sq, Sk, causal, window, doc_offsets)
        if not ok.any():
            continue
        s = scale * (k[b, ok, hk] @ q[b, i, h])
        P = np.exp(s - lse_ref[r])
        assert abs(P.sum() - 1.0) < 1e-9, "probabilities do not sum to one"
        M = s.max()
        sum_w = np.exp(lse_ref[r] - M)
        surely_normal = (s - M) * np.log2(np.e) >= tau - 14
        sub = np.where(surely_normal, 0.0, np.minimum(P, 2.0 ** (tau - 18) / sum_w))
        e = (2.0 ** -4 + 2.0 ** -10) * P + sub
        out[r] = e @ np.abs(v[b, ok, hk]) + 2.0 ** -8 * np.abs(o_ref[r]) + 1e-6 * vmax
    return out


def all_rows(B, Hq, Sq):
    b, h, i = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(Sq), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), i.ravel()], 1)


def check(o, lse, o_ref, lse_ref, bound, what):
    """o, o_ref, bound: [n, D]; lse, lse_ref: [n] (the same rows)."""
    assert np.isfinite(o).all(), f"{what}: non-finite O"
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: -inf rows differ"
    err = np.abs(o - o_ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond their bound, "
                           f"worst excess {float((err - bound).max()):.3e}")
    cos = float((o * o_ref).sum() / (np.linalg.norm(o) * np.linalg.norm(o_ref) + 1e-300))
    assert cos >= COS_MIN, f"{what}: cosine similarity {cos:.5f}"
    lse_err = np.abs(np.where(empty, 0.0, lse) - np.where(empty, 0.0, lse_ref))
    assert lse_err.max() <= LSE_TOL, f"{what}: LSE abs {lse_err.max():.3e}"
    return cos


def by_rows(o, lse, rows):
    """Rows (b, hq, i) of O [B,S,H,D] and LSE [B,H,S]."""
    return o[rows[:, 0], rows[:, 2], rows[:, 1]], lse[rows[:, 0], rows[:, 1], rows[:, 2]]


def run_gpu(t, scale, *, causal=False, window=None, doc_offsets=None, tau=8.0, exp2_mode=1):
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    docs = None if doc_offsets is None else torch.as_tensor(doc_offsets, dtype=torch.int32,
                                                             device=DEV)
    opts = attn.default_options(rescale_threshold=tau, exp2_mode=exp2_mode)
    o, lse = attn.attention_fp8(q, k, v, q_descale=t["q_descale"], k_descale=t["k_descale"],
                                v_descale=t["v_descale"], scale=scale, causal=causal,
                                window=window, doc_offsets=docs, options=opts)
    torch.cuda.synchronize()
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def oracle_fp8(t, scale, **mask):
    return oracle.attn_fwd_fp8(t["q"], t["k"], t["v"], q_descale=t["q_descale"],
                               k_descale=t["k_descale"], v_descale=t["v_descale"],
                               scale=scale, **mask)


def run_case(B, Hq, Hkv, Sq, Sk, seed, *, causal=False, window=None, doc_offsets=None,
             tau=8.0, exp2_mode=1, qk_std=1.0):
    D = 128
    t = make_tensors_fp8(B, Hq, Hkv, Sq, Sk, D, seed, qk_std=qk_std)
    scale = 1.0 / math.sqrt(D)
    mask = dict(causal=causal, window=window, doc_offsets=doc_offsets)
    o, lse = run_gpu(t, scale, tau=tau, exp2_mode=exp2_mode, **mask)
    o_ref, lse_ref = oracle_fp8(t, scale, **mask)
    rows = all_rows(B, Hq, Sq)
    o_s, lse_s = by_rows(o, lse, rows)
    o_r, lse_r = by_rows(o_ref, lse_ref, rows)
    bound = row_bounds(t, rows, lse_r, o_r, scale, tau, **mask)
    return check(o_s, lse_s, o_r, lse_r, bound,
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
    configuration: sampled rows against the oracle element by element with
    their own bounds, finite results everywhere."""
    w = WORKLOADS["causal_s8192_fp8"]
    t = make_inputs(w)
    o, lse = run_gpu(t, w.scale, causal=w.causal)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    rng = np.random.default_rng(w.seed)
    fixed = [0, 1, 127, 128, 255, 256, w.S // 2, w.S - 129, w.S - 1]
    rows = [(b, h, i) for b in range(w.B) for h in (0, w.Hq - 1) for i in fixed]
    rows += [(int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.S)))
             for _ in range(150)]
    rows = np.array(rows, dtype=np.int64)
    o_ref, lse_ref = oracle_fp8(t, w.scale, causal=w.causal, rows=rows)
    o_s, lse_s = by_rows(o, lse, rows)
    bound = row_bounds(t, rows, lse_ref, o_ref, w.scale, 8.0, causal=w.causal)
    check(o_s, lse_s, o_ref, lse_ref, bound, "causal_s8192_fp8 sampled")
    vmax = float(np.abs(dequant(t, "v")).max())
    assert bound.max() <= 2.0 ** -3 * vmax, "the bound no longer binds"


def test_bound_catches_planted_oracle_mistakes():
    """The element-wise bound binds: an oracle given V with two key blocks
    swapped, or one head's probabilities negated, disagrees with the kernel
    beyond it (the mistakes are planted in the oracle's inputs and results,
    on the CPU)."""
    B, H, S, D = 1, 4, 700, 128
    t = make_tensors_fp8(B, H, H, S, S, D, seed=508)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_gpu(t, scale, causal=True)
    rows = all_rows(B, H, S)
    o_s, lse_s = by_rows(o, lse, rows)
    o_ref, lse_ref = oracle_fp8(t, scale, causal=True)
    o_r, lse_r = by_rows(o_ref, lse_ref, rows)
    bound = row_bounds(t, rows, lse_r, o_r, scale, 8.0, causal=True)
    check(o_s, lse_s, o_r, lse_r, bound, "clean")
    # V with key blocks [128, 256) and [384, 512) swapped
    bad = dict(t)
    v = t["v"].clone()
    v[:, 128:256], v[:, 384:512] = t["v"][:, 384:512], t["v"][:, 128:256]
    bad["v"] = v
    o_bad, _ = oracle_fp8(bad, scale, causal=True)
    assert (np.abs(o_s - by_rows(o_bad, lse_ref, rows)[0]) > bound).any()
    # one head's probabilities negated: its output flips sign
    o_neg = o_ref.copy()
    o_neg[:, :, 2] *= -1.0
    assert (np.abs(o_s - by_rows(o_neg, lse_ref, rows)[0]) > bound).any()


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
