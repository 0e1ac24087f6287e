"""GPU parity of the attention backward against the fp64 oracle.

The CUDA backward runs on the CUDA forward's O and LSE; the oracle computes
its own O and LSE in fp64 from the same bf16 inputs.  Tolerance (fixed for
this operation): for each of dQ, dK, dV the max-abs error is at most
5e-2 times the max magnitude of that gradient.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_blackwell_b200 import attn, build
from tiled_attention_blackwell_b200.workloads import WORKLOADS, make_inputs, make_tensors

pytestmark = pytest.mark.gpu

GRAD_TOL = 5e-2
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    attn.lib()
    yield
    assert attn.device_status() == attn.ATTN_OK


def gpu_grads(t, *, scale, causal=False, window=None, doc_offsets=None, softcap=None,
              alibi_slopes=None):
    q, k, v, dout = (t[n].to(DEV) for n in ("q", "k", "v", "dout"))
    docs = None if doc_offsets is None else torch.as_tensor(doc_offsets, dtype=torch.int32,
                                                             device=DEV)
    slopes = None if alibi_slopes is None else torch.as_tensor(alibi_slopes, device=DEV)
    o, lse = attn.attention(q, k, v, scale=scale, causal=causal, window=window, doc_offsets=docs,
                            softcap=softcap, alibi_slopes=slopes)
    dq, dk, dv = attn.attention_backward(q, k, v, o, lse, dout, scale=scale, causal=causal,
                                         window=window, doc_offsets=docs, softcap=softcap,
                                         alibi_slopes=slopes)
    torch.cuda.synchronize()
    return [x.float().cpu().numpy().astype(np.float64) for x in (dq, dk, dv)]


def check_grads(got, ref, what):
    # A gradient can be exactly zero (one key per row makes dQ vanish); its
    # scale is then floored at 1e-3 of the largest of the three gradients.
    floor = 1e-3 * max(np.abs(r).max() for r in ref)
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        assert np.isfinite(g).all(), f"{what}: non-finite {name}"
        scale = max(np.abs(r).max(), floor, 1e-12)
        err = np.abs(g - r).max()
        assert err <= GRAD_TOL * scale, f"{what}: {name} max-abs {err:.3e} vs {GRAD_TOL}*{scale:.3e}"


def case(B, Hq, Hkv, Sq, Sk, D, seed, *, causal=False, window=None, docs=None, softcap=None,
         alibi_slopes=None, qk_std=1.0):
    t = make_tensors(B, Hq, Hkv, Sq, Sk, D, seed, with_dout=True, qk_std=qk_std)
    scale = 1.0 / math.sqrt(D)
    got = gpu_grads(t, scale=scale, causal=causal, window=window, doc_offsets=docs,
                    softcap=softcap, alibi_slopes=alibi_slopes)
    dq, dk, dv, _, _ = oracle.attn_bwd(t["q"], t["k"], t["v"], t["dout"], scale=scale,
                                       causal=causal, window=window, doc_offsets=docs,
                                       softcap=softcap or 0.0, alibi_slopes=alibi_slopes)
    check_grads(got, (dq, dk, dv), f"B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} D{D} causal={causal} "
                                   f"softcap={softcap} alibi={alibi_slopes is not None}")


def geometric_slopes(H):
    """Per-head ALiBi slopes 2^(-8 (h+1) / H) as fp32 (an input, like Q)."""
    return np.float32(2.0) ** (-8.0 * np.arange(1, H + 1, dtype=np.float32) / H)


@pytest.mark.parametrize("softcap", [3.0, 30.0])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_softcap_backward(softcap, D, causal):
    case(1, 2, 2, 400, 400, D, seed=301, causal=causal, softcap=softcap, qk_std=2.0)


@pytest.mark.parametrize("Sq,Sk", [(400, 400), (200, 520), (520, 200)])
@pytest.mark.parametrize("causal", [False, True])
def test_alibi_backward(Sq, Sk, causal):
    case(1, 4, 4, Sq, Sk, 128, seed=302, causal=causal, alibi_slopes=geometric_slopes(4))


@pytest.mark.parametrize("D", [64, 128])
def test_softcap_and_alibi_backward_with_gqa_window_and_documents(D):
    case(2, 4, 2, 450, 450, D, seed=303, causal=True, softcap=6.0,
         alibi_slopes=geometric_slopes(4), qk_std=1.5)
    case(1, 4, 1, 450, 450, D, seed=304, window=(100, 30), softcap=6.0,
         alibi_slopes=geometric_slopes(4))
    case(1, 2, 2, 400, 400, D, seed=305, causal=True, docs=[0, 1, 129, 250, 400], softcap=10.0,
         alibi_slopes=geometric_slopes(2))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [1, 100, 128, 129, 300, 513])
@pytest.mark.parametrize("causal", [False, True])
def test_shapes_and_ragged_tails(D, S, causal):
    case(1, 2, 2, S, S, D, seed=200 + S, causal=causal)


@pytest.mark.parametrize("heads", [(4, 1), (4, 2), (6, 3)])
def test_grouped_heads_sum_over_group(heads):
    case(2, heads[0], heads[1], 400, 400, 128, seed=9, causal=True)


@pytest.mark.parametrize("window", [(50, 0), (100, 100), (-1, 30)])
def test_sliding_window(window):
    case(1, 2, 2, 500, 500, 128, seed=10, window=window)


@pytest.mark.parametrize("docs", [[0, 200, 201, 600], [0, 130, 390, 600]])
def test_document_mask(docs):
    case(1, 4, 2, 600, 600, 128, seed=11, docs=docs, causal=True)


@pytest.mark.parametrize("Sq,Sk", [(300, 700), (700, 300), (129, 1000)])
def test_unequal_lengths(Sq, Sk):
    case(1, 2, 2, Sq, Sk, 128, seed=12, causal=True)


def test_outputs_fully_written_and_deterministic():
    t = make_tensors(1, 4, 2, 333, 333, 128, seed=13, with_dout=True)
    q, k, v, dout = (t[n].to(DEV) for n in ("q", "k", "v", "dout"))
    o, lse = attn.attention(q, k, v, causal=True)
    dq = torch.full(q.shape, float("nan"), device=DEV)
    dk = torch.full(k.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    dv = torch.full(v.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = torch.full((attn.bwd_workspace_size(1, 4, 2, 333, 333, 128),), 255, dtype=torch.uint8,
                    device=DEV)
    attn.attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, ws, scale=1 / math.sqrt(128), causal=True)
    torch.cuda.synchronize()
    assert not (torch.isnan(dq).any() or torch.isnan(dk).any() or torch.isnan(dv).any())
    dq2, dk2, dv2 = attn.attention_backward(q, k, v, o, lse, dout, causal=True)
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)


def test_full_size_causal_backward_workload():
    """The causal S=4096 backward workload at full size, every element
    compared with the oracle."""
    w = WORKLOADS["causal_bwd_s4096"]
    t = make_inputs(w)
    got = gpu_grads(t, scale=w.scale, causal=w.causal)
    dq, dk, dv, _, _ = oracle.attn_bwd(t["q"], t["k"], t["v"], t["dout"], scale=w.scale,
                                       causal=w.causal)
    check_grads(got, (dq, dk, dv), w.name)


@pytest.mark.parametrize("case_kw", [dict(window=(64, 16)), dict(docs=[0, 1, 100, 333, 400]),
                                     dict(causal=True, window=(200, 0))])
def test_head_dim_64_masks(case_kw):
    kw = dict(case_kw)
    case(1, 4, 2, 400, 400, 64, seed=311, causal=kw.pop("causal", kw.get("docs") is not None),
         **kw)
