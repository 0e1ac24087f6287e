"""GPU parity of the attention forward against the fp64 oracle.

Every case runs the CUDA path through the C ABI and compares, element by
element, with the oracle on the same seeded bf16 inputs.  Tolerances (fixed
for this operation): O max-abs error <= 2e-2 and mean-abs error <= 2e-3;
LSE abs error <= 1e-3; rows with no allowed key must give O = 0 and
LSE = -inf exactly.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_blackwell_b200 import attn, build
from tiled_attention_blackwell_b200.workloads import WORKLOADS, make_inputs, make_tensors

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    attn.lib()
    yield
    assert attn.device_status() == attn.ATTN_OK


def run_gpu(t, *, causal=False, window=None, doc_offsets=None, scale=None, options=None):
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    docs = None if doc_offsets is None else torch.as_tensor(doc_offsets, dtype=torch.int32,
                                                             device=DEV)
    o, lse = attn.attention(q, k, v, scale=scale, causal=causal, window=window,
                            doc_offsets=docs, options=options)
    torch.cuda.synchronize()
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def check(o, lse, o_ref, lse_ref, what=""):
    assert not np.isnan(o).any(), f"{what}: NaN in O"
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: -inf rows differ"
    err = np.abs(o - o_ref)
    assert err.max() <= O_MAX, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: O mean-abs {err.mean():.3e}"
    lse_err = np.abs(np.where(empty, 0.0, lse) - np.where(empty, 0.0, lse_ref))
    assert lse_err.max() <= LSE_TOL, f"{what}: LSE abs {lse_err.max():.3e}"
    if empty.any():
        # rows with no key: O exactly zero (LSE layout [B,H,S] vs O [B,S,H,D])
        b, h, i = np.nonzero(empty)
        assert np.all(o[b, i, h] == 0.0), f"{what}: empty rows not zero"


def full_case(B, Hq, Hkv, Sq, Sk, D, seed, *, causal=False, window=None, doc_offsets=None,
              options=None, qk_std=1.0, outliers=0.0):
    t = make_tensors(B, Hq, Hkv, Sq, Sk, D, seed, qk_std=qk_std, k_outlier_frac=outliers)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_gpu(t, causal=causal, window=window, doc_offsets=doc_offsets, scale=scale,
                     options=options)
    o_ref, lse_ref = oracle.attn_fwd(t["q"], t["k"], t["v"], scale=scale, causal=causal,
                                     window=window, doc_offsets=doc_offsets)
    check(o, lse, o_ref, lse_ref, f"B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} D{D}")


# ------------------------------------------------------------------ configs

def test_tiny_d64_workload_full():
    w = WORKLOADS["tiny_d64"]
    t = make_inputs(w)
    o, lse = run_gpu(t, causal=w.causal, scale=w.scale)
    o_ref, lse_ref = oracle.attn_fwd(t["q"], t["k"], t["v"], scale=w.scale, causal=w.causal)
    check(o, lse, o_ref, lse_ref, "tiny_d64")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [1, 5, 127, 128, 129, 255, 256, 257, 700])
@pytest.mark.parametrize("causal", [False, True])
def test_shapes_and_ragged_tails(D, S, causal):
    full_case(2, 2, 2, S, S, D, seed=100 + S, causal=causal)


@pytest.mark.parametrize("heads", [(4, 1), (4, 2), (6, 3), (8, 8)])
@pytest.mark.parametrize("D", [64, 128])
def test_grouped_heads(heads, D):
    full_case(2, heads[0], heads[1], 520, 520, D, seed=7, causal=True)


@pytest.mark.parametrize("window", [(0, 0), (37, 50), (100, 0), (300, -1), (-1, 90), (5, 400)])
def test_sliding_window(window):
    full_case(1, 2, 2, 900, 900, 128, seed=11, window=window)
    full_case(1, 2, 1, 600, 600, 64, seed=12, window=window, causal=True)


@pytest.mark.parametrize("docs", [[0, 700], [0, 1, 2, 300, 301, 700], [0, 128, 256, 640, 700],
                                  [0, 97, 400, 401, 555, 700]])
@pytest.mark.parametrize("causal", [True, False])
def test_document_mask(docs, causal):
    full_case(2, 4, 2, 700, 700, 128, seed=13, doc_offsets=docs, causal=causal)


@pytest.mark.parametrize("Sq,Sk", [(300, 1000), (1000, 300), (1, 777), (777, 1), (129, 1025)])
@pytest.mark.parametrize("causal", [False, True])
def test_unequal_lengths_bottom_right(Sq, Sk, causal):
    full_case(1, 2, 2, Sq, Sk, 128, seed=21, causal=causal)


@pytest.mark.parametrize("tau", [0.0, 8.0, 16.0])
@pytest.mark.parametrize("exp2_mode", [0, 1, 2])
@pytest.mark.parametrize("causal", [False, True])
def test_rescale_threshold_and_exp2_split(tau, exp2_mode, causal):
    opts = attn.default_options(rescale_threshold=tau, exp2_mode=exp2_mode)
    full_case(2, 2, 2, 1000, 1000, 128, seed=31, causal=causal, options=opts, qk_std=1.5,
              outliers=0.01)


def test_large_logits_stay_finite():
    """Logits far from zero (|s| up to hundreds) must not overflow or underflow."""
    t = make_tensors(1, 2, 2, 600, 600, 128, seed=41, qk_std=4.0)
    for exp2_mode in (0, 2):
        opts = attn.default_options(exp2_mode=exp2_mode)
        o, lse = run_gpu(t, causal=True, scale=1 / math.sqrt(128), options=opts)
        o_ref, lse_ref = oracle.attn_fwd(t["q"], t["k"], t["v"], scale=1 / math.sqrt(128),
                                         causal=True)
        check(o, lse, o_ref, lse_ref, f"large logits exp2_mode={exp2_mode}")


# ---------------------------------------------------------- score modifiers

def geometric_slopes(H):
    """Per-head ALiBi slopes 2^(-8 (h+1) / H) as fp32 (an input, like Q)."""
    return np.float32(2.0) ** (-8.0 * np.arange(1, H + 1, dtype=np.float32) / H)


def modifier_case(B, Hq, Hkv, Sq, Sk, D, seed, *, softcap=None, alibi=False, causal=False,
                  window=None, doc_offsets=None, qk_std=1.0):
    t = make_tensors(B, Hq, Hkv, Sq, Sk, D, seed, qk_std=qk_std)
    scale = 1.0 / math.sqrt(D)
    slopes = geometric_slopes(Hq) if alibi else None
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    docs = None if doc_offsets is None else torch.as_tensor(doc_offsets, dtype=torch.int32,
                                                             device=DEV)
    o, lse = attn.attention(q, k, v, scale=scale, causal=causal, window=window, doc_offsets=docs,
                            softcap=softcap,
                            alibi_slopes=None if slopes is None else torch.from_numpy(slopes).to(DEV))
    torch.cuda.synchronize()
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    o_ref, lse_ref = oracle.attn_fwd(t["q"], t["k"], t["v"], scale=scale, causal=causal,
                                     window=window, doc_offsets=doc_offsets,
                                     softcap=softcap or 0.0, alibi_slopes=slopes)
    check(o, lse, o_ref, lse_ref, f"softcap={softcap} alibi={alibi} causal={causal} D{D}")


@pytest.mark.parametrize("softcap", [2.0, 5.0, 30.0])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_softcap(softcap, D, causal):
    # qk_std 2 gives scaled scores of std ~4, so a cap of 2 or 5 is active.
    modifier_case(2, 2, 2, 700, 700, D, seed=71, softcap=softcap, causal=causal, qk_std=2.0)


@pytest.mark.parametrize("Sq,Sk", [(700, 700), (300, 1000), (1000, 300), (1, 515)])
@pytest.mark.parametrize("causal", [False, True])
def test_alibi(Sq, Sk, causal):
    modifier_case(1, 8, 8, Sq, Sk, 128, seed=72, alibi=True, causal=causal)


@pytest.mark.parametrize("D", [64, 128])
def test_softcap_and_alibi_with_gqa_window_and_documents(D):
    modifier_case(2, 8, 2, 900, 900, D, seed=73, softcap=8.0, alibi=True, causal=True,
                  qk_std=1.5)
    modifier_case(1, 4, 2, 900, 900, D, seed=74, softcap=8.0, alibi=True, window=(200, 50))
    modifier_case(1, 4, 1, 700, 700, D, seed=75, softcap=20.0, alibi=True, causal=True,
                  doc_offsets=[0, 1, 130, 400, 700])


def test_modifier_options_struct_path():
    """The same modifiers given through the options struct instead of the
    keyword arguments."""
    t = make_tensors(1, 4, 4, 333, 333, 128, seed=76, qk_std=2.0)
    slopes = torch.from_numpy(geometric_slopes(4)).to(DEV)
    opts = attn.default_options(softcap=6.0, alibi_slopes=slopes.data_ptr())
    o, lse = run_gpu(t, causal=True, scale=1 / math.sqrt(128), options=opts)
    o_ref, lse_ref = oracle.attn_fwd(t["q"], t["k"], t["v"], scale=1 / math.sqrt(128),
                                     causal=True, softcap=6.0,
                                     alibi_slopes=geometric_slopes(4))
    check(o, lse, o_ref, lse_ref, "options struct")


# -------------------------------------------------------- memory discipline

def test_writes_stay_in_bounds_and_cover_every_row():
    B, H, S, D = 2, 3, 333, 128
    t = make_tensors(B, H, H, S, S, D, seed=51)
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    n_o, n_l, guard = B * S * H * D, B * H * S, 4096
    o_buf = torch.full((n_o + guard,), float("nan"), dtype=torch.bfloat16, device=DEV)
    l_buf = torch.full((n_l + guard,), float("nan"), dtype=torch.float32, device=DEV)
    o = o_buf[:n_o].view(B, S, H, D)
    lse = l_buf[:n_l].view(B, H, S)
    attn.attn_fwd(q, k, v, o, lse, scale=0.1, causal=True)
    torch.cuda.synchronize()
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    assert torch.isnan(o_buf[n_o:]).all() and torch.isnan(l_buf[n_l:]).all()


def test_deterministic_and_stream_aware():
    t = make_tensors(1, 4, 2, 1000, 1000, 128, seed=61)
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    o1, l1 = attn.attention(q, k, v, causal=True)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o2, l2 = attn.attention(q, k, v, causal=True, stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ---------------------------------------------- full-size workloads (full)

@pytest.mark.parametrize("name", ["outlier_s4096", "causal_s8192", "gqa_doc_s16384",
                                  "causal_bwd_s4096", "window_s16384"])
def test_full_size_workload_full(name):
    """The benchmark's workloads at full size, in the benchmark's launch
    configuration, compared with the oracle on every element of O and LSE:
    max-abs and mean-abs over the whole tensor (every row here has at least
    one key)."""
    w = WORKLOADS[name]
    t = make_inputs(w)
    window = None if tuple(w.window) == (-1, -1) else w.window
    o, lse = run_gpu(t, causal=w.causal, window=window, doc_offsets=t["doc_offsets"],
                     scale=w.scale)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    o_ref, lse_ref = oracle.attn_fwd(t["q"], t["k"], t["v"], scale=w.scale, causal=w.causal,
                                     window=window, doc_offsets=t["doc_offsets"])
    check(o, lse, o_ref, lse_ref, name)


# ----------------------------------------------------------- failure path

def test_device_wait_timeout_is_reported_and_recoverable():
    """A wait that runs out (the first CTA withholds a key copy, nothing
    faults) makes the call report ATTN_ERR_DEVICE_TIMEOUT through the status
    word; reading clears it, and the device keeps computing correct results."""
    t = make_tensors(1, 2, 2, 512, 512, 128, seed=81)
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    opts = attn.default_options(wait_timeout_us=20000, debug_withhold_kv=1)
    attn.attention(q, k, v, causal=True, options=opts)
    assert attn.device_status() == attn.ATTN_ERR_DEVICE_TIMEOUT
    assert attn.device_status() == attn.ATTN_OK
    o, lse = run_gpu(t, causal=True, scale=1 / math.sqrt(128))
    o_ref, lse_ref = oracle.attn_fwd(t["q"], t["k"], t["v"], scale=1 / math.sqrt(128),
                                     causal=True)
    check(o, lse, o_ref, lse_ref, "after a timeout")


# ------------------------------------------------------------ maximum sizes

def test_large_tensors_need_64bit_offsets():
    """O with 2^31 elements (B=1, S=65536, Hq=256, Hkv=4, D=128, causal): every
    row's output and LSE offsets past 2^31 must land where they belong.
    Inputs are seeded normals drawn on the device (the host copy for the
    oracle is taken from the same tensors); rows sampled near the end of the
    sequence and the last heads are checked against the oracle."""
    B, S, Hq, Hkv, D = 1, 65536, 256, 4, 128
    need = (2 * B * S * Hq * D + 2 * B * S * Hkv * D) * 2 + B * Hq * S * 4
    free, _ = torch.cuda.mem_get_info()
    if free < need + (4 << 30):
        pytest.skip("not enough device memory for the 2^31-element case")
    g = torch.Generator(device=DEV).manual_seed(91)
    q = torch.randn((B, S, Hq, D), generator=g, device=DEV, dtype=torch.bfloat16)
    k = torch.randn((B, S, Hkv, D), generator=g, device=DEV, dtype=torch.bfloat16)
    v = torch.randn((B, S, Hkv, D), generator=g, device=DEV, dtype=torch.bfloat16)
    scale = 1.0 / math.sqrt(D)
    o, lse = attn.attention(q, k, v, scale=scale, causal=True)
    torch.cuda.synchronize()
    assert attn.device_status() == attn.ATTN_OK
    rows = np.array([(0, h, i) for h in (0, 1, Hq - 2, Hq - 1)
                     for i in (0, 1, 127, 128, S // 2, S - 129, S - 2, S - 1)], dtype=np.int64)
    # the element offset of the last row's output is beyond 2^31
    assert ((S - 1) * Hq + Hq - 1) * D >= 2 ** 31 - D
    o_ref, lse_ref = oracle.attn_fwd(q.cpu(), k.cpu(), v.cpu(), scale=scale, causal=True,
                                     rows=rows)
    o_s = o[rows[:, 0], rows[:, 2], rows[:, 1]].float().cpu().numpy().astype(np.float64)
    lse_s = lse[rows[:, 0], rows[:, 1], rows[:, 2]].cpu().numpy().astype(np.float64)
    err = np.abs(o_s - o_ref)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN, (err.max(), err.mean())
    assert np.abs(lse_s - lse_ref).max() <= LSE_TOL
    # and the whole output is finite (nothing left unwritten or NaN)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


def test_forward_and_backward_replay_in_a_cuda_graph():
    """The entry points only enqueue work on the given stream, so a CUDA graph
    captured around them replays the same results as eager calls."""
    t = make_tensors(1, 4, 2, 700, 700, 128, seed=95, with_dout=True)
    q, k, v, do = (t[n].to(DEV) for n in ("q", "k", "v", "dout"))
    o = torch.empty_like(q)
    lse = torch.empty((1, 4, 700), dtype=torch.float32, device=DEV)
    dq = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(attn.bwd_workspace_size(1, 4, 2, 700, 700, 128), dtype=torch.uint8,
                     device=DEV)

    def run(stream):
        attn.attn_fwd(q, k, v, o, lse, scale=0.1, causal=True, stream=stream)
        attn.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, scale=0.1, causal=True,
                      stream=stream)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        run(s)                      # eager: reference results
    s.synchronize()
    ref = [x.clone() for x in (o, lse, dq, dk, dv)]
    for x in (o, lse, dq, dk, dv):
        x.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run(s)
    for x in (o, lse, dq, dk, dv):
        x.zero_()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    for got, want in zip((o, lse, dq, dk, dv), ref):
        assert torch.equal(got, want)
    assert attn.device_status() == attn.ATTN_OK


@pytest.mark.parametrize("Sq,Sk,window", [(1, 65536, None), (3, 70001, (4000, -1)),
                                          (130, 65536, (1000, 0))])
def test_decode_like_rows_against_long_key_sequences(Sq, Sk, window):
    """Few query rows (bottom-right aligned) against tens of thousands of keys:
    hundreds of key blocks per tile, ragged key tail."""
    full_case(1, 4, 2, Sq, Sk, 128, seed=97, causal=True, window=window)
