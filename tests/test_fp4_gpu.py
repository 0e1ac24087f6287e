"""GPU parity of the FP4 Direct-P forward against the oracle (B200).

Inputs with power-of-two NVFP4 block scales and a power-of-two score factor
make every log2 score an exact dyadic number in both fp32 (kernel) and fp64
(oracle), so the quantised decisions -- block exponents and E2M1 codes --
are the same on both sides and the comparison is element by element at the
output's own rounding: |O - O_ref| <= 2^-8 |O_ref| + 2^-20 max|V| (bf16
output, fp32 accumulation of exact products), |LSE - LSE_ref| <= 2e-5 +
1e-6 |LSE_ref|.  General NVFP4 inputs (e4m3 block scales) round the scores
in fp32 first, so a code may differ from the oracle's where a score sits
within rounding of a decision boundary; those cases are held to the
attention tolerance (O max-abs 2e-2, mean-abs 2e-3; LSE 1e-3).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_blackwell_b200 import attn
from tiled_attention_blackwell_b200.workloads import (WORKLOADS, draw_doc_offsets,
                                                      make_inputs, make_tensors_fp4)

pytestmark = pytest.mark.gpu

NAMES = ("q_codes", "q_scales", "q_global", "k_codes", "k_scales", "k_global", "v_codes",
         "v_scales", "v_global")


def _dev(t):
    return [t[n].cuda() if torch.is_tensor(t[n]) else t[n] for n in NAMES]


def _vmax(t):
    c = t["v_codes"].numpy()
    mag = np.maximum(np.abs(c & 7), np.abs((c >> 4) & 7)).max()
    return [0, 0.5, 1, 1.5, 2, 3, 4, 6][mag] * 2.0 ** (int(t["v_scales"].numpy().max()) - 127)


# The two tensor-core paths of the D = 128 forward: block-scaled FP4 products
# (the default there) and f16 products of the widened values.  D = 64 has the
# f16 path only.
MMAS = ("block_scaled", "f16")


def _mma_ok(mma, D):
    return mma != "block_scaled" or D == 128


def _run(t, classifier, mma="auto", **kw):
    o, lse = attn.attention_fp4(*_dev(t), classifier=classifier, mma=mma, **kw)
    attn.check_device_status()
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _ref(t, classifier, **kw):
    return oracle.attn_fwd_fp4(*[t[n] for n in NAMES], classifier=classifier, **kw)


def _tight(o, lse, o_ref, lse_ref, vmax):
    err = np.abs(o - o_ref)
    bound = 2.0 ** -8 * np.abs(o_ref) + 2.0 ** -20 * vmax
    bad = err > bound
    assert not bad.any(), (int(bad.sum()), float(err.max()), np.argwhere(bad)[:5])
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    lerr = np.abs(lse[fin] - lse_ref[fin])
    assert (lerr <= 2e-5 + 1e-6 * np.abs(lse_ref[fin])).all(), float(lerr.max())


CASES = [
    # B, Hq, Hkv, Sq, Sk, D, mask kwargs
    (1, 2, 2, 300, 300, 128, dict(causal=True)),
    (1, 2, 2, 300, 300, 64, dict(causal=False)),
    (2, 4, 2, 257, 383, 128, dict(causal=True)),
    (1, 2, 1, 600, 600, 128, dict(causal=True, window=(64, 0))),
    (1, 2, 2, 333, 333, 64, dict(causal=False, window=(40, 17))),
    (1, 2, 2, 1, 1000, 128, dict(causal=True)),
    (1, 1, 1, 1, 1, 64, dict(causal=False)),
    (1, 3, 3, 129, 129, 128, dict(causal=False)),
    # Sq > Sk, causal (bottom-right): the first 190 rows see no key
    (1, 2, 2, 450, 260, 128, dict(causal=True)),
    (1, 2, 1, 3, 4100, 64, dict(causal=True)),
]


@pytest.mark.parametrize("mma", MMAS)
@pytest.mark.parametrize("classifier", ["affine", "exp2"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[:6]}-{sorted(c[6].items())}")
def test_fp4_parity_exact_decisions(case, classifier, mma):
    B, Hq, Hkv, Sq, Sk, D, mask = case
    if not _mma_ok(mma, D):
        pytest.skip("block-scaled products are built for D = 128")
    scale = 1.0 / math.sqrt(D)
    t = make_tensors_fp4(B, Hq, Hkv, Sq, Sk, D, seed=11 + Sq + D, scale=scale)
    o, lse = _run(t, classifier, mma=mma, scale=scale, **mask)
    o_ref, lse_ref = _ref(t, classifier, scale=scale, **mask)
    _tight(o, lse, o_ref, lse_ref, _vmax(t))


@pytest.mark.parametrize("mma", MMAS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("classifier", ["affine", "exp2"])
def test_fp4_parity_document_mask(classifier, D, mma):
    if not _mma_ok(mma, D):
        pytest.skip("block-scaled products are built for D = 128")
    S = 700
    scale = 1.0 / math.sqrt(D)
    t = make_tensors_fp4(1, 4, 2, S, S, D, seed=21, scale=scale)
    docs = np.array([0, 100, 450, 451, 700], dtype=np.int32)
    o, lse = _run(t, classifier, mma=mma, scale=scale, causal=True,
                  doc_offsets=torch.from_numpy(docs).cuda())
    o_ref, lse_ref = _ref(t, classifier, scale=scale, causal=True, doc_offsets=docs)
    _tight(o, lse, o_ref, lse_ref, _vmax(t))


@pytest.mark.parametrize("mma", MMAS)
@pytest.mark.parametrize("tau", [0.0, 3.0, 8.0])
def test_fp4_rescale_threshold_does_not_change_the_result(tau, mma):
    # The anchor is an integer and every rescale an exact power of two: the
    # result for any threshold matches the oracle, which has no anchor.
    S, D = 520, 128
    scale = 1.0 / math.sqrt(D)
    t = make_tensors_fp4(1, 2, 2, S, S, D, seed=31, scale=scale)
    o, lse = _run(t, "affine", mma=mma, scale=scale, causal=True,
                  options=attn.fp4_options(rescale_threshold=tau))
    o_ref, lse_ref = _ref(t, "affine", scale=scale, causal=True)
    _tight(o, lse, o_ref, lse_ref, _vmax(t))


@pytest.mark.parametrize("classifier", ["affine", "exp2"])
def test_fp4_block_scaled_matches_f16_products(classifier):
    # Every product of two FP4 values is exact in fp32, so the two paths
    # differ only in the order of the fp32 accumulation: O within one bf16
    # rounding step of each other (plus accumulation noise), LSE to fp32
    # rounding.
    S, D = 900, 128
    scale = 1.0 / math.sqrt(D)
    t = make_tensors_fp4(2, 4, 2, S, S, D, seed=33, scale=scale, pow2_scales=False)
    o_bs, l_bs = _run(t, classifier, mma="block_scaled", scale=scale, causal=True)
    o_f, l_f = _run(t, classifier, mma="f16", scale=scale, causal=True)
    err = np.abs(o_bs - o_f)
    assert (err <= 2.0 ** -7 * np.abs(o_f) + 1e-6).all(), float(err.max())
    assert np.abs(l_bs - l_f).max() <= 1e-5 + 1e-6 * np.abs(l_f).max()


def drop_bounds(t, rows, scale, tau, classifier):
    """Per-row bound on what the kernel's range guard may drop.

    The kernel drops a 32-key block (aligned to the key index) whose
    maximum log2 score lies more than 26 - ceil(tau) octaves below its
    anchor, the running maximum rounded up to an integer (never above
    ceil(M), M the row maximum).  So only blocks with floor(block max) <
    ceil(M) - 26 + ceil(tau) can be dropped, and the kernel's output is the
    Direct-P output of the row without some subset of them: the weights of
    the kept blocks do not depend on the dropped ones.  With W_d / W the
    fraction of the Direct-P weight in those blocks (from the oracle's row
    function with and without them), |O - O_ref| <= 2 max|V| W_d / W and
    |LSE - LSE_ref| <= -ln(1 - W_d / W).  Returns (frac [n], vmax_row [n])."""
    q, k, v = _decode(t, "q"), _decode(t, "k"), _decode_v(t)
    Hq, Hkv = q.shape[2], k.shape[2]
    Sq, Sk = q.shape[1], k.shape[1]
    frac, vrow = np.zeros(len(rows)), np.zeros(len(rows))
    for r, (b, h, i) in enumerate(rows):
        hk = h // (Hq // Hkv)
        allow = np.arange(Sk) <= i + Sk - Sq
        if not allow.any():
            continue
        y = (k[b, :, hk] @ q[b, i, h]) * (scale * 1.4426950408889634)
        M = y[allow].max()
        ym = np.where(allow, y, -np.inf)
        nblk = (Sk + 31) // 32
        bmax = np.array([ym[32 * g:32 * g + 32].max() for g in range(nblk)])
        droppable = np.floor(bmax) < math.ceil(M) - 26 + math.ceil(tau)
        keep = allow & ~np.repeat(droppable, 32)[:Sk]
        vrow[r] = np.abs(v[b, allow, hk]).max()
        if not droppable[np.isfinite(bmax)].any():
            continue
        _, l_all = oracle.direct_p_row(y, v[b, :, hk], allow=allow, classifier=classifier)
        _, l_keep = oracle.direct_p_row(y, v[b, :, hk], allow=keep, classifier=classifier)
        frac[r] = 1.0 - math.exp(l_keep - l_all) if keep.any() else 1.0
    return frac, vrow


@pytest.mark.parametrize("mma", MMAS)
@pytest.mark.parametrize("classifier", ["affine", "exp2"])
@pytest.mark.parametrize("tau", [0.0, 8.0])
def test_fp4_wide_logits(classifier, tau, mma):
    # Score factor 2^3 instead of ~2^-3: log2 scores spread over hundreds of
    # units, so the anchor moves by large steps and many blocks sit far below
    # it (the range guard).  Element-wise parity with a per-row bound for
    # what the guard may drop (drop_bounds), at the default threshold 8 and
    # at 0.
    S, D = 400, 128
    t = make_tensors_fp4(1, 2, 2, S, S, D, seed=41, scale=8.0)
    o, lse = _run(t, classifier, mma=mma, scale=8.0, causal=True,
                  options=attn.fp4_options(rescale_threshold=tau))
    o_ref, lse_ref = _ref(t, classifier, scale=8.0, causal=True)
    assert np.abs(lse_ref).max() > 100
    rows = np.array([(0, h, i) for h in range(2) for i in range(S)])
    frac, vrow = drop_bounds(t, rows, 8.0, tau, classifier)
    assert (frac > 0).any(), "no row has a block the guard may drop: the case tests nothing"
    got = o[rows[:, 0], rows[:, 2], rows[:, 1]]
    want = o_ref[rows[:, 0], rows[:, 2], rows[:, 1]]
    bound = 2.0 ** -8 * np.abs(want) + 2.0 ** -20 * _vmax(t) + 2.0 * (frac * vrow)[:, None]
    err = np.abs(got - want)
    assert (err <= bound).all(), (float((err - bound).max()), int((err > bound).sum()))
    l_got = lse[rows[:, 0], rows[:, 1], rows[:, 2]]
    l_want = lse_ref[rows[:, 0], rows[:, 1], rows[:, 2]]
    l_bound = 2e-5 + 1e-6 * np.abs(l_want) - np.log1p(-np.minimum(frac, 1 - 1e-16))
    assert (np.abs(l_got - l_want) <= l_bound).all(), float(np.abs(l_got - l_want).max())


@pytest.mark.parametrize("mma", MMAS)
@pytest.mark.parametrize("classifier", ["affine", "exp2"])
@pytest.mark.parametrize("D", [64, 128])
def test_fp4_general_nvfp4_scales(classifier, D, mma):
    if not _mma_ok(mma, D):
        pytest.skip("block-scaled products are built for D = 128")
    S = 300
    scale = 1.0 / math.sqrt(D)
    t = make_tensors_fp4(1, 2, 2, S, S, D, seed=51, scale=scale, pow2_scales=False)
    o, lse = _run(t, classifier, mma=mma, scale=scale, causal=True)
    o_ref, lse_ref = _ref(t, classifier, scale=scale, causal=True)
    err = np.abs(o - o_ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    assert np.abs(lse - lse_ref).max() <= 1e-3


@pytest.mark.parametrize("mma", MMAS)
def test_fp4_full_size_sampled_rows(mma):
    # The benchmark's workload and launch (B2 H16 S8192 D128 causal; the
    # benchmark runs the block-scaled path), checked on sampled rows the
    # oracle computes one by one.
    w = WORKLOADS["causal_s8192_fp4"]
    t = make_inputs(w)
    rng = np.random.default_rng(5)
    rows = np.stack([rng.integers(0, w.B, 48), rng.integers(0, w.Hq, 48),
                     rng.integers(0, w.S, 48)], 1)
    rows = np.concatenate([rows, [[0, 0, 0], [1, 15, w.S - 1], [0, 3, 127], [1, 8, 128]]])
    for classifier in ("affine", "exp2"):
        o, lse = _run(t, classifier, mma=mma, scale=w.scale, causal=True)
        o_ref, lse_ref = _ref(t, classifier, scale=w.scale, causal=True, rows=rows)
        got = o[rows[:, 0], rows[:, 2], rows[:, 1]]
        got_lse = lse[rows[:, 0], rows[:, 1], rows[:, 2]]
        _tight(got, got_lse, o_ref, lse_ref, _vmax(t))


@pytest.mark.parametrize("mma,D", [("f16", 64), ("f16", 128), ("block_scaled", 128)])
def test_fp4_range_error_reported(mma, D):
    S = 64
    scale = 1.0 / math.sqrt(D)
    t = make_tensors_fp4(1, 1, 1, S, S, D, seed=61, scale=scale)
    # an out-of-range V scale under nonzero codes: reported, read as zero
    t["v_scales"] = t["v_scales"].clone()
    t["v_scales"][0, 0, 0, 0] = 200
    t["v_codes"] = t["v_codes"].clone()
    t["v_codes"][0, 0, 0, 0] = 0x11
    o, _ = attn.attention_fp4(*_dev(t), causal=True, scale=scale, mma=mma)
    assert attn.device_status() == attn.ATTN_ERR_RANGE
    assert attn.device_status() == attn.ATTN_OK  # reading clears it
    zeroed = dict(t, v_codes=t["v_codes"].clone())
    zeroed["v_codes"][0, :32, 0, 0] &= 0xF0  # column d = 0 of keys 0-31 reads as zero
    o_ref, _ = _ref(zeroed, "affine", scale=scale, causal=True)
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= 2e-2
    # the same scale under zero codes is harmless
    t["v_codes"][:, :32, 0, 0] = 0
    attn.attention_fp4(*_dev(t), causal=True, scale=scale, mma=mma)
    assert attn.device_status() == attn.ATTN_OK
    # NaN and negative NVFP4 scales under nonzero codes: reported, and the
    # output is the oracle's, which reads those blocks as zero; -0 is a zero
    # scale and reports nothing
    for bad in (0x7F, 0xB8):
        t2 = make_tensors_fp4(1, 1, 1, S, S, D, seed=62, scale=scale)
        t2["q_scales"] = t2["q_scales"].clone()
        t2["q_scales"][0, 3, 0, 1] = bad
        t2["q_codes"] = t2["q_codes"].clone()
        t2["q_codes"][0, 3, 0, 8] = 0x22
        o2, _ = attn.attention_fp4(*_dev(t2), causal=True, scale=scale, mma=mma)
        assert attn.device_status() == attn.ATTN_ERR_RANGE
        o2_ref, _ = _ref(t2, "affine", scale=scale, causal=True)
        assert np.abs(o2.float().cpu().numpy() - o2_ref).max() <= 2e-2
    t2["q_scales"][0, 3, 0, 1] = 0x80
    attn.attention_fp4(*_dev(t2), causal=True, scale=scale, mma=mma)
    assert attn.device_status() == attn.ATTN_OK


def test_fp4_cosine_against_bf16_exact():
    # Accuracy record (not parity): mean cosine similarity of the Direct-P
    # output against exact attention of the decoded inputs, on Gaussian
    # inputs with general NVFP4 scales; the page reports about 0.944 for its
    # fast path against BF16.
    S, D = 1024, 128
    scale = 1.0 / math.sqrt(D)
    t = make_tensors_fp4(1, 4, 4, S, S, D, seed=71, scale=scale, pow2_scales=False)
    q = torch.from_numpy(_decode(t, "q")).to(torch.float64)
    k = torch.from_numpy(_decode(t, "k")).to(torch.float64)
    v = torch.from_numpy(_decode_v(t)).to(torch.float64)
    ref, _ = oracle.attn_fwd(q.numpy(), k.numpy(), v.numpy(), scale=scale)
    for classifier, floor in (("affine", 0.9), ("exp2", 0.95)):
        o, _ = _run(t, classifier, scale=scale)
        a, b = o.reshape(-1, D), ref.reshape(-1, D)
        cos = (a * b).sum(1) / np.linalg.norm(a, axis=1) / np.linalg.norm(b, axis=1)
        print(f"{classifier}: mean cosine {cos.mean():.4f}")
        assert cos.mean() >= floor


def _nibbles(c):
    c = c.numpy()
    return np.stack([c & 15, c >> 4], -1).reshape(*c.shape[:-1], -1)


_E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])


def _decode(t, name):
    mag = _E2M1[_nibbles(t[name + "_codes"])]
    sc = t[name + "_scales"].view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    return t[name + "_global"] * mag * np.repeat(sc, 16, axis=-1)


def _decode_v(t):
    mag = _E2M1[_nibbles(t["v_codes"])]
    S = mag.shape[1]
    sc = np.exp2(t["v_scales"].numpy().astype(np.float64) - 127)
    return t["v_global"] * mag * np.repeat(sc, 32, axis=1)[:, :S]


def _fp4_buffers(t, scale):
    B, Sq, Hq, Dh = t["q_codes"].shape
    Sk, Hkv = t["k_codes"].shape[1], t["k_codes"].shape[2]
    D = 2 * Dh
    o = torch.empty((B, Sq, Hq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")
    ws = torch.empty(attn.fp4_workspace_size(B, Hq, Hkv, Sq, Sk, D), dtype=torch.uint8,
                     device="cuda")
    return o, lse, ws


def test_fp4_cuda_graph_replay_and_determinism():
    # The entry point only enqueues work on the caller's stream, so it can be
    # captured; replays and repeated eager calls give bit-identical results.
    S, D = 700, 128
    scale = 1.0 / math.sqrt(D)
    t = make_tensors_fp4(1, 4, 2, S, S, D, seed=81, scale=scale)
    args = _dev(t)
    o, lse, ws = _fp4_buffers(t, scale)
    attn.attn_fwd_fp4(*args, o, lse, ws, scale=scale, causal=True, classifier="exp2")
    torch.cuda.synchronize()
    o_ref, lse_ref = o.clone(), lse.clone()
    attn.attn_fwd_fp4(*args, o, lse, ws, scale=scale, causal=True, classifier="exp2")
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        o.zero_()
        lse.zero_()
        with torch.cuda.graph(g, stream=s):
            attn.attn_fwd_fp4(*args, o, lse, ws, scale=scale, causal=True, classifier="exp2",
                              stream=s)
    for _ in range(3):
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    attn.check_device_status()


def test_fp4_on_a_side_stream():
    S, D = 333, 64
    scale = 1.0 / math.sqrt(D)
    t = make_tensors_fp4(2, 2, 2, S, S, D, seed=82, scale=scale)
    args = _dev(t)
    o, lse, ws = _fp4_buffers(t, scale)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        attn.attn_fwd_fp4(*args, o, lse, ws, scale=scale, causal=False, window=(50, 20),
                          stream=s)
    s.synchronize()
    attn.check_device_status()
    o_ref, lse_ref = _ref(t, "affine", scale=scale, causal=False, window=(50, 20))
    _tight(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, _vmax(t))
