"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: a worked
example derived by hand, closed forms, invariants of the softmax, textbook
library routines on the dense masked score matrix, and finite differences
for the backward.  Chosen so that a dropped term, a wrong sign, a wrong index
or a transposed operand in the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from tiled_attention_blackwell_b200.workloads import draw_doc_offsets, make_tensors

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def randn(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


# ----------------------------------------------------------------- helpers

def dense_mask(Sq, Sk, causal=False, window=(-1, -1), doc_offsets=None):
    """Boolean [Sq, Sk] allowed-matrix built from triangular/block matrices
    (a different construction from the oracle's per-pair predicate)."""
    m = np.ones((Sq, Sk), dtype=bool)
    off = Sk - Sq
    if causal:
        m &= np.tril(np.ones((Sq, Sk), dtype=bool), k=off)
    wl, wr = window
    if wl >= 0:
        m &= np.triu(np.ones((Sq, Sk), dtype=bool), k=off - wl)
    if wr >= 0:
        m &= np.tril(np.ones((Sq, Sk), dtype=bool), k=off + wr)
    if doc_offsets is not None:
        lengths = np.diff(doc_offsets)
        ids = np.repeat(np.arange(len(lengths)), lengths)
        m &= ids[:, None] == ids[None, :]
    return m


def dense_reference(q, k, v, scale, mask):
    """scipy softmax / logsumexp over the dense masked score matrix."""
    B, Sq, Hq, D = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            s = scale * q[b, :, h, :] @ k[b, :, h // g, :].T
            s = np.where(mask, s, -np.inf)
            lse[b, h] = scipy.special.logsumexp(s, axis=1)
            p = scipy.special.softmax(s, axis=1)
            o[b, :, h, :] = p @ v[b, :, h // g, :]
    return o, lse


# ------------------------------------------------------------ worked example

def test_golden_two_keys():
    rows = np.loadtxt(os.path.join(GOLDEN, "two_keys_logistic.txt"))
    q = np.array([[1.0, 0.0], [-2.0, 0.0]]).reshape(1, 2, 1, 2)
    k = np.array([[0.0, 0.0], [1.0, 0.0]]).reshape(1, 2, 1, 2)
    v = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    o, lse = oracle.attn_fwd(q, k, v, scale=1.0)
    for r in rows:
        i = int(r[0])
        np.testing.assert_allclose(o[0, i, 0], r[1:3], rtol=0, atol=1e-15)
        assert abs(lse[0, 0, i] - r[3]) < 1e-15


# -------------------------------------------------------------- closed forms

@pytest.mark.parametrize("mode", ["none", "causal", "window", "doc", "gqa_causal"])
def test_equal_logits_give_mean_of_allowed_v(mode):
    """Q = 0 makes every allowed logit equal: O = mean of the allowed V rows,
    LSE = log(number of allowed keys)."""
    B, S, D = 2, 37, 8
    Hq, Hkv = (4, 2) if mode == "gqa_causal" else (2, 2)
    q = np.zeros((B, S, Hq, D))
    k = randn(B, S, Hkv, D)
    v = randn(B, S, Hkv, D)
    causal = mode in ("causal", "gqa_causal", "doc")
    window = (5, 0) if mode == "window" else None
    offs = np.array([0, 10, 11, 30, 37]) if mode == "doc" else None
    o, lse = oracle.attn_fwd(q, k, v, scale=0.3, causal=causal, window=window,
                             doc_offsets=offs)
    g = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            vv = v[b, :, h // g, :]
            for i in range(S):
                if mode == "none":
                    lo, hi = 0, S
                elif mode == "window":
                    lo, hi = max(0, i - 5), i + 1
                elif mode == "doc":
                    d = np.searchsorted(offs, i, side="right") - 1
                    lo, hi = offs[d], i + 1
                else:
                    lo, hi = 0, i + 1
                np.testing.assert_allclose(o[b, i, h], vv[lo:hi].mean(axis=0), atol=1e-13)
                assert abs(lse[b, h, i] - math.log(hi - lo)) < 1e-13


def test_one_dominant_logit_selects_its_v_row():
    """One logit +30 above all others (all others 0): O is that V row up to
    (n-1) e^-30 relative weight; LSE = 30 + log(1 + (n-1) e^-30)."""
    n, D = 50, 4
    q = np.zeros((1, 3, 1, D))
    q[..., 0] = 1.0
    k = np.zeros((1, n, 1, D))
    k[0, :, 0, 1:] = randn(n, D - 1)  # orthogonal to q: logit 0
    star = 17
    k[0, star, 0, 0] = 30.0
    v = randn(1, n, 1, D)
    o, lse = oracle.attn_fwd(q, k, v, scale=1.0)
    w = (n - 1) * math.exp(-30.0)
    for i in range(3):
        err = np.abs(o[0, i, 0] - v[0, star, 0]).max()
        assert err <= 2 * w * np.abs(v).max() + 1e-15
        assert abs(lse[0, 0, i] - (30.0 + math.log1p(w))) < 1e-13


@pytest.mark.parametrize("causal,window,docs", [(False, None, None), (True, None, None),
                                                (False, (3, 4), None),
                                                (True, None, [0, 6, 20, 21, 40])])
def test_rows_of_p_sum_to_one(causal, window, docs):
    """With every V row equal to c, O = (sum_j P_ij) c must equal c."""
    B, S, H, D = 1, 40, 3, 6
    q, k = randn(B, S, H, D, scale=2.0), randn(B, S, H, D, scale=2.0)
    c = randn(D)
    v = np.broadcast_to(c, (B, S, H, D)).copy()
    o, _ = oracle.attn_fwd(q, k, v, scale=0.7, causal=causal, window=window,
                           doc_offsets=docs)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), atol=1e-13)


def test_causal_row_zero_is_v0():
    B, S, H, D = 2, 16, 2, 8
    q, k, v = randn(B, S, H, D), randn(B, S, H, D), randn(B, S, H, D)
    o, lse = oracle.attn_fwd(q, k, v, scale=0.25, causal=True)
    np.testing.assert_array_equal(o[:, 0], v[:, 0])
    for b in range(B):
        for h in range(H):
            assert abs(lse[b, h, 0] - 0.25 * q[b, 0, h] @ k[b, 0, h]) < 1e-14


def test_fully_masked_row_is_zero_and_minus_inf():
    """Sq > Sk with a causal (bottom-right) mask leaves the first rows empty."""
    q, k, v = randn(1, 6, 1, 4), randn(1, 3, 1, 4), randn(1, 3, 1, 4)
    o, lse = oracle.attn_fwd(q, k, v, scale=1.0, causal=True)
    assert np.all(o[0, :3] == 0.0) and np.all(np.isneginf(lse[0, 0, :3]))
    assert np.all(np.isfinite(lse[0, 0, 3:]))


# ----------------------------------------------- textbook library routines

@pytest.mark.parametrize("case", [
    dict(causal=False), dict(causal=True), dict(causal=False, window=(4, 2)),
    dict(causal=True, window=(7, -1)), dict(causal=True, docs=[0, 9, 10, 31, 45]),
    dict(causal=False, docs=[0, 20, 45]), dict(causal=True, Sq=30),
])
def test_matches_scipy_softmax_on_dense_scores(case):
    B, Sk, Hq, Hkv, D = 2, 45, 4, 2, 16
    Sq = case.get("Sq", Sk)
    q, k, v = randn(B, Sq, Hq, D), randn(B, Sk, Hkv, D), randn(B, Sk, Hkv, D)
    window = case.get("window", (-1, -1))
    docs = case.get("docs")
    mask = dense_mask(Sq, Sk, case["causal"], window,
                      None if docs is None else np.array(docs))
    ref_o, ref_lse = dense_reference(q, k, v, 0.2, mask)
    o, lse = oracle.attn_fwd(q, k, v, scale=0.2, causal=case["causal"],
                             window=None if window == (-1, -1) else window,
                             doc_offsets=docs)
    np.testing.assert_allclose(o, ref_o, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12)


def test_matches_torch_sdpa_float64():
    B, S, H, D = 2, 33, 3, 8
    q, k, v = randn(B, S, H, D), randn(B, S, H, D), randn(B, S, H, D)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                           scale=0.4)
    o, _ = oracle.attn_fwd(q, k, v, scale=0.4, causal=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12)


def test_row_subset_matches_full():
    B, S, Hq, Hkv, D = 2, 50, 4, 2, 8
    q, k, v = randn(B, S, Hq, D), randn(B, S, Hkv, D), randn(B, S, Hkv, D)
    o, lse = oracle.attn_fwd(q, k, v, scale=0.3, causal=True)
    rows = np.array([[1, 3, 49], [0, 0, 0], [1, 1, 17], [0, 2, 33]])
    o_r, lse_r = oracle.attn_fwd(q, k, v, scale=0.3, causal=True, rows=rows)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(o_r[n], o[b, i, h])
        assert lse_r[n] == lse[b, h, i]


def test_bf16_inputs_convert_exactly():
    t = make_tensors(1, 2, 2, 40, 40, 16, seed=9)
    o_bf, lse_bf = oracle.attn_fwd(t["q"], t["k"], t["v"], scale=0.25, causal=True)
    f = [t[n].to(torch.float64).numpy() for n in ("q", "k", "v")]
    o64, lse64 = oracle.attn_fwd(*f, scale=0.25, causal=True)
    np.testing.assert_array_equal(o_bf, o64)
    np.testing.assert_array_equal(lse_bf, lse64)


# ----------------------------------------------------------------- invariants

def test_document_mask_is_concatenated_causal_runs():
    S, D = 64, 8
    offs = np.array([0, 7, 8, 40, 64])
    q, k, v = randn(1, S, 2, D), randn(1, S, 2, D), randn(1, S, 2, D)
    o, lse = oracle.attn_fwd(q, k, v, scale=0.5, causal=True, doc_offsets=offs)
    for a, b in zip(offs[:-1], offs[1:]):
        o_d, lse_d = oracle.attn_fwd(q[:, a:b], k[:, a:b], v[:, a:b], scale=0.5, causal=True)
        np.testing.assert_array_equal(o[:, a:b], o_d)
        np.testing.assert_array_equal(lse[:, :, a:b], lse_d)


def test_window_covering_everything_is_causal():
    S = 29
    q, k, v = randn(1, S, 2, 8), randn(1, S, 2, 8), randn(1, S, 2, 8)
    o1, l1 = oracle.attn_fwd(q, k, v, scale=0.5, causal=True)
    o2, l2 = oracle.attn_fwd(q, k, v, scale=0.5, window=(S, 0))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_gqa_equals_mha_with_repeated_kv():
    B, S, Hq, Hkv, D = 1, 30, 6, 2, 8
    q, k, v = randn(B, S, Hq, D), randn(B, S, Hkv, D), randn(B, S, Hkv, D)
    o1, l1 = oracle.attn_fwd(q, k, v, scale=0.5, causal=True)
    rep = Hq // Hkv
    o2, l2 = oracle.attn_fwd(q, np.repeat(k, rep, axis=2), np.repeat(v, rep, axis=2),
                             scale=0.5, causal=True)
    np.testing.assert_allclose(o1, o2, atol=1e-15)
    np.testing.assert_allclose(l1, l2, atol=1e-15)


def test_noncausal_invariant_to_joint_kv_permutation():
    q, k, v = randn(1, 20, 2, 8), randn(1, 31, 2, 8), randn(1, 31, 2, 8)
    perm = rng.permutation(31)
    o1, l1 = oracle.attn_fwd(q, k, v, scale=0.5)
    o2, l2 = oracle.attn_fwd(q, k[:, perm], v[:, perm], scale=0.5)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_doc_offsets_generator_rules():
    offs = draw_doc_offsets(16384, 4)
    lengths = np.diff(offs)
    assert offs[0] == 0 and offs[-1] == 16384
    assert np.all(lengths[:-1] >= 512) and np.all(lengths <= 4096) and lengths[-1] >= 1


# ------------------------------------------------------------------ backward

def _loss(q, k, v, dout, **kw):
    o, _ = oracle.attn_fwd(q, k, v, **kw)
    return float(np.sum(o * dout))


@pytest.mark.parametrize("kw", [dict(causal=False), dict(causal=True),
                                dict(causal=True, doc_offsets=[0, 3, 7]),
                                dict(causal=False, window=(2, 1))])
@pytest.mark.parametrize("heads", [(2, 2), (2, 1)])
def test_backward_matches_central_differences(kw, heads):
    B, S, D = 1, 7, 3
    Hq, Hkv = heads
    q, k, v = randn(B, S, Hq, D), randn(B, S, Hkv, D), randn(B, S, Hkv, D)
    dout = randn(B, S, Hq, D)
    kw = dict(kw, scale=0.8)
    dq, dk, dv, o, lse = oracle.attn_bwd(q, k, v, dout, **kw)
    o_f, lse_f = oracle.attn_fwd(q, k, v, **kw)
    np.testing.assert_allclose(o, o_f, atol=1e-15)
    np.testing.assert_allclose(lse, lse_f, atol=1e-15)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            lp = _loss(**{**args, name: xp}, dout=dout, **kw)
            lm = _loss(**{**args, name: xm}, dout=dout, **kw)
            fd[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, fd, atol=2e-8, rtol=1e-6, err_msg=name)


def test_backward_dk_sums_to_zero_over_keys():
    """Adding one vector to every key shifts a row's logits by a constant, so
    the softmax gradient rows sum to zero and sum_j dK_j = 0."""
    q, k, v, dout = randn(2, 24, 4, 8), randn(2, 24, 2, 8), randn(2, 24, 2, 8), randn(2, 24, 4, 8)
    for kw in (dict(causal=True), dict(causal=False), dict(causal=True, doc_offsets=[0, 5, 24])):
        _, dk, _, _, _ = oracle.attn_bwd(q, k, v, dout, scale=0.4, **kw)
        np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)


def test_backward_matches_torch_autograd_float64():
    B, S, Hq, Hkv, D = 1, 19, 4, 2, 8
    q, k, v, dout = randn(B, S, Hq, D), randn(B, S, Hkv, D), randn(B, S, Hkv, D), randn(B, S, Hq, D)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3).requires_grad_() for x in (q, k, v))
    rep = Hq // Hkv
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(rep, dim=1), tv.repeat_interleave(rep, dim=1),
        is_causal=True, scale=0.3)
    out.backward(torch.from_numpy(dout).permute(0, 2, 1, 3))
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, dout, scale=0.3, causal=True)
    np.testing.assert_allclose(dq, tq.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)


# ------------------------------------------- score modifiers (soft-cap, ALiBi)

def test_alibi_equal_logits_give_geometric_weights():
    """Q = 0 and a causal mask leave only the ALiBi bias -m (i - j): weights
    r^(i-j) / sum_t r^t with r = e^-m, so LSE_i = log((1 - r^(i+1)) / (1 - r))."""
    S, D, m = 23, 4, 0.37
    q = np.zeros((1, S, 2, D))
    k, v = randn(1, S, 1, D), randn(1, S, 1, D)
    slopes = [m, 2 * m]
    o, lse = oracle.attn_fwd(q, k, v, scale=0.5, causal=True, alibi_slopes=slopes)
    for h, mh in enumerate(slopes):
        r = math.exp(-mh)
        for i in range(S):
            w = r ** (i - np.arange(i + 1))
            np.testing.assert_allclose(o[0, i, h], (w[:, None] * v[0, :i + 1, 0]).sum(0) / w.sum(),
                                       atol=1e-13)
            assert abs(lse[0, h, i] - math.log((1 - r ** (i + 1)) / (1 - r))) < 1e-12


def test_softcap_two_keys_is_logistic_of_capped_gap():
    """Two keys with scaled scores 0 and a: the cap maps a to c tanh(a / c),
    so the weights are the logistic function of that value."""
    c, a = 2.5, 4.0
    q = np.array([[a, 0.0]]).reshape(1, 1, 1, 2)
    k = np.array([[0.0, 0.0], [1.0, 0.0]]).reshape(1, 2, 1, 2)
    v = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    o, lse = oracle.attn_fwd(q, k, v, scale=1.0, softcap=c)
    z = c * math.tanh(a / c)
    np.testing.assert_allclose(o[0, 0, 0], [1 / (1 + math.exp(z)), math.exp(z) / (1 + math.exp(z))],
                               atol=1e-15)
    assert abs(lse[0, 0, 0] - math.log1p(math.exp(z))) < 1e-14


def test_huge_softcap_is_no_softcap():
    q, k, v = randn(1, 30, 2, 8), randn(1, 30, 2, 8), randn(1, 30, 2, 8)
    o1, l1 = oracle.attn_fwd(q, k, v, scale=0.3, causal=True)
    o2, l2 = oracle.attn_fwd(q, k, v, scale=0.3, causal=True, softcap=1e9)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


@pytest.mark.parametrize("causal,Sq", [(True, 40), (False, 40), (True, 25)])
def test_modifiers_match_scipy_on_dense_scores(causal, Sq):
    B, Sk, Hq, Hkv, D = 1, 40, 4, 2, 8
    q, k, v = randn(B, Sq, Hq, D, scale=3.0), randn(B, Sk, Hkv, D, scale=3.0), randn(B, Sk, Hkv, D)
    cap, slopes = 3.0, np.array([0.5, 0.25, 0.125, 0.0625])
    mask = dense_mask(Sq, Sk, causal)
    dist = np.abs(np.arange(Sq)[:, None] + (Sk - Sq) - np.arange(Sk)[None, :])
    o_ref = np.zeros_like(q)
    lse_ref = np.zeros((B, Hq, Sq))
    g = Hq // Hkv
    for h in range(Hq):
        s = 0.4 * q[0, :, h, :] @ k[0, :, h // g, :].T
        s = cap * np.tanh(s / cap) - slopes[h] * dist
        s = np.where(mask, s, -np.inf)
        lse_ref[0, h] = scipy.special.logsumexp(s, axis=1)
        o_ref[0, :, h, :] = scipy.special.softmax(s, axis=1) @ v[0, :, h // g, :]
    o, lse = oracle.attn_fwd(q, k, v, scale=0.4, causal=causal, softcap=cap, alibi_slopes=slopes)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


@pytest.mark.parametrize("mods", [dict(softcap=1.5), dict(alibi_slopes=[0.3, 0.7]),
                                  dict(softcap=2.0, alibi_slopes=[0.2, 0.05])])
def test_backward_with_modifiers_matches_central_differences(mods):
    B, S, Hq, Hkv, D = 1, 6, 2, 1, 3
    q, k, v = randn(B, S, Hq, D, scale=2.0), randn(B, S, Hkv, D, scale=2.0), randn(B, S, Hkv, D)
    dout = randn(B, S, Hq, D)
    kw = dict(mods, scale=0.9, causal=True)
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, dout, **kw)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            fd[idx] = (_loss(**{**args, name: xp}, dout=dout, **kw) -
                       _loss(**{**args, name: xm}, dout=dout, **kw)) / (2 * h)
        np.testing.assert_allclose(g, fd, atol=2e-8, rtol=1e-6, err_msg=name)


# ------------------------------------------------------------- fp8 (e4m3) inputs

def test_e4m3_decode_matches_torch_for_every_code():
    """All 256 e4m3 codes against torch's float8_e4m3fn conversion."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_float(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    np.testing.assert_array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


@pytest.mark.parametrize("code,value", [(0x38, 1.0), (0xB8, -1.0), (0x7E, 448.0),
                                        (0x08, 2.0 ** -6), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9),
                                        (0x3C, 1.5), (0x00, 0.0)])
def test_e4m3_known_codes(code, value):
    # The format's own corner values: one, the largest finite value, the
    # smallest normal and subnormal, a mantissa step.
    assert oracle.e4m3_to_float(code) == value


def quantize_e4m3(x, amax_target=448.0):
    """Per-tensor e4m3 quantisation with torch: codes and the descale factor."""
    descale = float(x.abs().max()) / amax_target
    return (x / descale).to(torch.float8_e4m3fn), descale


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_forward_is_exact_attention_of_the_dequantized_inputs(causal):
    g = torch.Generator().manual_seed(21)
    B, S, Hq, Hkv, D = 2, 37, 4, 2, 16
    q8, qd = quantize_e4m3(torch.randn(B, S, Hq, D, generator=g) * 2)
    k8, kd = quantize_e4m3(torch.randn(B, S, Hkv, D, generator=g))
    v8, vd = quantize_e4m3(torch.randn(B, S, Hkv, D, generator=g) * 3)
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, q_descale=qd, k_descale=kd, v_descale=vd,
                                 scale=0.3, causal=causal)
    # independent dequantisation (torch's decode), then the dense scipy reference
    deq = [x.to(torch.float64).numpy() * d for x, d in ((q8, qd), (k8, kd), (v8, vd))]
    o_ref, lse_ref = dense_reference(*deq, 0.3, dense_mask(S, S, causal=causal))
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


def test_fp8_descales_act_on_their_own_tensor():
    g = torch.Generator().manual_seed(22)
    q8, _ = quantize_e4m3(torch.randn(1, 20, 2, 8, generator=g))
    k8, _ = quantize_e4m3(torch.randn(1, 20, 2, 8, generator=g))
    v8, _ = quantize_e4m3(torch.randn(1, 20, 2, 8, generator=g))
    base = oracle.attn_fwd_fp8(q8, k8, v8, q_descale=0.01, k_descale=0.02, v_descale=0.03,
                               scale=0.5)
    # V's factor scales O only; Q's and K's enter the scores as a product.
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, q_descale=0.01, k_descale=0.02, v_descale=0.09,
                                 scale=0.5)
    np.testing.assert_allclose(o, 3 * base[0], rtol=1e-13)
    np.testing.assert_allclose(lse, base[1], rtol=1e-13)
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, q_descale=0.04, k_descale=0.005, v_descale=0.03,
                                 scale=0.5)
    np.testing.assert_allclose(o, base[0], rtol=1e-12)
    np.testing.assert_allclose(lse, base[1], rtol=1e-12)
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, q_descale=0.02, k_descale=0.02, v_descale=0.03,
                                 scale=0.5)
    o2, lse2 = oracle.attn_fwd_fp8(q8, k8, v8, q_descale=0.01, k_descale=0.02, v_descale=0.03,
                                   scale=1.0)
    np.testing.assert_allclose(o, o2, rtol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=1e-12)


def test_fp8_row_subset_matches_full():
    g = torch.Generator().manual_seed(23)
    q8, qd = quantize_e4m3(torch.randn(1, 60, 2, 8, generator=g))
    k8, kd = quantize_e4m3(torch.randn(1, 60, 1, 8, generator=g))
    v8, vd = quantize_e4m3(torch.randn(1, 60, 1, 8, generator=g))
    kw = dict(q_descale=qd, k_descale=kd, v_descale=vd, scale=0.4, causal=True)
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, **kw)
    rows = np.array([[0, 1, 59], [0, 0, 3]])
    o_r, lse_r = oracle.attn_fwd_fp8(q8, k8, v8, rows=rows, **kw)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(o_r[n], o[b, i, h])
        assert lse_r[n] == lse[b, h, i]


def test_fp8_path_equals_bf16_path_on_shared_values():
    """e4m3 values are exact in bf16: with unit factors the fp8 oracle and the
    bf16 oracle see identical numbers and must agree bit for bit."""
    g = torch.Generator().manual_seed(24)
    q8, _ = quantize_e4m3(torch.randn(1, 30, 2, 16, generator=g))
    k8, _ = quantize_e4m3(torch.randn(1, 30, 2, 16, generator=g))
    v8, _ = quantize_e4m3(torch.randn(1, 30, 2, 16, generator=g))
    o8, l8 = oracle.attn_fwd_fp8(q8, k8, v8, q_descale=1.0, k_descale=1.0, v_descale=1.0,
                                 scale=0.02, causal=True)
    ob, lb = oracle.attn_fwd(q8.to(torch.bfloat16), k8.to(torch.bfloat16),
                             v8.to(torch.bfloat16), scale=0.02, causal=True)
    np.testing.assert_array_equal(o8, ob)
    np.testing.assert_array_equal(l8, lb)


def test_workload_fp8_quantization_is_within_e4m3_rounding():
    """The fp8 workload generator: descale * code reproduces the fp32 draw to
    e4m3's round-to-nearest precision (relative 2^-4 in the normal range,
    absolute half a subnormal step below it), and the largest magnitude maps
    to the largest code."""
    from tiled_attention_blackwell_b200.workloads import quantize_e4m3 as wq
    x = torch.randn(4096, generator=torch.Generator().manual_seed(25)) * 3
    codes, descale = wq(x)
    back = codes.to(torch.float64) * descale
    xs = x.to(torch.float64) / descale
    normal = xs.abs() >= 2.0 ** -6
    rel = ((back / descale - xs).abs() / xs.abs())[normal]
    assert float(rel.max()) <= 2.0 ** -4
    assert float((back / descale - xs).abs()[~normal].max()) <= 2.0 ** -10
    assert float(codes.to(torch.float32).abs().max()) == 448.0
