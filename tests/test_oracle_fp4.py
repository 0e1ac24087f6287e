"""Pins for the oracle's FP4 formats and Direct-P forward (CPU only).

"Hardware-Aware FP4 FlashAttention-4", "Metodología", item 1 (Direct-P)
gives no worked values, so each pin is a case whose answer follows from the
format definitions or from the method's own structure: the E2M1 table,
brute-force nearest rounding, worked constant-score rows (hand-derived
codes), exact agreement with the softmax when every score sits on the E2M1
grid, invariance under integer shifts of a row's log2 scores, masking, the
NVFP4/MXFP4 decoding of the full entry point against direct decoding, and
the generator's quantiser against the oracle's rounding.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from tiled_attention_blackwell_b200.workloads import (e2m1_encode, fp4_k_global,
                                                      make_tensors_fp4, quantize_mxfp4_keys,
                                                      quantize_nvfp4)

rng = np.random.default_rng(4321)
CLASSIFIERS = ("affine", "exp2")
# The eight E2M1 magnitudes of the OCP microscaling formats (sign, two
# exponent bits with bias 1, one mantissa bit).
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


# ------------------------------------------------------------- formats

def test_e2m1_decode_table():
    got = [oracle.e2m1_to_float(c) for c in range(16)]
    assert got[:8] == E2M1_TABLE
    assert got[8:] == [-x for x in E2M1_TABLE]
    assert math.copysign(1.0, got[8]) == -1.0  # code 8 is -0


def test_ue8m0_decode():
    for u in (0, 1, 100, 126, 127, 128, 200, 254):
        assert oracle.ue8m0_to_float(u) == math.ldexp(1.0, u - 127)
    assert math.isnan(oracle.ue8m0_to_float(255))


def _nearest_even(x):
    """Brute force: the table entry nearest to x, ties to the even index."""
    d = [abs(x - m) for m in E2M1_TABLE]
    best = min(d)
    cands = [i for i, di in enumerate(d) if di == best]
    return E2M1_TABLE[min(cands, key=lambda i: i % 2)]


def test_e2m1_round_brute_force():
    xs = np.concatenate([np.linspace(0, 6, 2401), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0],
                         rng.uniform(0, 6, 500)])
    for x in xs:
        assert oracle.e2m1_round(float(x)) == _nearest_even(float(x)), x
    # saturating above the largest magnitude
    for x in (6.0, 6.5, 7.0, 7.999, 100.0):
        assert oracle.e2m1_round(x) == 6.0
    # ties: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    assert [oracle.e2m1_round(x) for x in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)] == \
        [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]


def test_generator_encoder_matches_oracle_rounding():
    x = np.concatenate([rng.standard_normal(4000) * 3, [0.25, -0.75, 2.5, -5.0, 9.0, -0.0]])
    codes = e2m1_encode(x)
    for xi, c in zip(x, codes):
        want = math.copysign(oracle.e2m1_round(abs(float(xi))), xi)
        assert oracle.e2m1_to_float(int(c)) == want or (want == 0 and c in (0, 8)), (xi, c)


# ----------------------------------------------------- Direct-P, one row

# Worked rows: every score equal to y0.  Then every 32-key block has
# E = floor(y0) - 2 and r = frac(y0) + 2, so all keys get the same code:
#   exp2 classifier:   2^r rounded to E2M1 (ties even, saturating at 6);
#   affine classifier: index rint(2 r + 2), clamped to 7.
# Hand-derived (y0, code_exp2, code_affine):
#   y0 = 0.2:  2^2.2 = 4.59 -> 4;  rint(6.4) = 6 -> 4
#   y0 = 0.3:  2^2.3 = 4.92 -> 4;  rint(6.6) = 7 -> 6
#   y0 = 0.5:  2^2.5 = 5.66 -> 6;  rint(7.0) = 7 -> 6
#   y0 = 0.9:  2^2.9 = 7.46 -> 6;  rint(7.8) = 8 -> 7 -> 6
#   y0 = -3.7: floor -4, frac 0.3 -> as 0.3, scaled by 2^(-4-2)
WORKED = [(0.2, 4.0, 4.0), (0.3, 4.0, 6.0), (0.5, 6.0, 6.0), (0.9, 6.0, 6.0),
          (-3.7, 4.0, 6.0)]


@pytest.mark.parametrize("classifier", CLASSIFIERS)
@pytest.mark.parametrize("y0,code_exp2,code_affine", WORKED)
def test_direct_p_constant_row(classifier, y0, code_exp2, code_affine):
    n, D = 100, 8
    v = rng.standard_normal((n, D))
    o, lse = oracle.direct_p_row(np.full(n, y0), v, classifier=classifier)
    np.testing.assert_allclose(o, v.mean(axis=0), rtol=0, atol=1e-13)
    code = code_exp2 if classifier == "exp2" else code_affine
    w = code * 2.0 ** (math.floor(y0) - 2)
    assert lse == pytest.approx(math.log(n * w), abs=1e-13)


@pytest.mark.parametrize("classifier", CLASSIFIERS)
def test_direct_p_two_constant_blocks(classifier):
    # keys 0-31 at y = 0.2 (code 4, E = -2: weight 1), keys 32-63 at
    # y = 1.3 (E = -1, r = 2.3: exp2 code 4 -> weight 2; affine index
    # rint(6.6) = 7, code 6 -> weight 3); V constant per block.
    y = np.concatenate([np.full(32, 0.2), np.full(32, 1.3)])
    va, vb = rng.standard_normal(5), rng.standard_normal(5)
    v = np.vstack([np.tile(va, (32, 1)), np.tile(vb, (32, 1))])
    wb = 2.0 if classifier == "exp2" else 3.0
    o, lse = oracle.direct_p_row(y, v, classifier=classifier)
    np.testing.assert_allclose(o, (va + wb * vb) / (1 + wb), rtol=0, atol=1e-13)
    assert lse == pytest.approx(math.log(32 + 32 * wb), abs=1e-13)


@pytest.mark.parametrize("classifier,reach", [("exp2", 3), ("affine", 2)])
def test_direct_p_exact_on_the_grid(classifier, reach):
    # Integer log2 scores no more than `reach` below their block maximum map
    # to r in {2, 1, 0, -1} (exp2) or {2, 1, 0} (affine), i.e. to exactly
    # 2^r: the weights are exactly 2^y and Direct-P equals the softmax.
    n, D = 96, 6
    bmax = rng.integers(-5, 5, size=3)
    y = np.concatenate([bm - rng.integers(0, reach + 1, size=32) for bm in bmax]).astype(float)
    for g, bm in enumerate(bmax):
        y[32 * g] = bm  # each block reaches its maximum
    v = rng.standard_normal((n, D))
    o, lse = oracle.direct_p_row(y, v, classifier=classifier)
    p = scipy.special.softmax(y * math.log(2.0))
    np.testing.assert_allclose(o, p @ v, rtol=0, atol=1e-12)
    assert lse == pytest.approx(scipy.special.logsumexp(y * math.log(2.0)), abs=1e-12)


@pytest.mark.parametrize("classifier", CLASSIFIERS)
def test_direct_p_integer_shift_invariance(classifier):
    n, D = 200, 7
    y = rng.standard_normal(n) * 3
    v = rng.standard_normal((n, D))
    o0, l0 = oracle.direct_p_row(y, v, classifier=classifier)
    for k in (-700, -3, 1, 5, 900):
        o1, l1 = oracle.direct_p_row(y + k, v, classifier=classifier)
        np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-13)
        assert l1 == pytest.approx(l0 + k * math.log(2.0), abs=1e-9)


@pytest.mark.parametrize("classifier", CLASSIFIERS)
def test_direct_p_mask_and_single_key(classifier):
    n, D = 70, 4
    y = rng.standard_normal(n)
    v = rng.standard_normal((n, D))
    allow = np.ones(n, dtype=bool)
    allow[[3, 40, 69]] = False
    o0, l0 = oracle.direct_p_row(y, v, allow=allow, classifier=classifier)
    # a masked key changes nothing, however large its score (and it must not
    # move its block's exponent)
    y2 = y.copy()
    y2[3], y2[40] = 100.0, -1e9
    v2 = v.copy()
    v2[69] = 1e6
    o1, l1 = oracle.direct_p_row(y2, v2, allow=allow, classifier=classifier)
    np.testing.assert_array_equal(o1, o0)
    assert l1 == l0
    # exactly one allowed key: O is that row of V
    one = np.zeros(n, dtype=bool)
    one[17] = True
    o, _ = oracle.direct_p_row(y, v, allow=one, classifier=classifier)
    np.testing.assert_allclose(o, v[17], rtol=0, atol=1e-15)
    # no allowed key: O = 0, LSE = -inf
    o, lse = oracle.direct_p_row(y, v, allow=np.zeros(n, dtype=bool), classifier=classifier)
    assert not o.any() and lse == -math.inf


@pytest.mark.parametrize("classifier", CLASSIFIERS)
def test_direct_p_blocks_follow_key_index(classifier):
    # The 32-key blocks are aligned to the key index: moving one large score
    # from block 0 to block 1 changes the result, moving it within block 0
    # does not (with equal V rows within the block).
    n, D = 64, 3
    y = np.full(n, 0.0)
    v = np.vstack([np.tile(rng.standard_normal(D), (32, 1)), rng.standard_normal((32, D))])
    ya = y.copy()
    ya[5] = 3.4
    yb = y.copy()
    yb[20] = 3.4
    oa, la = oracle.direct_p_row(ya, v, classifier=classifier)
    ob, lb = oracle.direct_p_row(yb, v, classifier=classifier)
    np.testing.assert_allclose(oa, ob, rtol=0, atol=1e-14)
    assert la == lb
    v_mixed = v.copy()
    v_mixed[40] = v[40] + 1.0
    yc = y.copy()
    yc[40] = 3.4
    oc, _ = oracle.direct_p_row(yc, v_mixed, classifier=classifier)
    assert np.abs(oc - oa).max() > 1e-3


@pytest.mark.parametrize("classifier", CLASSIFIERS)
def test_direct_p_block_size_is_32(classifier):
    # One 32-key block: key 3 at y = 3.4, keys 16-31 at y = 0.6, keys 0-15
    # other than 3 masked.  E = floor(3.4) - 2 = 1 for the whole block:
    #   key 3:     r = 2.4 -> exp2 2^2.4 = 5.28 -> 6; affine rint(6.8) = 7 -> 6: w = 12
    #   keys 16-31: r = -0.4 -> exp2 2^-0.4 = 0.758 -> 1 (w = 2);
    #               affine rint(1.2) = 1 -> 0.5 (w = 1)
    # (16-key blocks would give keys 16-31 their own E = -2 and w = 1.5.)
    y = np.zeros(32)
    y[3] = 3.4
    y[16:] = 0.6
    allow = np.zeros(32, dtype=bool)
    allow[3] = True
    allow[16:] = True
    a, b = rng.standard_normal(4), rng.standard_normal(4)
    v = np.zeros((32, 4))
    v[3] = a
    v[16:] = b
    w = 2.0 if classifier == "exp2" else 1.0
    o, lse = oracle.direct_p_row(y, v, allow=allow, classifier=classifier)
    np.testing.assert_allclose(o, (12 * a + 16 * w * b) / (12 + 16 * w), rtol=0, atol=1e-13)
    assert lse == pytest.approx(math.log(12 + 16 * w), abs=1e-13)


# ------------------------------------------------------- full entry point

def _decode_nvfp4(codes, scales, g):
    c = codes.numpy()
    nib = np.stack([c & 15, c >> 4], -1).reshape(*c.shape[:-1], -1)
    mag = np.vectorize(oracle.e2m1_to_float)(nib)
    sc = scales.view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    return g * mag * np.repeat(sc, 16, axis=-1)


def _decode_mxfp4(codes, scales, g):
    c = codes.numpy()
    nib = np.stack([c & 15, c >> 4], -1).reshape(*c.shape[:-1], -1)
    mag = np.vectorize(oracle.e2m1_to_float)(nib)
    S = mag.shape[1]
    sc = np.exp2(scales.numpy().astype(np.float64) - 127)
    return g * mag * np.repeat(sc, 32, axis=1)[:, :S]


def _args(t):
    return (t["q_codes"], t["q_scales"], t["q_global"], t["k_codes"], t["k_scales"],
            t["k_global"], t["v_codes"], t["v_scales"], t["v_global"])


@pytest.mark.parametrize("classifier", CLASSIFIERS)
def test_fp4_zero_queries_give_mean_of_values(classifier):
    # Q codes all zero: every score is 0, every key gets the same weight and
    # O is the running mean of the decoded V rows (causal), LSE = ln(i + 1).
    B, H, S, D = 1, 2, 75, 64
    t = make_tensors_fp4(B, H, H, S, S, D, seed=7)
    t["q_codes"] = torch.zeros_like(t["q_codes"])
    o, lse = oracle.attn_fwd_fp4(*_args(t), scale=0.125, causal=True, classifier=classifier)
    v = _decode_mxfp4(t["v_codes"], t["v_scales"], t["v_global"])
    run_mean = np.cumsum(v, axis=1) / np.arange(1, S + 1)[None, :, None, None]
    np.testing.assert_allclose(o, run_mean, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(np.arange(1, S + 1)), lse.shape),
                               atol=1e-12)


@pytest.mark.parametrize("classifier", CLASSIFIERS)
@pytest.mark.parametrize("pow2", [True, False])
def test_fp4_forward_is_direct_p_of_decoded_scores(classifier, pow2):
    # The entry point = its decoded inputs' scores fed to the pinned row
    # function: checks NVFP4 / MXFP4 decoding, the score scale (c = scale x
    # q_global x k_global x log2 e), GQA and the causal mask together.
    B, Hq, Hkv, S, D = 1, 4, 2, 70, 64
    scale = 0.125
    t = make_tensors_fp4(B, Hq, Hkv, S, S, D, seed=8, scale=scale, pow2_scales=pow2)
    o, lse = oracle.attn_fwd_fp4(*_args(t), scale=scale, causal=True, classifier=classifier)
    q = _decode_nvfp4(t["q_codes"], t["q_scales"], 1.0)
    k = _decode_nvfp4(t["k_codes"], t["k_scales"], 1.0)
    v = _decode_mxfp4(t["v_codes"], t["v_scales"], t["v_global"])
    c = scale * t["q_global"] * t["k_global"] * 1.4426950408889634
    for h in range(Hq):
        hk = h // (Hq // Hkv)
        y = (q[0, :, h] @ k[0, :, hk].T) * c
        for i in (0, 1, 31, 32, 69):
            allow = np.arange(S) <= i
            oi, li = oracle.direct_p_row(y[i], v[0, :, hk], allow=allow, classifier=classifier)
            np.testing.assert_allclose(o[0, i, h], oi, rtol=0, atol=1e-12)
            assert lse[0, h, i] == pytest.approx(li, abs=1e-12)


def test_fp4_per_tensor_factors():
    # v_global scales O exactly and leaves LSE alone; q_global and k_global
    # enter only through their product (the score factor).
    t = make_tensors_fp4(1, 2, 2, 40, 40, 64, seed=12, scale=0.125)
    o1, l1 = oracle.attn_fwd_fp4(*_args(t), scale=0.125, causal=True)
    t2 = dict(t, v_global=2.0 * t["v_global"])
    o2, l2 = oracle.attn_fwd_fp4(*_args(t2), scale=0.125, causal=True)
    np.testing.assert_array_equal(o2, 2.0 * o1)
    np.testing.assert_array_equal(l2, l1)
    t3 = dict(t, q_global=4.0 * t["q_global"], k_global=t["k_global"] / 4.0)
    o3, l3 = oracle.attn_fwd_fp4(*_args(t3), scale=0.125, causal=True)
    np.testing.assert_array_equal(o3, o1)
    np.testing.assert_array_equal(l3, l1)


def test_fp4_out_of_format_nvfp4_scales_read_as_zero():
    # An NVFP4 scale is an unsigned e4m3 magnitude: a block whose scale byte
    # is NaN or has the sign bit set with a nonzero magnitude reads as 0,
    # exactly as if its 16 codes were zero; -0 (0x80) is a zero scale.
    t = make_tensors_fp4(1, 2, 2, 50, 50, 64, seed=13, scale=0.125)
    base, base_l = oracle.attn_fwd_fp4(*_args(t), scale=0.125, causal=True)
    zeroed = dict(t, q_codes=t["q_codes"].clone(), k_codes=t["k_codes"].clone())
    zeroed["q_codes"][0, 7, 1, 8:16] = 0      # Q row 7, head 1, elements 16-31
    zeroed["k_codes"][0, 20, 0, 0:8] = 0      # K row 20, head 0, elements 0-15
    want, want_l = oracle.attn_fwd_fp4(*_args(zeroed), scale=0.125, causal=True)
    assert not np.array_equal(want, base)     # the blocks mattered
    for qs, ks in ((0x7F, 0xFF), (0xB8, 0x81), (0x80 | 0x30, 0x80 | 0x7E)):
        bad = dict(t, q_scales=t["q_scales"].clone(), k_scales=t["k_scales"].clone())
        bad["q_scales"][0, 7, 1, 1] = qs
        bad["k_scales"][0, 20, 0, 0] = ks
        got, got_l = oracle.attn_fwd_fp4(*_args(bad), scale=0.125, causal=True)
        np.testing.assert_array_equal(got, want)
        np.testing.assert_array_equal(got_l, want_l)
    neg0 = dict(t, q_scales=t["q_scales"].clone(), k_scales=t["k_scales"].clone())
    neg0["q_scales"][0, 7, 1, 1] = 0x80
    neg0["k_scales"][0, 20, 0, 0] = 0x80
    got, got_l = oracle.attn_fwd_fp4(*_args(neg0), scale=0.125, causal=True)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(got_l, want_l)


def test_fp4_pow2_scores_are_dyadic():
    # With power-of-two block scales and c a power of two, every log2 score
    # is a multiple of a small power of two far inside fp32's 24 bits: the
    # kernel's fp32 arithmetic reproduces it exactly.
    scale = 1 / math.sqrt(128)
    t = make_tensors_fp4(1, 2, 2, 64, 64, 128, seed=9, scale=scale)
    c = np.float32(scale * t["q_global"] * t["k_global"] * 1.4426950408889634)
    assert math.log2(float(c)) == round(math.log2(float(c)))
    assert t["k_global"] == fp4_k_global(scale)
    q = _decode_nvfp4(t["q_codes"], t["q_scales"], 1.0)
    k = _decode_nvfp4(t["k_codes"], t["k_scales"], 1.0)
    y = (q[0, :, 0] @ k[0, :, 0].T) * float(c)
    assert np.array_equal(y.astype(np.float32).astype(np.float64), y)
    frac_bits = max(int(np.max(-np.log2(np.abs(y[y != 0]) % 1, where=(np.abs(y[y != 0]) % 1) > 0,
                                       out=np.zeros(np.count_nonzero(y))))), 0)
    assert frac_bits < 20


def test_quantizers_round_trip_within_e2m1():
    # NVFP4 encodings decode to within the largest half-step of E2M1 (one
    # block scale, between 4 and 6); MXFP4's OCP scale rule puts a block's
    # maximum at 2^(y - E) in [4, 8), where (6, 8) saturates to 6: within
    # two block scales.
    x = torch.randn(2, 64, 3, 64)
    for pow2 in (True, False):
        codes, scales, g = quantize_nvfp4(x, pow2_scales=pow2)
        xd = _decode_nvfp4(codes, scales, g)
        sc = g * np.repeat(scales.view(torch.float8_e4m3fn).float().numpy(), 16, -1)
        assert np.all(np.abs(xd - x.double().numpy()) <= 1.0 * sc + 1e-12)
    codes, scales = quantize_mxfp4_keys(x)
    xd = _decode_mxfp4(codes, scales, 1.0)
    sc = np.repeat(np.exp2(scales.numpy().astype(float) - 127), 32, axis=1)[:, :64]
    assert np.all(np.abs(xd - x.double().numpy()) <= 2.0 * sc + 1e-12)
    # the OCP rule: every block's largest magnitude decodes to 4 or 6 times
    # its scale (saturation at 6 included)
    blocks = np.abs(xd).reshape(2, 2, 32, 3, 64).max(axis=2)
    ratio = blocks / np.exp2(scales.numpy().astype(float) - 127)
    assert set(np.unique(ratio)) <= {4.0, 6.0}


@pytest.mark.parametrize("classifier,floor", [("affine", 0.9), ("exp2", 0.95)])
def test_fp4_accuracy_against_exact_attention(classifier, floor):
    # A reading check, not a parity pin: the page reports a mean cosine
    # similarity of about 0.944 for its fast Direct-P path against BF16 on
    # Gaussian softmax inputs.  Ours against exact attention of the decoded
    # inputs must be of that order.
    B, H, S, D = 1, 2, 256, 128
    scale = 1 / math.sqrt(D)
    t = make_tensors_fp4(B, H, H, S, S, D, seed=10, scale=scale, pow2_scales=False)
    o, _ = oracle.attn_fwd_fp4(*_args(t), scale=scale, causal=False, classifier=classifier)
    q = _decode_nvfp4(t["q_codes"], t["q_scales"], t["q_global"])
    k = _decode_nvfp4(t["k_codes"], t["k_scales"], t["k_global"])
    v = _decode_mxfp4(t["v_codes"], t["v_scales"], t["v_global"])
    ref, _ = oracle.attn_fwd(q, k, v, scale=scale)
    a, b = o.reshape(-1, D), ref.reshape(-1, D)
    cos = np.sum(a * b, 1) / np.linalg.norm(a, axis=1) / np.linalg.norm(b, axis=1)
    assert cos.mean() >= floor, cos.mean()
