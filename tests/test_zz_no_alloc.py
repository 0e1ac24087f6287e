"""attn_bwd_noalloc: the backward for callers that cannot allocate device
memory where they run it (a plugin handed only its input and output
pointers, or a hot loop that must not call cudaMalloc, which can stall every
stream and can fail mid-step).  It uses the library's fixed scratch instead
of a caller workspace; its results must match attn_bwd's, call after call.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import math

import numpy as np
import pytest
import torch

from tiled_attention_blackwell_b200 import attn, build
from tiled_attention_blackwell_b200.workloads import make_tensors

GRAD_TOL = 5e-2  # the backward tests' tolerance: max-abs <= 5e-2 * max|gradient|


def _close(got, ref):
    floor = 1e-3 * max(float(r.abs().max()) for r in ref)
    for g, r in zip(got, ref):
        g, r = g.float(), r.float()
        assert torch.isfinite(g).all()
        scale = max(float(r.abs().max()), floor, 1e-12)
        assert float((g - r).abs().max()) <= GRAD_TOL * scale


@pytest.mark.gpu
def test_noalloc_backward_matches_workspace_backward_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    dev = "cuda:0"
    # Two calls in a row with different shapes and masks: the second must not
    # see anything the first left in the shared scratch.
    for seed, shape, causal in ((71, (2, 4, 2, 777, 128), True), (72, (1, 2, 2, 300, 64), False)):
        B, Hq, Hkv, S, D = shape
        t = make_tensors(B, Hq, Hkv, S, S, D, seed, with_dout=True)
        q, k, v, dout = (t[n].to(dev) for n in ("q", "k", "v", "dout"))
        scale = 1.0 / math.sqrt(D)
        o, lse = attn.attention(q, k, v, scale=scale, causal=causal)
        ref = attn.attention_backward(q, k, v, o, lse, dout, scale=scale, causal=causal)
        dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
        dk = torch.empty_like(k)
        dv = torch.empty_like(v)
        attn.attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, scale=scale, causal=causal)
        torch.cuda.synchronize()
        assert attn.device_status() == attn.ATTN_OK
        _close((dq, dk, dv), ref)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    build.build()
    P = 0x10000  # never dereferenced: the size check comes first
    rows_too_many = (1, 32, 32769)  # B * Hq * Sq = 1048608 > 1048576
    B, Hq, Sq = rows_too_many
    st = attn.lib().attn_bwd_noalloc(*([P] * 9), B, Hq, Hq, Sq, Sq, 128, 0.1, 1, -1, -1,
                                     None, 0, None)
    assert st == attn.ATTN_ERR_UNSUPPORTED
    assert b"scratch" in attn.lib().attn_last_error_detail()
