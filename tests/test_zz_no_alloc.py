"""attn_bwd_noalloc: the backward for callers that cannot allocate device
memory where they run it (a plugin handed only its input and output
pointers, or a hot loop that must not call cudaMalloc, which can stall every
stream and can fail mid-step).  It uses the library's fixed scratch instead
of a caller workspace.  It runs the same deterministic kernels as attn_bwd,
so its results must equal attn_bwd's bit for bit, call after call.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_blackwell_b200 import attn, build
from tiled_attention_blackwell_b200.workloads import make_tensors

GRAD_TOL = 5e-2  # the backward tests' tolerance: max-abs <= 5e-2 * max|gradient|
LIMIT_ROWS = 1 << 20  # B * Hq * Sq the built-in scratch holds


@pytest.mark.gpu
def test_noalloc_backward_equals_workspace_backward_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    dev = "cuda:0"
    # Three calls in a row, the largest first: each later call reads only
    # entries it wrote itself, never what an earlier (larger) call left in
    # the shared scratch.  The first fills the scratch to its limit.
    cases = (
        (70, (64, 16, 4, 1024, 128), True),   # B * Hq * Sq = 1048576: the limit
        (71, (2, 4, 2, 777, 128), True),
        (72, (1, 2, 2, 300, 64), False),
    )
    for seed, (B, Hq, Hkv, S, D), causal in cases:
        assert B * Hq * S <= LIMIT_ROWS
        t = make_tensors(B, Hq, Hkv, S, S, D, seed, with_dout=True)
        q, k, v, dout = (t[n].to(dev) for n in ("q", "k", "v", "dout"))
        scale = 1.0 / math.sqrt(D)
        o, lse = attn.attention(q, k, v, scale=scale, causal=causal)
        ref = attn.attention_backward(q, k, v, o, lse, dout, scale=scale, causal=causal)
        dq = torch.full(q.shape, float("nan"), dtype=torch.float32, device=dev)
        dk = torch.full_like(k, float("nan"))
        dv = torch.full_like(v, float("nan"))
        attn.attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, scale=scale, causal=causal)
        torch.cuda.synchronize()
        assert attn.device_status() == attn.ATTN_OK
        for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            assert torch.equal(got, want), f"{name} differs from attn_bwd (shape {B, Hq, S})"
        if B * Hq * S == LIMIT_ROWS:
            # At the limit, also against the oracle on the first and last
            # batch (batches are independent problems).
            for b in (0, B - 1):
                sl = slice(b, b + 1)
                dq_r, dk_r, dv_r, _, _ = oracle.attn_bwd(t["q"][sl], t["k"][sl], t["v"][sl],
                                                         t["dout"][sl], scale=scale,
                                                         causal=causal)
                for got, r in ((dq[sl], dq_r), (dk[sl], dk_r), (dv[sl], dv_r)):
                    g = got.float().cpu().numpy().astype(np.float64)
                    assert np.isfinite(g).all()
                    assert np.abs(g - r).max() <= GRAD_TOL * np.abs(r).max()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    build.build()
    P = 0x10000  # never dereferenced: the size check comes first
    rows_too_many = (1, 32, 32769)  # B * Hq * Sq = 1048608 > 1048576
    B, Hq, Sq = rows_too_many
    st = attn.lib().attn_bwd_noalloc(*([P] * 9), B, Hq, Hq, Sq, Sq, 128, 0.1, 1, -1, -1,
                                     None, 0, None)
    assert st == attn.ATTN_ERR_UNSUPPORTED
    assert b"scratch" in attn.lib().attn_last_error_detail()
