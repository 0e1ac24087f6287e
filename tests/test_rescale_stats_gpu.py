"""The rescale-statistics build counts what the forward's threshold skips.

Checked against closed forms on inputs whose running maximum is known:
  * causal S=1024, 128-row tiles: tile t iterates key blocks 0..t, so the
    row-blocks after each row's first number 128 * sum_t t per head;
  * Q = 0: every score is 0, no block raises a row's maximum;
  * scores constant within a key block and 16 higher (log2 units) in each
    next block: every block after the first raises it by more than the
    threshold, so every raise is a rescale at threshold 8 as well;
  * random scores: at threshold 0 every raise is a rescale, at 8 fewer.
"""
import math

import pytest
import torch

from tiled_attention_blackwell_b200 import rescale_stats as rs
from tiled_attention_blackwell_b200.workloads import make_tensors

pytestmark = pytest.mark.gpu


def run_counts(q, k, v, tau):
    from tiled_attention_blackwell_b200 import attn
    counts = torch.zeros(4, dtype=torch.int64, device="cuda")
    with rs.counting_library() as set_counts:
        set_counts(counts)
        attn.attention(q, k, v, scale=1 / math.sqrt(q.shape[-1]), causal=True,
                       options=attn.default_options(rescale_threshold=tau))
        torch.cuda.synchronize()
        set_counts(None)
        attn.check_device_status()
    return [int(x) for x in counts.cpu()]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def test_counts_match_closed_forms():
    B, H, S, D = 1, 2, 1024, 128
    expected_blocks = H * 128 * sum(range(S // 128))
    t = make_tensors(B, H, H, S, S, D, seed=3)
    q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
    # all scores equal: nothing raises the maximum
    blocks, raises, taken, _ = run_counts(torch.zeros_like(q), k, v, 8.0)
    assert blocks == expected_blocks and raises == 0 and taken == 0
    # scores constant within a key block and 16 higher (log2 units) in each
    # next block: every block raises every row's maximum by more than the
    # threshold (bf16 rounding of K moves a block's score by under 1)
    ramp = torch.div(torch.arange(S, device="cuda"), 128, rounding_mode="floor").float()
    qq = torch.zeros_like(q)
    qq[..., 0] = 1.0
    kk = torch.zeros_like(k)
    kk[..., 0] = (ramp * 16.0 * math.sqrt(D) / math.log2(math.e)).to(torch.bfloat16)[None, :, None]
    blocks, raises, taken, warp = run_counts(qq, kk, v, 8.0)
    assert blocks == expected_blocks and raises == blocks and taken == blocks
    assert warp * 32 == blocks
    # random scores: at threshold 0 every raise is taken; at 8 fewer are
    b0, r0, t0, _ = run_counts(q, k, v, 0.0)
    b8, r8, t8, _ = run_counts(q, k, v, 8.0)
    assert b0 == b8 == expected_blocks
    assert t0 == r0 > 0 and t8 <= r8 and t8 < t0


def test_module_reports_fractions():
    out = rs.rescale_stats("tiny_d64", 8.0)
    assert out["row_blocks_after_first"] >= 0
    assert 0 <= out["rescales"] <= out["rescales_without_threshold"]
    assert out["skipped_fraction"] is None or 0.0 <= out["skipped_fraction"] <= 1.0
