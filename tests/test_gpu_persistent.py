"""The backward's persistent CTAs: one per SM, each walking several (head, key
tile) items claimed from the work counter in the workspace.

The small-shape tests elsewhere give most CTAs a single item; these shapes have
two to five items per CTA (148 SMs), of different lengths under the causal
mask, with a ragged last key tile, so the paths that run only between items are
compared in full against the fp64 oracle: the next item's first S^T and dP^T
issued from the current item's last step, the alternating K, V buffers (d = 64)
or the single buffer refilled after the epilogue (d = 128), the epilogues that
run while the next item starts, and the claimed order.  Both softmax warp
layouts, and dropout at d = 64 (whose backward is persistent), are covered.
A second call on the same workspace checks that the pre-pass re-arms the
counter.
"""
import math

import pytest
import torch

from exact_io_aware_53_b200.workloads import random_tensors
from oracle import oracle
from tests._parity import BF16_TOL, LSE_TOL, max_abs

pytestmark = pytest.mark.gpu

SHAPES = [
    # (B, H, N, d, causal): B*H*ceil(N/128) items over 148 CTAs
    (4, 40, 300, 64, True),    # 480 items of 1-3 query tiles
    (4, 40, 300, 64, False),   # 480 items of 3 query tiles
    (2, 50, 520, 128, True),   # 500 items of 1-5 query tiles
    (3, 30, 383, 128, False),  # 360 items of 3 query tiles
]


@pytest.mark.parametrize("warps", [8, 4])
@pytest.mark.parametrize("shape", SHAPES)
def test_persistent_backward_many_items_per_cta(fa_lib, shape, warps):
    fa = fa_lib
    B, H, N, d, causal = shape
    q, k, v, do = random_tensors((B, H, N, d), torch.bfloat16, seed=400 + N + d)
    scale = 1 / math.sqrt(d)
    qc, kc, vc, dc = (t.cuda() for t in (q, k, v, do))
    assert fa._lib.fa_set_bwd_softmax_warps(warps) == fa.FA_OK
    try:
        o, lse = fa.fwd(qc, kc, vc, causal=causal, scale=scale)
        ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
        outs = []
        for _ in range(2):  # the second call reuses the workspace (the counter is re-armed)
            g = fa.bwd(qc, kc, vc, o, lse, dc, causal=causal, scale=scale, workspace=ws)
            torch.cuda.synchronize()
            assert fa.check_device_status() == fa.FA_OK
            outs.append([t.cpu() for t in g])
    finally:
        fa._lib.fa_set_bwd_softmax_warps(0)
    rdq, rdk, rdv = oracle.attn_bwd(q, k, v, do, scale, causal)
    for got in outs:
        for name, g, r in (("dq", got[0], rdq), ("dk", got[1], rdk), ("dv", got[2], rdv)):
            assert max_abs(g, r) <= BF16_TOL, name
    # dK and dV come from one CTA per item with a fixed order of additions
    assert torch.equal(outs[0][1], outs[1][1]) and torch.equal(outs[0][2], outs[1][2])


def test_persistent_dropout_backward_many_items_per_cta(fa_lib):
    fa = fa_lib
    B, H, N, d, causal, keep_t, seed, offset = 4, 40, 300, 64, True, 200, 123, 7
    q, k, v, do = random_tensors((B, H, N, d), torch.bfloat16, seed=77)
    scale = 1 / math.sqrt(d)
    qc, kc, vc, dc = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd_dropout(qc, kc, vc, keep_t, seed, offset, causal=causal, scale=scale)
    dq, dk, dv = fa.bwd_dropout(qc, kc, vc, o, lse, dc, keep_t, seed, offset, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.check_device_status() == fa.FA_OK
    rdq, rdk, rdv = oracle.attn_bwd_dropout(q, k, v, do, scale, causal, keep_t, seed, offset)
    # The kept weights enter every gradient scaled by z = 256 / keep_t, so the bf16
    # rounding of P o Z and dS is scaled by z too: the plain bar times z (1.28 here;
    # over these 160 heads the largest dK error is 0.0208, the same value bit for bit
    # as the one-CTA-per-item kernel gives).
    tol = BF16_TOL * 256.0 / keep_t
    for name, g, r in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        assert max_abs(g, r) <= tol, name


@pytest.mark.parametrize("B,H,N,d,causal", [
    (4, 40, 300, 64, False), (4, 40, 300, 128, False), (2, 40, 550, 64, True), (2, 30, 550, 128, True),
])
def test_forward_items_with_a_q_tile_past_n(fa_lib, B, H, N, d, causal):
    """The forward's persistent CTAs take several items each here, and with an odd
    number of 128-row Q tiles per head every head's last item has its second Q tile
    past N: that tile only passes the shared O staging tile on.  Its eight warps
    must all have seen the tile free before it is passed on; passing it on after
    the first warp had seen it let a slower warp wait for the next item's phase
    and stall that item (a bounded wait expired)."""
    q, k, v = random_tensors((B, H, N, d), torch.bfloat16, seed=900 + N + d, count=3)
    scale = 1 / math.sqrt(d)
    o, lse = fa_lib.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa_lib.check_device_status() == fa_lib.FA_OK
    ro, rlse = oracle.attn_fwd(q, k, v, scale, causal)
    assert max_abs(o, ro) <= BF16_TOL
    assert max_abs(lse, rlse) <= LSE_TOL
