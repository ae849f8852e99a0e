"""Block-sparse forward against the fp64 oracle's block-mask attention on the
same bf16-rounded inputs (128 x 128 tiles).

Bar: max-abs <= 2e-2 on O and the square forward's LSE bound; rows with no
allowed key must come out exactly O = 0, LSE = -inf.  Shapes span several
tiles with ragged tails, shared and per-head masks, empty query tiles, and
masks that reduce to the dense problem; the bench workload (4 x 16 heads,
N = 4096, d = 128, half the tile pairs) is compared on whole heads.
"""
import math

import numpy as np
import pytest
import torch

from exact_io_aware_53_b200.workloads import BLOCKSPARSE_WORKLOADS, make_block_mask, random_tensors
from oracle import oracle
from tests._parity import BF16_TOL, LSE_TOL, max_abs

pytestmark = pytest.mark.gpu


def _masks(T, H, seed, per_head, density=0.5):
    g = torch.Generator().manual_seed(seed)
    m = (torch.rand((H if per_head else 1, T, T), generator=g) < density).to(torch.uint8)
    return m


def _run(fa_lib, q, k, v, mask, causal):
    d = q.shape[-1]
    o, lse = fa_lib.fwd_blocksparse(q.cuda(), k.cuda(), v.cuda(), mask.cuda(), causal=causal, scale=1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert fa_lib.check_device_status() == 0
    return o.cpu(), lse.cpu()


def _compare(o, lse, ro, rlse):
    assert max_abs(o, ro) <= BF16_TOL
    lse = lse.double().numpy()
    assert np.array_equal(np.isinf(lse), np.isinf(rlse))
    fin = np.isfinite(rlse)
    assert np.max(np.abs(lse[fin] - rlse[fin]), initial=0.0) <= LSE_TOL


CASES = [
    # (B, H, N, d, causal, per_head)
    (1, 1, 1, 64, False, False),
    (1, 2, 100, 128, True, False),
    (2, 1, 256, 64, False, True),
    (1, 3, 300, 128, False, True),
    (1, 2, 513, 64, True, True),
    (2, 2, 1000, 128, True, False),
    (1, 1, 1300, 128, False, False),
]


@pytest.mark.parametrize("B,H,N,d,causal,per_head", CASES)
def test_blocksparse_matches_oracle(fa_lib, B, H, N, d, causal, per_head):
    q, k, v, _ = random_tensors((B, H, N, d), torch.bfloat16, seed=N + d + causal)
    T = (N + 127) // 128
    mask = _masks(T, H, seed=N * 3 + d, per_head=per_head)
    mask[0, T - 1, :] = 0  # the last query tile of head 0 sees nothing
    o, lse = _run(fa_lib, q, k, v, mask, causal)
    ro, rlse = oracle.attn_fwd_blockmask(q, k, v, 1 / math.sqrt(d), causal, mask.numpy())
    _compare(o, lse, ro, rlse)
    rows = slice((T - 1) * 128, N)
    assert torch.all(o[:, 0, rows] == 0) and torch.all(lse[:, 0, rows] == -math.inf)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_full_mask_is_the_dense_forward(fa_lib, d, causal):
    q, k, v, _ = random_tensors((2, 2, 700, d), torch.bfloat16, seed=11 + d)
    mask = torch.ones((1, 6, 6), dtype=torch.uint8)
    o, lse = _run(fa_lib, q, k, v, mask, causal)
    ro, rlse = oracle.attn_fwd(q, k, v, 1 / math.sqrt(d), causal)
    _compare(o, lse, ro, rlse)


def test_mask_above_the_diagonal_is_ignored_under_causal(fa_lib):
    q, k, v, _ = random_tensors((1, 2, 640, 128), torch.bfloat16, seed=5)
    lower = torch.tril(torch.ones((5, 5), dtype=torch.uint8))
    mixed = lower.clone()
    mixed[0, 3] = mixed[1, 4] = mixed[2, 3] = 1
    o1, l1 = _run(fa_lib, q, k, v, lower, True)
    o2, l2 = _run(fa_lib, q, k, v, mixed, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_blocksparse_workload_full_size(fa_lib):
    w = BLOCKSPARSE_WORKLOADS["blocksparse_bf16_4x16x4096x128_d50"]
    q, k, v, _ = random_tensors((w.B, w.H, w.N, w.d), torch.bfloat16, seed=w.seed)
    mask = make_block_mask(w)
    o, lse = _run(fa_lib, q, k, v, mask, w.causal)
    assert fa_lib.last_launch_count() == 1
    for b, h in ((0, 0), (3, 15)):
        ro, rlse = oracle.attn_fwd_blockmask(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], w.scale,
                                             w.causal, mask.numpy())
        _compare(o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], ro, rlse)
