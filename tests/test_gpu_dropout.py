"""Forward with dropout against the fp64 oracle on the same bf16-rounded
inputs and the same keep mask (Philox4x64-10 from (seed, offset), regenerated
independently by the oracle's own implementation of the generator).

Bar: max-abs <= 2e-2 on O (the bf16 path's bar; kept weights are scaled by
256 / t <= 2 here) and the square forward's LSE bound.
"""
import math

import pytest
import torch

from exact_io_aware_53_b200.workloads import DROPOUT_WORKLOADS, random_tensors
from oracle import oracle
from tests._parity import BF16_TOL, LSE_TOL, max_abs

pytestmark = pytest.mark.gpu


def _run(fa_lib, q, k, v, keep_t, seed, offset, causal):
    d = q.shape[-1]
    o, lse = fa_lib.fwd_dropout(q.cuda(), k.cuda(), v.cuda(), keep_t, seed, offset, causal=causal,
                                scale=1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert fa_lib.check_device_status() == 0
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("B,H,N,d,causal,keep_t", [
    (1, 1, 1, 64, False, 230), (1, 2, 200, 128, True, 230), (2, 1, 300, 64, False, 128),
    (1, 2, 513, 128, True, 128), (1, 1, 1000, 128, False, 205), (2, 2, 383, 64, True, 250),
])
def test_dropout_matches_oracle(fa_lib, B, H, N, d, causal, keep_t):
    q, k, v, _ = random_tensors((B, H, N, d), torch.bfloat16, seed=N + d + keep_t)
    seed, offset = 1234567 + N, 3
    o, lse = _run(fa_lib, q, k, v, keep_t, seed, offset, causal)
    ro, rlse = oracle.attn_fwd_dropout(q, k, v, 1 / math.sqrt(d), causal, keep_t, seed, offset)
    assert max_abs(o, ro) <= BF16_TOL
    assert max_abs(lse, rlse) <= LSE_TOL


def test_keep_all_and_keep_none(fa_lib):
    q, k, v, _ = random_tensors((1, 2, 400, 128), torch.bfloat16, seed=3)
    o, lse = _run(fa_lib, q, k, v, 256, 1, 2, True)
    ro, rlse = oracle.attn_fwd(q, k, v, 1 / math.sqrt(128), True)
    assert max_abs(o, ro) <= BF16_TOL and max_abs(lse, rlse) <= LSE_TOL
    o0, lse0 = _run(fa_lib, q, k, v, 0, 1, 2, True)
    assert torch.all(o0 == 0) and torch.equal(lse0, lse)


def test_mask_is_a_function_of_seed_and_offset(fa_lib):
    q, k, v, _ = random_tensors((1, 1, 256, 64), torch.bfloat16, seed=4)
    a, _ = _run(fa_lib, q, k, v, 128, 77, 0, False)
    b, _ = _run(fa_lib, q, k, v, 128, 77, 0, False)
    c, _ = _run(fa_lib, q, k, v, 128, 77, 1, False)
    assert torch.equal(a, b) and not torch.equal(a, c)


def test_dropout_workload_sampled_heads(fa_lib):
    w = DROPOUT_WORKLOADS["dropout_bf16_4x16x4096x128_causal_keep230"]
    q, k, v, _ = random_tensors((w.B, w.H, w.N, w.d), torch.bfloat16, seed=w.seed)
    o, lse = _run(fa_lib, q, k, v, w.keep_t, w.seed, w.offset, w.causal)
    for b, h in ((0, 0), (3, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        ro, rlse = oracle.attn_fwd_dropout(q[sl], k[sl], v[sl], w.scale, w.causal, w.keep_t, w.seed, w.offset,
                                           bh0=b * w.H + h)
        assert max_abs(o[sl], ro) <= BF16_TOL
        assert max_abs(lse[sl], rlse) <= LSE_TOL
