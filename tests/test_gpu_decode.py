"""Split-KV forward (Nq queries against Nk keys) against the fp64 oracle's
rectangular attention on the same bf16-rounded inputs.

Bar: max-abs <= 2e-2 on O, LSE within the same bound as the square forward.
Shapes span several key tiles with ragged tails, several query tiles, empty
key ranges under the causal mask, and range counts from one to more than the
key tiles; the full-size decode workload (8 x 16 heads, one query, 16384
keys, d = 128, causal) is compared in full.
"""
import math

import pytest
import torch

from exact_io_aware_53_b200.workloads import random_tensors
from oracle import oracle
from tests._parity import BF16_TOL, LSE_TOL, max_abs

pytestmark = pytest.mark.gpu


def _inputs(B, H, Nq, Nk, d, seed, gain=1.0):
    q, = random_tensors((B, H, Nq, d), torch.bfloat16, seed=seed, count=1, gain=gain)
    k, v = random_tensors((B, H, Nk, d), torch.bfloat16, seed=seed + 1, count=2, gain=1.0)
    if gain != 1.0:
        k, = random_tensors((B, H, Nk, d), torch.bfloat16, seed=seed + 2, count=1, gain=gain)
    return q, k, v


def _run(fa_lib, q, k, v, causal, n_split):
    d = q.shape[-1]
    o, lse = fa_lib.fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=1 / math.sqrt(d),
                                n_split=n_split)
    torch.cuda.synchronize()
    assert fa_lib.check_device_status() == 0
    return o, lse


CASES = [
    # (B, H, Nq, Nk, d, causal, n_split)
    (1, 1, 1, 1, 64, False, 0),
    (1, 1, 1, 1, 128, True, 0),
    (2, 3, 1, 1000, 128, True, 0),
    (2, 3, 1, 1000, 128, True, 1),
    (2, 3, 1, 1000, 128, False, 3),
    (1, 2, 1, 4097, 64, True, 7),
    (1, 2, 16, 2000, 128, True, 5),
    (1, 2, 16, 2000, 64, False, 16),   # more ranges than key tiles: clipped
    (2, 1, 128, 700, 128, True, 2),
    (1, 1, 200, 1333, 128, True, 4),   # two query tiles, ragged both ways
    (1, 1, 200, 200, 64, True, 3),     # Nq == Nk: the square causal forward
    (1, 1, 300, 130, 64, False, 2),    # more queries than keys
    (1, 3, 5, 129, 128, True, 2),      # second range holds one key
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,n_split", CASES)
def test_splitkv_matches_oracle(fa_lib, B, H, Nq, Nk, d, causal, n_split):
    q, k, v = _inputs(B, H, Nq, Nk, d, seed=Nq * 31 + Nk + d + causal)
    o, lse = _run(fa_lib, q, k, v, causal, n_split)
    ro, rlse = oracle.attn_fwd_rect(q, k, v, 1 / math.sqrt(d), causal)
    assert max_abs(o, ro) <= BF16_TOL
    assert max_abs(lse, rlse) <= LSE_TOL


@pytest.mark.parametrize("d", [64, 128])
def test_split_count_does_not_change_the_result_beyond_rounding(fa_lib, d):
    q, k, v = _inputs(1, 4, 3, 3000, d, seed=5 + d)
    ro, rlse = oracle.attn_fwd_rect(q, k, v, 1 / math.sqrt(d), True)
    for n_split in (1, 2, 5, 24, 0):
        o, lse = _run(fa_lib, q, k, v, True, n_split)
        assert max_abs(o, ro) <= BF16_TOL, n_split
        assert max_abs(lse, rlse) <= LSE_TOL, n_split


def test_late_dominant_key_in_one_range(fa_lib):
    # scores with standard deviation ~6 (gain 2.5 on q and k): the running max moves
    # inside a range and the merge weights span many orders of magnitude
    q, k, v = _inputs(2, 2, 4, 2500, 128, seed=77, gain=2.5)
    k[:, :, 2400] = q[:, :, 0]  # one key far above the rest, in the last range
    o, lse = _run(fa_lib, q, k, v, False, 6)
    ro, rlse = oracle.attn_fwd_rect(q, k, v, 1 / math.sqrt(128), False)
    assert max_abs(o, ro) <= BF16_TOL
    assert max_abs(lse, rlse) <= LSE_TOL


def test_single_query_causal_equals_full(fa_lib):
    # the one query is the last position and sees every key
    q, k, v = _inputs(1, 2, 1, 1500, 64, seed=9)
    oc, lc = _run(fa_lib, q, k, v, True, 4)
    on, ln = _run(fa_lib, q, k, v, False, 4)
    assert torch.equal(oc, on) and torch.equal(lc, ln)


def test_decode_workload_full_size(fa_lib):
    # 8 x 16 heads, one query each, 16384 cached keys, d = 128, causal:
    # the launch configuration the decode bench times
    B, H, Nq, Nk, d = 8, 16, 1, 16384, 128
    q, k, v = _inputs(B, H, Nq, Nk, d, seed=2024)
    o, lse = _run(fa_lib, q, k, v, True, 0)
    ro, rlse = oracle.attn_fwd_rect(q, k, v, 1 / math.sqrt(d), True)
    assert max_abs(o, ro) <= BF16_TOL
    assert max_abs(lse, rlse) <= LSE_TOL
    assert fa_lib.last_launch_count() == 2
