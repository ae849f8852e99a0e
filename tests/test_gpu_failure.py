"""Failure detection without a GPU fault: a bounded wait that runs out is
reported through the device error word and leaves the context usable."""
import math
import time

import pytest
import torch

from exact_io_aware_53_b200.workloads import random_tensors
from oracle import oracle
from tests._parity import BF16_TOL, max_abs

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_then_cleared_and_kernels_still_run(fa_lib):
    fa = fa_lib
    assert fa.check_device_status() == fa.FA_OK
    t0 = time.perf_counter()
    gave_up = fa.selftest_wait_timeout(50_000_000)  # 50 ms
    elapsed = time.perf_counter() - t0
    assert gave_up == 32  # every lane of the waiting warp gave up
    assert 0.04 < elapsed < 5.0
    assert fa.check_device_status() == fa.FA_ERR_TIMEOUT
    assert fa.check_device_status() == fa.FA_OK  # reported once, then cleared
    # the context is intact: a forward + backward still matches the oracle
    q, k, v, do = random_tensors((1, 2, 200, 128), torch.bfloat16, seed=11)
    scale = 1 / math.sqrt(128)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, scale=scale)
    dq, dk, dv = fa.bwd(q.cuda(), k.cuda(), v.cuda(), o, lse, do.cuda(), causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.check_device_status() == fa.FA_OK
    ro, _ = oracle.attn_fwd(q, k, v, scale, True)
    rdq, rdk, rdv = oracle.attn_bwd(q, k, v, do, scale, True)
    assert max_abs(o, ro) <= BF16_TOL
    assert max(max_abs(dq, rdq), max_abs(dk, rdk), max_abs(dv, rdv)) <= BF16_TOL


def test_wait_limit_arguments_are_checked(fa_lib):
    import ctypes
    f = fa_lib._lib.fa_selftest_wait_timeout
    assert f(10, ctypes.c_void_p(16), None) == fa_lib.FA_ERR_INVALID_ARG
    assert f(50_000_000, None, None) == fa_lib.FA_ERR_INVALID_ARG
