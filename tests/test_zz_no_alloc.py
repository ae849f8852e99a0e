"""The allocation-free backward entry point (fa_bwd_noalloc).

It exists for callers that cannot allocate device memory themselves (hosts
that own all device memory and only pass a library its tensors, or loops that
must not call cudaMalloc / cudaFree).  It must give the same gradients as
fa_bwd with a caller-provided workspace, call after call: the built-in
scratch area keeps the previous call's contents, so two calls in a row with
different inputs and sizes are compared.  This file is collected last.
"""
import ctypes
import math

import pytest
import torch

from exact_io_aware_53_b200.workloads import random_tensors
from tests._parity import BF16_TOL, max_abs


def _inputs(shape, seed, fa):
    q, k, v, do = (t.cuda() for t in random_tensors(shape, torch.bfloat16, seed=seed))
    scale = 1 / math.sqrt(shape[-1])
    return q, k, v, do, scale


@pytest.mark.gpu
@pytest.mark.parametrize("first,second", [
    (((1, 2, 300, 128), True), ((2, 3, 513, 128), False)),
    (((2, 2, 383, 64), False), ((1, 4, 640, 64), True)),
    # a large call leaves its row terms in the scratch area; the smaller ragged
    # causal call after it must not read any of them (its padding rows included)
    (((2, 4, 1000, 128), False), ((1, 1, 130, 128), True)),
])
def test_noalloc_backward_matches_workspace_backward_twice(first, second):
    from exact_io_aware_53_b200 import fa
    for n, (shape, causal) in enumerate((first, second)):
        q, k, v, do, scale = _inputs(shape, 77 + n, fa)
        o, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
        ref = fa.bwd(q, k, v, o, lse, do, causal=causal, scale=scale)
        got = [torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda") for _ in range(3)]
        rc = fa.bwd_noalloc_raw(q, k, v, o, lse, do, *got, scale, causal)
        assert rc == fa.FA_OK, fa.status_string(rc)
        assert fa.last_launch_count() == 2  # pre-pass and main kernel
        torch.cuda.synchronize()
        assert fa.check_device_status() == fa.FA_OK
        for g, r in zip(got, ref):
            assert torch.isfinite(g).all()
            assert max_abs(g, r) <= BF16_TOL


@pytest.mark.gpu
def test_noalloc_rejects_workloads_beyond_its_scratch_area():
    from exact_io_aware_53_b200 import fa
    P = ctypes.c_void_p
    ptrs = [P(256)] * 9
    # 4 MiB of scratch holds two fp32 row vectors of 512K rows; 1M rows do not fit
    rc = fa._lib.fa_bwd_noalloc(*ptrs, 8, 128, 1024, 128, 0.1, 1, P(0))
    assert rc == fa.FA_ERR_UNSUPPORTED
    assert fa.last_launch_count() == 0
    assert fa._lib.fa_bwd_noalloc(*([P(0)] + ptrs[1:]), 1, 1, 8, 128, 0.1, 1, P(0)) == fa.FA_ERR_INVALID_ARG
