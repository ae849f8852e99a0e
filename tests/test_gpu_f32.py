"""fp32 path (CUDA cores) against the fp64 oracle at 1e-5 max-abs."""
import json
import math
import os

import numpy as np
import pytest
import torch

from exact_io_aware_53_b200.workloads import WORKLOADS, make_inputs, random_tensors
from oracle import oracle
from tests._parity import F32_TOL, max_abs

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _run(fa, x, causal, scale, block_k=0):
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd_f32(q, k, v, causal=causal, scale=scale, block_k=block_k)
    dq, dk, dv = fa.bwd_f32(q, k, v, o, lse, do, causal=causal, scale=scale, block_k=block_k)
    torch.cuda.synchronize()
    return o, lse, dq, dk, dv


def _check(fa, x, causal, scale, block_k=0):
    o, lse, dq, dk, dv = _run(fa, x, causal, scale, block_k)
    ro, rlse = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal)
    rdq, rdk, rdv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal)
    assert max_abs(o, ro) <= F32_TOL
    assert max_abs(lse, rlse) <= F32_TOL
    assert max_abs(dq, rdq) <= F32_TOL
    assert max_abs(dk, rdk) <= F32_TOL
    assert max_abs(dv, rdv) <= F32_TOL


def test_config1_fwd_bwd(fa_lib):
    w = WORKLOADS["c1_f32_1x2x256x64"]
    _check(fa_lib, make_inputs(w), w.causal, w.scale)


@pytest.mark.parametrize("shape,causal", [((1, 2, 1, 64), False), ((2, 1, 37, 16), True),
                                          ((1, 3, 130, 128), True), ((1, 1, 257, 7), False)])
def test_ragged_and_edge_shapes(fa_lib, shape, causal):
    q, k, v, do = random_tensors(shape, torch.float32, seed=sum(shape) + causal)
    _check(fa_lib, {"q": q, "k": k, "v": v, "do": do}, causal, 1 / math.sqrt(shape[-1]))


@pytest.mark.parametrize("block_k", [1, 2, 3, 7, 64, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_block_size_never_changes_the_answer(fa_lib, block_k, causal):
    """Forward and backward walk keys (and, for dK / dV, queries) in blocks of
    block_k; every block size, divisors of N or not, gives the oracle's answer."""
    w = WORKLOADS["c1_f32_1x2x256x64"]
    x = make_inputs(w)
    o, lse, dq, dk, dv = _run(fa_lib, x, causal, w.scale, block_k)
    ro, rlse = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, causal)
    rdq, rdk, rdv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], w.scale, causal)
    assert max_abs(o, ro) <= F32_TOL
    assert max_abs(lse, rlse) <= F32_TOL
    assert max_abs(dq, rdq) <= F32_TOL
    assert max_abs(dk, rdk) <= F32_TOL
    assert max_abs(dv, rdv) <= F32_TOL


def test_worked_row_through_the_gpu():
    """The page's row [2,1,3,0] (block 2) as attention: q0 = e1, k_j = s_j e1,
    scale 1, V = I; row 0 of O must be the printed weights."""
    from exact_io_aware_53_b200 import fa
    with open(os.path.join(GOLDEN, "worked_row.json")) as f:
        g = json.load(f)
    N = d = 4
    q = torch.zeros(1, 1, N, d)
    k = torch.zeros(1, 1, N, d)
    q[0, 0, 0, 0] = 1.0
    k[0, 0, :, 0] = torch.tensor(g["row"])
    v = torch.eye(N)[None, None].contiguous()
    o, lse = fa.fwd_f32(q.cuda(), k.cuda(), v.cuda(), causal=False, scale=1.0, block_k=g["block"])
    torch.cuda.synchronize()
    assert [round(x, 4) for x in o[0, 0, 0].tolist()] == g["weights"]
    assert round(math.exp(lse[0, 0, 0].item() - 3.0), 4) == g["l_final"]
    ro, rlse = oracle.attn_fwd(q, k, v, 1.0, False)
    assert max_abs(o, ro) <= F32_TOL and max_abs(lse, rlse) <= F32_TOL
