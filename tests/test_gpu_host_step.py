"""The host-buffer step (fa_attention_host): forward + backward from pinned host
tensors, run in head chunks whose copies in, compute and copies out overlap on
three streams.

Every chunk runs the same kernels as one whole-tensor call, so O, LSE, dK and
dV must equal the device entry points' results bit for bit; dQ is summed by
reduce-adds in no fixed order, so it is held to a rounding-level bar.  One small
shape is also compared with the oracle.  Shapes cover one chunk, several
chunks with a short last one, an odd N (the LSE slices of later chunks start
at h0 * N floats), both head dimensions, and outputs left out (NULL).
"""
import math

import pytest
import torch

from exact_io_aware_53_b200.workloads import random_tensors
from oracle import oracle
from tests._parity import BF16_TOL, LSE_TOL, max_abs

pytestmark = pytest.mark.gpu

SHAPES = [
    # (B, H, N, d, causal): a first chunk of 4 heads, then chunks of G heads
    (1, 3, 200, 128, False),   # one chunk
    (2, 9, 333, 64, True),     # 18 heads: chunks 4, 4, 4, 4, 2; N odd
    (4, 16, 1024, 128, True),  # 64 heads: 4, then 8 chunks of 8 (the last 4)
    (3, 5, 130, 64, False),    # 15 heads: chunks 4, 4, 4, 3
]


def _host_step(fa, x, causal, scale, keep=("o", "lse", "dq", "dk", "dv")):
    B, H, N, d = x["q"].shape
    hx = {n: t.pin_memory() for n, t in x.items()}
    outs = {"o": torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16).pin_memory(),
            "lse": torch.full((B, H, N), float("nan")).pin_memory()}
    for n in ("dq", "dk", "dv"):
        outs[n] = torch.full((B, H, N, d), float("nan")).pin_memory()
    arena = torch.empty(fa.attention_host_arena_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    fa.attention_host(hx["q"], hx["k"], hx["v"], hx["do"], arena, {n: outs[n] for n in keep}, causal, scale)
    launches = fa.last_launch_count()
    torch.cuda.synchronize()
    assert fa.check_device_status() == fa.FA_OK
    return outs, launches


@pytest.mark.parametrize("shape", SHAPES)
def test_host_step_equals_device_calls(fa_lib, shape):
    fa = fa_lib
    B, H, N, d, causal = shape
    q, k, v, do = random_tensors((B, H, N, d), torch.bfloat16, seed=31 + N)
    x = {"q": q, "k": k, "v": v, "do": do}
    scale = 1 / math.sqrt(d)
    outs, launches = _host_step(fa, x, causal, scale)
    xc = {n: t.cuda() for n, t in x.items()}
    o, lse = fa.fwd(xc["q"], xc["k"], xc["v"], causal=causal, scale=scale)
    dq, dk, dv = fa.bwd(xc["q"], xc["k"], xc["v"], o, lse, xc["do"], causal=causal, scale=scale)
    torch.cuda.synchronize()
    BH = B * H  # a first chunk of min(BH, 4) heads, then chunks of G (a multiple of 4) heads
    G0 = min(BH, 4)
    G = max(4, 4 * math.ceil(math.ceil((BH - G0) / 8) / 4))
    assert launches == 3 * (1 + math.ceil((BH - G0) / G))  # forward, pre-pass and main kernel per chunk
    assert torch.equal(outs["o"], o.cpu())
    assert torch.equal(outs["lse"], lse.cpu())
    assert torch.equal(outs["dk"], dk.cpu())
    assert torch.equal(outs["dv"], dv.cpu())
    # dQ: the same terms added in another order
    assert max_abs(outs["dq"], dq) <= 1e-4 * max(1.0, float(dq.abs().max()))


def test_host_step_against_oracle(fa_lib):
    fa = fa_lib
    B, H, N, d, causal = 2, 9, 333, 64, True
    q, k, v, do = random_tensors((B, H, N, d), torch.bfloat16, seed=5)
    scale = 1 / math.sqrt(d)
    outs, _ = _host_step(fa, {"q": q, "k": k, "v": v, "do": do}, causal, scale)
    ro, rlse = oracle.attn_fwd(q, k, v, scale, causal)
    rdq, rdk, rdv = oracle.attn_bwd(q, k, v, do, scale, causal)
    assert max_abs(outs["o"], ro) <= BF16_TOL
    assert max_abs(outs["lse"], rlse) <= LSE_TOL
    for got, ref in ((outs["dq"], rdq), (outs["dk"], rdk), (outs["dv"], rdv)):
        assert max_abs(got, ref) <= BF16_TOL


def test_host_step_skips_null_outputs(fa_lib):
    fa = fa_lib
    B, H, N, d, causal = 2, 9, 333, 128, False
    q, k, v, do = random_tensors((B, H, N, d), torch.bfloat16, seed=6)
    outs, _ = _host_step(fa, {"q": q, "k": k, "v": v, "do": do}, causal, 1 / math.sqrt(d), keep=("o", "dk"))
    assert torch.isfinite(outs["o"].float()).all() and torch.isfinite(outs["dk"]).all()
    # the outputs left out were never written
    for n in ("lse", "dq", "dv"):
        assert torch.isnan(outs[n]).all()
