"""e4m3 forward against the fp64 oracle on the dequantized inputs (x8 * descale).

Bound, derived from the arithmetic: the scores are exact e4m3 products summed
in fp32 (as in the bf16 path); the only new rounding is P -> e4m3 before P V.
Round-to-nearest e4m3 has |Q(p) - p| <= max(2^-4 p, 2^-10) (3 mantissa bits;
subnormal spacing 2^-9).  The kernel's p are 2^(s - m) for a running max m no
larger than the row max, so its row sum l >= l_norm = e^(LSE - max_j s_j) and
  |dO_i| <= 2^-4 sum_j P_ij |v_j| + 2^-10 sum_j |v_j| / l_norm
           + 2^-8 max|O_i| (bf16 output rounding) + 1e-3 (fp32 sums, ex2.approx).
The LSE uses the unrounded fp32 p, so the bf16 path's LSE bar applies.
"""
import math

import numpy as np
import pytest
import torch

from exact_io_aware_53_b200.workloads import FP8_WORKLOADS, make_fp8_inputs
from oracle import oracle
from tests._parity import LSE_TOL

pytestmark = pytest.mark.gpu


def _dequant(x):
    return {n: x[n].double() * s for n, s in zip(("q", "k", "v"), x["descales"])}


def _bound(q, k, v, lse, scale, causal, rows=None):
    """Per-row error bound above (fp64, numpy), for all rows or the given ones of every head."""
    q, k, v = (t.numpy() for t in (q, k, v))
    N = q.shape[2]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    s = np.einsum("bhid,bhjd->bhij", q[:, :, rows], k) * scale
    if causal:
        s = np.where(np.arange(N)[None, :] <= rows[:, None], s, -np.inf)
    P = np.exp(s - lse[:, :, rows, None])
    av = np.abs(v)
    l_norm = np.exp(lse[:, :, rows] - s.max(axis=-1))
    allowed = np.isfinite(s)
    small = 2.0 ** -10 * np.einsum("bhij,bhjd->bhid", allowed.astype(np.float64), av) / l_norm[..., None]
    rel = 2.0 ** -4 * np.einsum("bhij,bhjd->bhid", P, av)
    o = np.einsum("bhij,bhjd->bhid", P, v)
    return rel + small + 2.0 ** -8 * np.abs(o).max(axis=-1, keepdims=True) + 1e-3


def _run(fa_lib, x, causal, scale):
    o, lse = fa_lib.fwd_fp8(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), x["descales"], causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa_lib.check_device_status() == 0
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


@pytest.mark.parametrize("B,H,N,causal,gain", [
    # N not a multiple of 16: one CTA per query tile
    (1, 1, 1, False, 1.0), (2, 1, 200, False, 1.0), (1, 2, 513, True, 1.0),
    (1, 1, 1000, False, 1.0), (1, 2, 700, True, 2.0), (2, 2, 383, False, 2.0),
    # N a multiple of 16: the persistent kernel with K read through its permuted
    # view; 400 = 3 * 128 + 16 leaves a last key tile that reaches into the next
    # head's rows (masked), 16 a single short tile
    (1, 2, 128, True, 1.0), (2, 2, 400, True, 1.0), (2, 2, 400, False, 2.0), (1, 3, 16, False, 1.0),
    (1, 1, 1024, True, 1.0), (3, 1, 768, False, 1.0),
])
def test_fp8_matches_oracle_within_the_derived_bound(fa_lib, B, H, N, causal, gain):
    x = make_fp8_inputs((B, H, N, 128), seed=N * 5 + causal, gain=gain)
    scale = 1 / math.sqrt(128)
    o, lse = _run(fa_lib, x, causal, scale)
    dq = _dequant(x)
    ro, rlse = oracle.attn_fwd(dq["q"], dq["k"], dq["v"], scale, causal)
    assert np.max(np.abs(lse - rlse)) <= LSE_TOL
    bound = _bound(dq["q"], dq["k"], dq["v"], rlse, scale, causal)
    err = np.abs(o - ro)
    assert np.all(err <= bound), (float(err.max()), float((err - bound).max()))


@pytest.mark.parametrize("N", [300, 320])
def test_fp8_descales_are_applied(fa_lib, N):
    # q's descale doubled and k's halved leave every score unchanged (powers
    # of two are exact), so the result is bit for bit the same; v's descale
    # doubled doubles O exactly
    x = make_fp8_inputs((1, 2, N, 128), seed=3)
    qd, kd, vd = x["descales"]
    o1, l1 = _run(fa_lib, x, False, 0.1)
    o2, l2 = _run(fa_lib, dict(x, descales=(qd * 2.0, kd / 2.0, vd)), False, 0.1)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    o3, l3 = _run(fa_lib, dict(x, descales=(qd, kd, vd * 2.0)), False, 0.1)
    assert np.array_equal(o3, 2.0 * o1) and np.array_equal(l3, l1)


def test_fp8_workload_sampled_rows(fa_lib):
    w = FP8_WORKLOADS["fp8_e4m3_4x16x4096x128_causal"]
    x = make_fp8_inputs((w.B, w.H, w.N, w.d), seed=w.seed)
    o, lse = _run(fa_lib, x, w.causal, w.scale)
    assert fa_lib.last_launch_count() == 1
    dq = _dequant(x)
    # head (0, 0) on sampled rows, head (3, 15) whole
    for b, h, rows in ((0, 0, [0, 1, 127, 128, 1000, 2047, 3071, 4095]), (3, 15, list(range(w.N)))):
        sl = (slice(b, b + 1), slice(h, h + 1))
        qh, kh, vh = (dq[n][sl] for n in ("q", "k", "v"))
        ro, rlse = oracle.attn_fwd_rows(qh[0, 0], kh[0, 0], vh[0, 0], 0, w.N, w.scale, w.causal)
        assert np.max(np.abs(lse[b, h] - rlse)) <= LSE_TOL
        bound = _bound(qh, kh, vh, rlse[None, None], w.scale, w.causal, rows)[0, 0]
        err = np.abs(o[b, h, rows] - ro[rows])
        assert np.all(err <= bound), (float(err.max()), float((err - bound).max()))
