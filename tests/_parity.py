"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, compare element by element."""
import numpy as np
import torch

from oracle import oracle

BF16_TOL = 2e-2   # max-abs on O, dQ, dK, dV against the oracle on bf16-rounded inputs
F32_TOL = 1e-5    # max-abs for the fp32 path
# LSE: |d lse| <= |d l / l| + |d s|; l is a sum of <= N fp32 terms (relative
# error <= N * 2^-24 ~ 1e-3 at N = 16384) and each score is an fp32 sum of exact
# bf16 products (~d * 2^-24 |q||k|), so 5e-3 bounds it with room.
LSE_TOL = 5e-3


def max_abs(a, b) -> float:
    a = a.detach().cpu().double().numpy() if hasattr(a, "detach") else np.asarray(a, dtype=np.float64)
    b = b.detach().cpu().double().numpy() if hasattr(b, "detach") else np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def to_cuda(d):
    return {k: v.cuda() for k, v in d.items()}


def gpu_fwd_bwd(fa, x, scale, causal, backward=True):
    o, lse = fa.fwd(x["q"], x["k"], x["v"], causal=causal, scale=scale)
    out = {"o": o, "lse": lse}
    if backward:
        dq, dk, dv = fa.bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal, scale=scale)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert fa.check_device_status() == 0
    return out
