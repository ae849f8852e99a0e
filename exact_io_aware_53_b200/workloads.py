"""Seeded synthetic workloads shared by the tests, the smoke entry and the bench.

This module only draws random inputs and names shapes; it contains none of the
attention arithmetic, so the CUDA path and the CPU oracle can both be fed from
it without sharing any of the method.

Recipe (fixed so every run sees the same numbers): a torch CPU ``Generator``
seeded with ``seed``; fp32 standard normals drawn in the order q, k, v, dO,
each of shape [B, H, N, d]; q and k are multiplied by ``qk_gain`` (exact, a
power of two) and then every tensor is rounded to the workload's dtype with
round-to-nearest-even (``Tensor.to``).  The oracle runs on those rounded values.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str           # "f32" or "bf16"
    B: int
    H: int
    N: int
    d: int
    causal: bool
    backward: bool
    qk_gain: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def flops_fwd(self) -> float:
        """4*B*H*N^2*d, halved under the causal mask."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def flops_bwd(self) -> float:
        return 2.5 * self.flops_fwd()


# The five workloads the attention path is measured and checked on.
WORKLOADS = {
    "c1_f32_1x2x256x64": Workload("c1_f32_1x2x256x64", "f32", 1, 2, 256, 64, False, True, seed=1001),
    "c2_bf16_16x16x512x64": Workload("c2_bf16_16x16x512x64", "bf16", 16, 16, 512, 64, False, False, seed=1002),
    "c3_bf16_8x12x1024x64_causal": Workload("c3_bf16_8x12x1024x64_causal", "bf16", 8, 12, 1024, 64, True, True, seed=1003),
    "c4_bf16_4x16x4096x128_causal": Workload("c4_bf16_4x16x4096x128_causal", "bf16", 4, 16, 4096, 128, True, True, seed=1004),
    "c5_bf16_1x16x16384x128_causal_qk2": Workload("c5_bf16_1x16x16384x128_causal_qk2", "bf16", 1, 16, 16384, 128, True, True, qk_gain=2.0, seed=1005),
}


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """Nq queries per head against a resident cache of Nk keys and values."""
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def bytes_min(self) -> float:
        """Bytes a split-KV forward must move at least: read q, k, v (bf16),
        write o (bf16) and lse (fp32)."""
        BH = self.B * self.H
        return BH * (2.0 * self.Nq * self.d * 2 + 2.0 * self.Nk * self.d * 2 + 4.0 * self.Nq)


# Decoding shapes (one query per head against a long cache).
DECODE_WORKLOADS = {
    "decode_bf16_8x16x1x16384x128_causal": DecodeWorkload("decode_bf16_8x16x1x16384x128_causal", 8, 16, 1, 16384, 128,
                                                          True, seed=2001),
}


@dataclasses.dataclass(frozen=True)
class BlockSparseWorkload:
    """Square attention restricted to a seeded block mask over 128 x 128
    (query tile, key tile) pairs: each pair is kept with probability
    ``density``, the diagonal pairs always (no empty row), one mask shared by
    every head and batch entry."""
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    density: float
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def tiles(self) -> int:
        return (self.N + 127) // 128

    def flops(self, mask) -> float:
        """4 * 128 * 128 * d per allowed (query tile, key tile) pair and head
        (N a multiple of 128; with causal, the diagonal pairs count half)."""
        m = mask.to(torch.bool)
        if self.causal:
            m = torch.tril(m)
        pairs = float(m.sum()) - (0.5 * self.tiles if self.causal else 0.0)
        return 4.0 * 128 * 128 * self.d * pairs * self.B * self.H


BLOCKSPARSE_WORKLOADS = {
    "blocksparse_bf16_4x16x4096x128_d50": BlockSparseWorkload("blocksparse_bf16_4x16x4096x128_d50", 4, 16, 4096, 128,
                                                              False, 0.5, seed=3001),
}


def make_block_mask(w: BlockSparseWorkload, seed: int | None = None):
    """uint8 [T, T] mask: Bernoulli(density) from a torch CPU Generator, diagonal set."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    T = w.tiles
    m = torch.rand((T, T), generator=g) < w.density
    m |= torch.eye(T, dtype=torch.bool)
    return m.to(torch.uint8)


@dataclasses.dataclass(frozen=True)
class Fp8Workload:
    """Square attention with e4m3 q, k, v (one descale factor per tensor)."""
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """4*B*H*N^2*d, halved under the causal mask (the bf16 convention)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f


FP8_WORKLOADS = {
    "fp8_e4m3_4x16x4096x128_causal": Fp8Workload("fp8_e4m3_4x16x4096x128_causal", 4, 16, 4096, 128, True, seed=4001),
}


@dataclasses.dataclass(frozen=True)
class DropoutWorkload:
    """Square attention with dropout: keep probability keep_t / 256 from the
    Philox4x64-10 contract, generator key (seed, offset)."""
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    keep_t: int
    seed: int = 0
    offset: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """4*B*H*N^2*d, halved under the causal mask (dropped weights are still computed)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f


DROPOUT_WORKLOADS = {
    "dropout_bf16_4x16x4096x128_causal_keep230": DropoutWorkload("dropout_bf16_4x16x4096x128_causal_keep230", 4, 16,
                                                                 4096, 128, True, 230, seed=5001, offset=0),
}


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor e4m3 quantization of an fp32 tensor: descale = amax / 448
    (448 is e4m3's largest finite value), x8 = (x / descale) rounded to
    float8_e4m3fn.  Returns (x8, descale); x8 * descale are the values the
    attention sees."""
    amax = float(x.abs().max())
    descale = amax / 448.0 if amax > 0 else 1.0
    return (x / descale).to(torch.float8_e4m3fn), descale


def make_fp8_inputs(shape, seed: int, gain: float = 1.0):
    """q, k, v as fp32 standard normals (q, k times ``gain``) from a torch CPU
    Generator in the order q, k, v, each quantized by ``quantize_e4m3``.
    Returns {"q": q8, "k": k8, "v": v8, "descales": (dq, dk, dv)}."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn(shape, generator=g, dtype=torch.float32) * gain
    k = torch.randn(shape, generator=g, dtype=torch.float32) * gain
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    (q8, dq), (k8, dk), (v8, dv) = quantize_e4m3(q), quantize_e4m3(k), quantize_e4m3(v)
    return {"q": q8, "k": k8, "v": v8, "descales": (dq, dk, dv)}


def make_decode_inputs(w: DecodeWorkload, seed: int | None = None, B: int | None = None, H: int | None = None):
    """Draw (q, k, v) on the CPU for decode workload ``w``: fp32 standard
    normals in the order q [B,H,Nq,d], k [B,H,Nk,d], v [B,H,Nk,d], rounded to
    bf16."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    q = torch.randn((B, H, w.Nq, w.d), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, w.Nk, w.d), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, w.Nk, w.d), generator=g, dtype=torch.float32)
    return {"q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16), "v": v.to(torch.bfloat16)}


def make_inputs(w: Workload, seed: int | None = None, B: int | None = None, H: int | None = None,
                N: int | None = None):
    """Draw (q, k, v, dO) on the CPU for workload ``w`` (shape overrides allowed).

    Returns a dict of CPU tensors in the workload's dtype.
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    shape = (B, H, N, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32)
    if w.qk_gain != 1.0:
        q = q * w.qk_gain
        k = k * w.qk_gain
    dt = w.torch_dtype
    return {"q": q.to(dt), "k": k.to(dt), "v": v.to(dt), "do": do.to(dt)}


def random_tensors(shape, dtype, seed: int, count: int = 4, gain: float = 1.0):
    """``count`` seeded standard-normal tensors of ``shape`` (times ``gain``), rounded to ``dtype``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return [(torch.randn(shape, generator=g, dtype=torch.float32) * gain).to(dtype)
            for _ in range(count)]
