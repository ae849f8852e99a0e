"""Python access to the fp64 CPU attention oracle (``attn_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke entry and the bench's CPU
baseline / reference arm use this module; the CUDA library never does.  It
shares no code with the CUDA path.  The C source states what each function
computes and which passage of the FlashAttention pages it follows.

All arrays are float64, laid out [B, H, N, d] (lse: [B, H, N]).

ORACLE_LIB, when set, names a prebuilt library to load instead of building
``attn_oracle.c``: the mutation tests point it at deliberately broken builds to
check that the pins catch each mistake.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


GCC_FLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def compile_source(src: str, out: str) -> None:
    """gcc `src` into the shared library `out` with the oracle's flags."""
    tmp = out + ".tmp.%d" % os.getpid()
    subprocess.check_call(["gcc", *GCC_FLAGS, src, "-o", tmp, "-lm"])
    os.replace(tmp, out)


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (OpenMP, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        override = os.environ.get("ORACLE_LIB")
        if override:
            lib = ctypes.CDLL(override)
        else:
            build()
            lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        L = ctypes.c_long
        D = ctypes.c_double
        I = ctypes.c_int
        lib.oracle_num_threads.restype = I
        lib.oracle_softmax_naive.argtypes = [P, L, P]
        lib.oracle_softmax_online.argtypes = [P, L, L, P, P, P]
        lib.oracle_attn_fwd.argtypes = [P, P, P, P, P, L, L, L, D, I]
        lib.oracle_attn_fwd.restype = I
        lib.oracle_attn_fwd_rows.argtypes = [P, P, P, P, P, L, L, L, L, D, I]
        lib.oracle_attn_fwd_rows.restype = I
        lib.oracle_attn_fwd_rect.argtypes = [P, P, P, P, P, L, L, L, L, D, I]
        lib.oracle_attn_fwd_rect.restype = I
        U = ctypes.c_uint64
        lib.oracle_philox4x64_10.argtypes = [P, P, P]
        lib.oracle_philox4x64_10.restype = None
        lib.oracle_dropout_mask.argtypes = [P, L, L, I, U, U]
        lib.oracle_dropout_mask.restype = I
        lib.oracle_attn_fwd_dropout.argtypes = [P, P, P, P, P, L, L, L, D, I, I, U, U, L]
        lib.oracle_attn_fwd_dropout.restype = I
        lib.oracle_attn_bwd_dropout.argtypes = [P, P, P, P, P, P, P, L, L, L, D, I, I, U, U, L]
        lib.oracle_attn_bwd_dropout.restype = I
        lib.oracle_attn_fwd_blockmask.argtypes = [P, P, P, P, P, L, L, L, L, D, I, P, L, L, L]
        lib.oracle_attn_fwd_blockmask.restype = I
        lib.oracle_attn_fwd_tiled.argtypes = [P, P, P, P, P, L, L, L, D, I, L]
        lib.oracle_attn_fwd_tiled.restype = I
        lib.oracle_attn_bwd.argtypes = [P, P, P, P, P, P, P, L, L, L, D, I]
        lib.oracle_attn_bwd.restype = I
        lib.oracle_attn_bwd_dq_rows.argtypes = [P, P, P, P, P, L, L, L, L, D, I]
        lib.oracle_attn_bwd_dq_rows.restype = I
        lib.oracle_attn_bwd_kv_rows.argtypes = [P, P, P, P, P, P, L, L, L, L, D, I]
        lib.oracle_attn_bwd_kv_rows.restype = I
        lib.oracle_attn_bwd_head.argtypes = [P, P, P, P, P, P, P, L, L, D, I, I, U, U, L]
        lib.oracle_attn_bwd_head.restype = I
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact conversion of a numpy array or torch tensor (fp32 / bf16 / fp64) to C-contiguous fp64."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def softmax_naive(row):
    s = _f64(row).ravel()
    w = np.empty_like(s)
    _load().oracle_softmax_naive(_ptr(s), s.size, _ptr(w))
    return w


def softmax_online(row, block: int):
    """Returns (weights, m after each block, l after each block)."""
    s = _f64(row).ravel()
    nb = -(-s.size // block)
    w = np.empty_like(s)
    mt = np.empty(nb)
    lt = np.empty(nb)
    _load().oracle_softmax_online(_ptr(s), s.size, block, _ptr(w), _ptr(mt), _ptr(lt))
    return w, mt, lt


def _check4(q, k, v):
    q, k, v = _f64(q), _f64(k), _f64(v)
    assert q.ndim == 4 and q.shape == k.shape == v.shape, (q.shape, k.shape, v.shape)
    return q, k, v


def attn_fwd(q, k, v, scale: float, causal: bool):
    """Exact attention forward.  Returns (O [B,H,N,d], LSE [B,H,N])."""
    q, k, v = _check4(q, k, v)
    B, H, N, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, N))
    rc = _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                 B * H, N, d, float(scale), int(bool(causal)))
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd failed (%d)" % rc)
    return o, lse


def attn_fwd_rect(q, k, v, scale: float, causal: bool):
    """Nq queries against Nk keys: q [B,H,Nq,d], k and v [B,H,Nk,d].  Causal:
    query i sees keys j <= Nk - Nq + i (needs Nk >= Nq).  Returns (O, LSE)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    assert k.shape == (B, H, Nk, d) and v.shape == k.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, Nq))
    rc = _load().oracle_attn_fwd_rect(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                      B * H, Nq, Nk, d, float(scale), int(bool(causal)))
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd_rect failed (%d)" % rc)
    return o, lse


def attn_fwd_blockmask(q, k, v, scale: float, causal: bool, mask, br: int = 128, bc: int = 128):
    """Square attention restricted to a block mask: q, k, v [B,H,N,d]; mask
    uint8-like [Hm, ceil(N/br), ceil(N/bc)] with Hm = 1 (shared) or H.  Key j is
    allowed for query i iff mask[h, i // br, j // bc] and (not causal or
    j <= i).  Rows with no allowed key: O = 0, LSE = -inf.  Returns (O, LSE)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    assert k.shape == q.shape and v.shape == q.shape
    m = np.ascontiguousarray(np.asarray(mask.cpu() if hasattr(mask, "cpu") else mask) != 0, dtype=np.uint8)
    if m.ndim == 2:
        m = m[None]
    nqb, nkb = -(-N // br), -(-N // bc)
    assert m.shape[1:] == (nqb, nkb) and m.shape[0] in (1, H), m.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, N))
    rc = _load().oracle_attn_fwd_blockmask(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B * H, H, N, d,
                                           float(scale), int(bool(causal)), m.ctypes.data_as(ctypes.c_void_p),
                                           0 if m.shape[0] == 1 else nqb * nkb, br, bc)
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd_blockmask failed (%d)" % rc)
    return o, lse


def philox4x64_10(counter, key):
    """Philox4x64-10 of a 4-word counter under a 2-word key -> 4 uint64 words."""
    c = np.ascontiguousarray(counter, dtype=np.uint64)
    k = np.ascontiguousarray(key, dtype=np.uint64)
    out = np.zeros(4, dtype=np.uint64)
    _load().oracle_philox4x64_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def dropout_mask(bh: int, N: int, keep_t: int, seed: int, offset: int):
    """uint8 [N, N] keep mask of head bh (1 = kept) under the dropout contract."""
    z = np.zeros((N, N), dtype=np.uint8)
    rc = _load().oracle_dropout_mask(_ptr(z), bh, N, int(keep_t), int(seed), int(offset))
    if rc != 0:
        raise RuntimeError("oracle_dropout_mask failed (%d)" % rc)
    return z


def attn_fwd_dropout(q, k, v, scale: float, causal: bool, keep_t: int, seed: int, offset: int, bh0: int = 0):
    """Forward with dropout: keep probability keep_t / 256, kept weights x 256 / keep_t.
    The heads given are heads bh0, bh0 + 1, ... (b * H + h) of the whole problem.
    Returns (O, LSE); LSE is that of the undropped softmax."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, N))
    rc = _load().oracle_attn_fwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B * H, N, d,
                                         float(scale), int(bool(causal)), int(keep_t), int(seed), int(offset),
                                         int(bh0))
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd_dropout failed (%d)" % rc)
    return o, lse


def attn_bwd_dropout(q, k, v, do, scale: float, causal: bool, keep_t: int, seed: int, offset: int, bh0: int = 0):
    """(dQ, dK, dV) of L = sum(O * dO) for the dropout forward above; the heads
    given are heads bh0, bh0 + 1, ... of the whole problem."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = _load().oracle_attn_bwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                                         B * H, N, d, float(scale), int(bool(causal)), int(keep_t), int(seed),
                                         int(offset), int(bh0))
    if rc != 0:
        raise RuntimeError("oracle_attn_bwd_dropout failed (%d)" % rc)
    return dq, dk, dv


def attn_fwd_rows(q, k, v, i0: int, i1: int, scale: float, causal: bool):
    """Rows [i0, i1) of ONE head; q, k, v are that head's [N, d] arrays."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, d = q.shape
    o = np.empty((i1 - i0, d))
    lse = np.empty(i1 - i0)
    rc = _load().oracle_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                      N, d, i0, i1, float(scale), int(bool(causal)))
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd_rows failed (%d)" % rc)
    return o, lse


def attn_fwd_tiled(q, k, v, scale: float, causal: bool, block: int):
    """The online-softmax restatement with key block size ``block``."""
    q, k, v = _check4(q, k, v)
    B, H, N, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, N))
    rc = _load().oracle_attn_fwd_tiled(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                       B * H, N, d, float(scale), int(bool(causal)), int(block))
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd_tiled failed (%d)" % rc)
    return o, lse


def attn_bwd(q, k, v, do, scale: float, causal: bool):
    """Exact attention backward for L = sum(O * dO).  Returns (dQ, dK, dV)."""
    q, k, v = _check4(q, k, v)
    do = _f64(do)
    assert do.shape == q.shape
    B, H, N, d = q.shape
    dq = np.empty_like(q)
    dk = np.empty_like(q)
    dv = np.empty_like(q)
    rc = _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk),
                                 _ptr(dv), B * H, N, d, float(scale), int(bool(causal)))
    if rc != 0:
        raise RuntimeError("oracle_attn_bwd failed (%d)" % rc)
    return dq, dk, dv


def attn_bwd_dq_rows(q, k, v, do, i0: int, i1: int, scale: float, causal: bool):
    """dQ rows [i0, i1) of ONE head; q, k, v, do are that head's [N, d] arrays."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    N, d = q.shape
    dq = np.empty((i1 - i0, d))
    rc = _load().oracle_attn_bwd_dq_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), N, d, i0, i1,
                                         float(scale), int(bool(causal)))
    if rc != 0:
        raise RuntimeError("oracle_attn_bwd_dq_rows failed (%d)" % rc)
    return dq


def attn_bwd_kv_rows(q, k, v, do, j0: int, j1: int, scale: float, causal: bool):
    """(dK, dV) rows [j0, j1) of ONE head; q, k, v, do are that head's [N, d] arrays."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    N, d = q.shape
    dk = np.empty((j1 - j0, d))
    dv = np.empty((j1 - j0, d))
    rc = _load().oracle_attn_bwd_kv_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dk), _ptr(dv), N, d,
                                         j0, j1, float(scale), int(bool(causal)))
    if rc != 0:
        raise RuntimeError("oracle_attn_bwd_kv_rows failed (%d)" % rc)
    return dk, dv


def attn_bwd_head(q, k, v, do, scale: float, causal: bool, keep_t: int = 256, seed: int = 0, offset: int = 0,
                  bh: int = 0):
    """(dQ, dK, dV) of ONE head ([N, d] arrays), the work spread over threads
    (rows, then keys).  keep_t = 256: plain attention, as attn_bwd; otherwise
    the dropout backward of head index bh (b * H + h) of the whole problem."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    N, d = q.shape
    assert k.shape == v.shape == do.shape == (N, d)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = _load().oracle_attn_bwd_head(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), N, d,
                                      float(scale), int(bool(causal)), int(keep_t), int(seed), int(offset), int(bh))
    if rc != 0:
        raise RuntimeError("oracle_attn_bwd_head failed (%d)" % rc)
    return dq, dk, dv
