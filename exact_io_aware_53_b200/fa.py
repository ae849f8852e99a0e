"""Python binding of the C ABI in ``include/fa.h`` (argument marshalling only).

Every step of attention runs in the CUDA library ``libfa_sm100.so``; this
module checks torch tensors, passes their device pointers and the current
stream, and turns status codes into exceptions.  Importing it fails loudly if
the library has not been built: there is no fallback path.

``check_build()`` returns the same binding over ``libfa_sm100_check.so``, the
build with jittered barrier waits and tested tile coordinates that the
race-stress tests run.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# "check" when this module object was made by check_build() (set before the
# module's code runs); the ordinary import binds the release library
VARIANT = globals().get("VARIANT", "")
LIB_PATH = os.path.join(_PKG, "libfa_sm100_check.so" if VARIANT == "check" else "libfa_sm100.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("%s is not built; run `python -m exact_io_aware_53_b200.build%s` "
                      "(or __graft_entry__.build()) first" % (os.path.basename(LIB_PATH),
                                                               " --check" if VARIANT == "check" else ""))

_lib = ctypes.CDLL(LIB_PATH)

P = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
SZ = ctypes.c_size_t

_SIGS = {
    "fa_fwd": ([P, P, P, P, P, I, I, I, I, F, I, P], I),
    "fa_bwd_workspace_bytes": ([I, I, I, I], SZ),
    "fa_bwd": ([P, P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P], I),
    "fa_bwd_prep": ([P, P, P, P, P, I, I, I, I, P], I),
    "fa_bwd_main": ([P, P, P, P, P, P, P, P, I, I, I, I, F, I, P], I),
    "fa_bwd_noalloc": ([P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P], I),
    "fa_fwd_f32": ([P, P, P, P, P, I, I, I, I, F, I, I, P], I),
    "fa_bwd_f32": ([P, P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, I, P], I),
    "fa_attention_host_arena_bytes": ([I, I, I, I], SZ),
    "fa_attention_host": ([P, P, P, P, P, P, P, P, P, P, SZ, I, I, I, I, F, I, P], I),
    "fa_check_device_status": ([P], I),
    "fa_set_wait_limit_ns": ([ctypes.c_ulonglong], None),
    "fa_set_fwd_queue_words": ([I], I),
    "fa_set_bwd_softmax_warps": ([I], I),
    "fa_fwd_splitkv_workspace_bytes": ([I, I, I, I, I, I], ctypes.c_size_t),
    "fa_fwd_splitkv": ([P, P, P, P, P, P, I, I, I, I, I, ctypes.c_float, I, I, P], I),
    "fa_fwd_blocksparse": ([P, P, P, P, P, P, ctypes.c_longlong, I, I, I, I, ctypes.c_float, I, P], I),
    "fa_fwd_fp8": ([P, P, P, P, P, ctypes.c_float, ctypes.c_float, ctypes.c_float, I, I, I, I, ctypes.c_float, I, P],
                   I),
    "fa_fwd_dropout": ([P, P, P, P, P, I, I, I, I, ctypes.c_float, I, I, ctypes.c_ulonglong, ctypes.c_ulonglong, P],
                       I),
    "fa_bwd_dropout": ([P, P, P, P, P, P, P, P, P, P, I, I, I, I, ctypes.c_float, I, I, ctypes.c_ulonglong,
                        ctypes.c_ulonglong, P], I),
    "fa_status_string": ([I], ctypes.c_char_p),
    "fa_last_launch_count": ([], I),
    "fa_last_cuda_error": ([], I),
    "fa_cuda_error_string": ([I], ctypes.c_char_p),
    "fa_selftest_umma": ([P, P, P, I, I, I, I, I, I, I, P], I),
    "fa_selftest_exp2": ([P, P, I, I, P], I),
    "fa_selftest_wait_timeout": ([ctypes.c_ulonglong, P, P], I),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_MISALIGNED = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = "%s: %s" % (what, _lib.fa_status_string(status).decode())
        if status == FA_ERR_CUDA:
            code = int(_lib.fa_last_cuda_error())
            msg += " (CUDA error %d: %s)" % (code, _lib.fa_cuda_error_string(code).decode())
        super().__init__(msg)


def _check(status: int, what: str):
    if status != FA_OK:
        raise FAError(status, what)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def exported_symbols():
    return list(_SIGS)


_check_module = None


def check_build():
    """This binding over the check build (libfa_sm100_check.so): the same kernels
    compiled with FA_CHECK_BUILD, whose bounded waits sleep a pseudo-random
    0-2 us once in four after they succeed and whose tile copies test their
    coordinates first (a bad one raises the device error word instead of being
    issued).  A separate module object with the same functions; loaded once."""
    global _check_module
    if VARIANT == "check":
        return globals()["__check_self__"]
    if _check_module is None:
        import importlib.util
        spec = importlib.util.spec_from_file_location(__name__ + "_check", __file__)
        mod = importlib.util.module_from_spec(spec)
        mod.VARIANT = "check"
        mod.__check_self__ = mod
        spec.loader.exec_module(mod)
        _check_module = mod
    return _check_module


def status_string(status: int) -> str:
    return _lib.fa_status_string(status).decode()


def last_launch_count() -> int:
    return int(_lib.fa_last_launch_count())


def set_wait_limit_ns(ns: int):
    _lib.fa_set_wait_limit_ns(int(ns))


def check_device_status(stream=None) -> int:
    return int(_lib.fa_check_device_status(_stream(stream)))


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _same(*ts, dtype):
    ref = ts[0]
    for t in ts:
        if t.shape != ref.shape or t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA %s of shape %s" % (dtype, tuple(ref.shape)))


# ------------------------------------------------------------------ bf16 path

def fwd_raw(q, k, v, o, lse, scale: float, causal: bool, stream=None) -> int:
    B, H, N, d = _shape(q)
    return _lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale), int(causal),
                       _stream(stream))


def splitkv_workspace_bytes(B: int, H: int, Nq: int, Nk: int, d: int, n_split: int = 0) -> int:
    return int(_lib.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, int(n_split)))


def fwd_splitkv_raw(q, k, v, o, lse, workspace, scale: float, causal: bool, n_split: int = 0, stream=None) -> int:
    """Enqueue the split-KV forward on preallocated tensors; returns the status code."""
    B, H, Nq, d = (int(x) for x in q.shape)
    return _lib.fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(workspace), B, H, Nq,
                               int(k.shape[2]), d, float(scale), int(bool(causal)), int(n_split), _stream(stream))


def fwd_splitkv(q, k, v, causal: bool = False, scale: float | None = None, n_split: int = 0, stream=None):
    """O, LSE for Nq queries against Nk keys: q bf16 [B,H,Nq,d], k and v bf16
    [B,H,Nk,d].  Causal: query i sees keys j <= Nk - Nq + i.  n_split key
    ranges are processed in parallel and merged (0: the library picks)."""
    _same(q, dtype=torch.bfloat16)
    _same(k, v, dtype=torch.bfloat16)
    B, H, Nq, d = (int(x) for x in q.shape)
    Nk = int(k.shape[2])
    if tuple(k.shape) != (B, H, Nk, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B, H, Nk, d] with q's B, H, d")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    ws = torch.empty(max(splitkv_workspace_bytes(B, H, Nq, Nk, d, n_split), 16), dtype=torch.uint8,
                     device=q.device)
    _check(fwd_splitkv_raw(q, k, v, o, lse, ws, scale, causal, n_split, stream), "fa_fwd_splitkv")
    return o, lse


def _check_mask(m, H: int, N: int, device):
    """The kernel reads mask row i of head h at h * stride + i * T: the mask must be
    a uint8 tensor [T, T] or [1 or H, T, T] on the same GPU as q whose last two
    dimensions are dense."""
    T = (N + 127) // 128
    shape = tuple(m.shape)
    ok = (m.dtype == torch.uint8 and m.is_cuda and m.device == device and
          (shape == (T, T) or (m.dim() == 3 and shape[1:] == (T, T) and shape[0] in (1, H))) and
          m.stride(-1) == 1 and m.stride(-2) == T)
    if not ok:
        raise ValueError("block_mask must be a uint8 tensor [T, T] or [1 or H, T, T] with dense rows on %s, "
                         "T = ceil(N / 128) = %d; got %s %s strides %s on %s"
                         % (device, T, m.dtype, shape, tuple(m.stride()), m.device))


def fwd_blocksparse_raw(q, k, v, o, lse, block_mask, scale: float, causal: bool, stream=None) -> int:
    """Enqueue the block-sparse forward on preallocated tensors; block_mask is
    a CUDA uint8 tensor [T, T] (shared by every head) or [H, T, T], T = ceil(N/128)."""
    B, H, N, d = _shape(q)
    _check_mask(block_mask, H, N, q.device)
    stride = 0 if block_mask.dim() == 2 or block_mask.shape[0] == 1 else int(block_mask.stride(0))
    return _lib.fa_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(block_mask), stride,
                                   B, H, N, d, float(scale), int(bool(causal)), _stream(stream))


def fwd_blocksparse(q, k, v, block_mask, causal: bool = False, scale: float | None = None, stream=None):
    """O, LSE of attention restricted to the allowed (128-query, 128-key) tile
    pairs of block_mask (bool or uint8, [T, T] or [H, T, T], T = ceil(N/128))."""
    _same(q, k, v, dtype=torch.bfloat16)
    B, H, N, d = _shape(q)
    T = (N + 127) // 128
    m = block_mask
    if m.dim() == 2:
        m = m.unsqueeze(0)
    if m.dim() != 3 or tuple(m.shape[1:]) != (T, T) or m.shape[0] not in (1, H):
        raise ValueError("block_mask must be [T, T] or [H, T, T] with T = ceil(N / 128) = %d" % T)
    m = m.to(device=q.device, dtype=torch.uint8).contiguous()
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check(fwd_blocksparse_raw(q, k, v, o, lse, m, scale, causal, stream), "fa_fwd_blocksparse")
    return o, lse


def fwd_dropout_raw(q, k, v, o, lse, scale: float, causal: bool, keep_t: int, seed: int, offset: int = 0,
                    stream=None) -> int:
    """Enqueue the dropout forward on preallocated tensors (keep probability keep_t / 256)."""
    B, H, N, d = _shape(q)
    return _lib.fa_fwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                               int(bool(causal)), int(keep_t), int(seed), int(offset), _stream(stream))


def fwd_dropout(q, k, v, keep_t: int, seed: int, offset: int = 0, causal: bool = False, scale: float | None = None,
                stream=None):
    """O, LSE with dropout: weights kept with probability keep_t / 256 (Philox4x64-10
    mask from (seed, offset)) and scaled by 256 / keep_t; LSE of the undropped softmax."""
    _same(q, k, v, dtype=torch.bfloat16)
    B, H, N, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check(fwd_dropout_raw(q, k, v, o, lse, scale, causal, keep_t, seed, offset, stream), "fa_fwd_dropout")
    return o, lse


def bwd_dropout_raw(q, k, v, o, lse, do, dq, dk, dv, ws, scale: float, causal: bool, keep_t: int, seed: int,
                    offset: int = 0, stream=None) -> int:
    """Enqueue the dropout backward on preallocated tensors (ws: bwd_workspace_bytes)."""
    B, H, N, d = _shape(q)
    return _lib.fa_bwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                               _ptr(dv), _ptr(ws), B, H, N, d, float(scale), int(bool(causal)), int(keep_t),
                               int(seed), int(offset), _stream(stream))


def bwd_dropout(q, k, v, o, lse, do, keep_t: int, seed: int, offset: int = 0, causal: bool = False,
                scale: float | None = None, stream=None):
    """dQ, dK, dV (fp32) of L = sum(O * dO) for fwd_dropout's O with the same
    keep_t, seed and offset; the keep mask is regenerated, not stored."""
    _same(q, k, v, o, do, dtype=torch.bfloat16)
    B, H, N, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty_like(dq)
    dv = torch.empty_like(dq)
    ws = torch.empty(max(1, bwd_workspace_bytes(B, H, N, d)), dtype=torch.uint8, device=q.device)
    _check(bwd_dropout_raw(q, k, v, o, lse, do, dq, dk, dv, ws, scale, causal, keep_t, seed, offset, stream),
           "fa_bwd_dropout")
    return dq, dk, dv


def fwd_fp8_raw(q, k, v, o, lse, descales, scale: float, causal: bool, stream=None) -> int:
    """Enqueue the e4m3 forward on preallocated tensors; descales = (q, k, v) factors."""
    B, H, N, d = _shape(q)
    qd, kd, vd = (float(x) for x in descales)
    return _lib.fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), qd, kd, vd, B, H, N, d, float(scale),
                           int(bool(causal)), _stream(stream))


def fwd_fp8(q, k, v, descales=(1.0, 1.0, 1.0), causal: bool = False, scale: float | None = None, stream=None):
    """O (bf16), LSE for e4m3 q, k, v [B,H,N,128] whose values are x * descale."""
    _same(q, k, v, dtype=torch.float8_e4m3fn)
    B, H, N, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check(fwd_fp8_raw(q, k, v, o, lse, descales, scale, causal, stream), "fa_fwd_fp8")
    return o, lse


def fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None, stream=None):
    """O, LSE = attention(q, k, v); bf16 [B,H,N,d] in, bf16 O and fp32 LSE [B,H,N] out."""
    _same(q, k, v, dtype=torch.bfloat16)
    B, H, N, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(fwd_raw(q, k, v, o, lse, scale, causal, stream), "fa_fwd")
    return o, lse


def bwd_workspace_bytes(B, H, N, d) -> int:
    return int(_lib.fa_bwd_workspace_bytes(B, H, N, d))


def bwd_raw(q, k, v, o, lse, do, dq, dk, dv, ws, scale: float, causal: bool, stream=None) -> int:
    B, H, N, d = _shape(q)
    return _lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                       _ptr(ws), B, H, N, d, float(scale), int(causal), _stream(stream))


def bwd_prep_raw(o, lse, do, dq, ws, stream=None) -> int:
    B, H, N, d = _shape(o)
    return _lib.fa_bwd_prep(_ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(ws), B, H, N, d, _stream(stream))


def bwd_main_raw(q, k, v, do, dq, dk, dv, ws, scale: float, causal: bool, stream=None) -> int:
    B, H, N, d = _shape(q)
    return _lib.fa_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                            B, H, N, d, float(scale), int(causal), _stream(stream))


def bwd(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None, workspace=None, stream=None):
    """dQ, dK, dV (fp32) of L = sum(O * dO), recomputing the weights from lse."""
    _same(q, k, v, o, do, dtype=torch.bfloat16)
    B, H, N, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty_like(dq)
    dv = torch.empty_like(dq)
    if workspace is None:
        workspace = torch.empty(bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=q.device)
    _check(bwd_raw(q, k, v, o, lse, do, dq, dk, dv, workspace, scale, causal, stream), "fa_bwd")
    return dq, dk, dv


def bwd_noalloc_raw(q, k, v, o, lse, do, dq, dk, dv, scale: float, causal: bool, stream=None) -> int:
    """fa_bwd without a workspace argument: the library's built-in scratch area is used."""
    B, H, N, d = _shape(q)
    return _lib.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                               _ptr(dv), B, H, N, d, float(scale), int(causal), _stream(stream))


# ------------------------------------------------------------------ fp32 path

def fwd_f32(q, k, v, causal: bool = False, scale: float | None = None, block_k: int = 0, stream=None):
    _same(q, k, v, dtype=torch.float32)
    B, H, N, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check(_lib.fa_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale), int(causal),
                           int(block_k), _stream(stream)), "fa_fwd_f32")
    return o, lse


def bwd_f32(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None, block_k: int = 0,
            stream=None):
    _same(q, k, v, o, do, dtype=torch.float32)
    B, H, N, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq = torch.empty_like(q)
    dk = torch.empty_like(q)
    dv = torch.empty_like(q)
    ws = torch.empty(bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=q.device)
    _check(_lib.fa_bwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                           _ptr(ws), B, H, N, d, float(scale), int(causal), int(block_k), _stream(stream)),
           "fa_bwd_f32")
    return dq, dk, dv


# ------------------------------------------------------------------ host-buffer step

def attention_host_arena_bytes(B, H, N, d) -> int:
    return int(_lib.fa_attention_host_arena_bytes(B, H, N, d))


def attention_host(hq, hk, hv, hdo, arena, outs, causal: bool, scale: float | None = None, stream=None) -> None:
    """Forward + backward from host (pinned) bf16 tensors; ``outs`` = dict of host
    tensors o (bf16), lse, dq, dk, dv (fp32), any may be missing.  Enqueues only."""
    B, H, N, d = _shape(hq)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    g = outs.get
    _check(_lib.fa_attention_host(_ptr(hq), _ptr(hk), _ptr(hv), _ptr(hdo), _ptr(g("o")), _ptr(g("lse")),
                                  _ptr(g("dq")), _ptr(g("dk")), _ptr(g("dv")), _ptr(arena),
                                  arena.numel() * arena.element_size(), B, H, N, d, float(scale), int(causal),
                                  _stream(stream)), "fa_attention_host")


# ------------------------------------------------------------------ diagnostics

def selftest_umma(a, b, M, N, K, a_mn, b_mn, a_tmem=False, b_manual=False, stream=None):
    d = torch.empty((M, N), dtype=torch.float32, device=a.device)
    _check(_lib.fa_selftest_umma(_ptr(a), _ptr(b), _ptr(d), M, N, K, int(a_mn), int(b_mn), int(a_tmem),
                                 int(b_manual), _stream(stream)), "fa_selftest_umma")
    return d




def selftest_exp2(x, mode: int, stream=None):
    """2^x on the GPU by the FMA-pipe polynomial (mode 0) or ex2.approx (mode 1)."""
    y = torch.empty_like(x)
    _check(_lib.fa_selftest_exp2(_ptr(x), _ptr(y), x.numel(), int(mode), _stream(stream)), "fa_selftest_exp2")
    return y


def selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    """Runs the bounded-wait failure check; returns how many lanes gave up."""
    gave_up = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(_lib.fa_selftest_wait_timeout(int(limit_ns), _ptr(gave_up), _stream(stream)), "fa_selftest_wait_timeout")
    torch.cuda.synchronize()
    return int(gave_up.item())
