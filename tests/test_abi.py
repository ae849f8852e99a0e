"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments before touching the GPU (runs without a GPU)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_53_b200 import build
    build.build()
    from exact_io_aware_53_b200 import fa
    return fa


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?(?:int|void|size_t|char)\s*\*?\s*(fa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "fa_fwd" in names and "fa_bwd" in names and "fa_selftest_umma" in names
    so = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(so, n), n
    assert set(names) == set(lib.exported_symbols())


def test_check_build_exports_the_same_entry_points(lib):
    """The check build (jittered waits, tested tile coordinates) is the same
    interface: every declared symbol, loaded as a second binding."""
    from exact_io_aware_53_b200 import build
    build.build(check=True)
    chk = lib.check_build()
    assert chk is not lib and chk.LIB_PATH != lib.LIB_PATH
    assert chk.LIB_PATH.endswith("libfa_sm100_check.so")
    so = ctypes.CDLL(chk.LIB_PATH)
    for n in _declared():
        assert hasattr(so, n), n
    assert chk.status_string(5) == lib.status_string(5)


def test_status_strings(lib):
    assert lib.status_string(0) == "FA_OK"
    assert lib.status_string(5) == "FA_ERR_TIMEOUT"
    assert lib.status_string(99) == "FA_ERR_UNKNOWN"


def test_cuda_error_diagnostics(lib):
    # argument errors record no CUDA error; the description table needs no GPU
    assert _fwd(lib, q=0) == lib.FA_ERR_INVALID_ARG
    assert lib._lib.fa_last_cuda_error() == 0
    assert lib._lib.fa_cuda_error_string(0).decode() == "no error"
    assert "resources" in lib._lib.fa_cuda_error_string(701).decode()


def _fwd(lib, q=16, k=16, v=16, o=16, lse=16, B=1, H=1, N=8, d=64, scale=0.125, causal=0):
    P = ctypes.c_void_p
    return lib._lib.fa_fwd(P(q), P(k), P(v), P(o), P(lse), B, H, N, d, scale, causal, P(0))


def test_fwd_argument_errors_are_returned_before_any_launch(lib):
    assert _fwd(lib, q=0) == lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, N=0) == lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, B=-1) == lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, causal=2) == lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=0.0) == lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=-1.0) == lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, d=96) == lib.FA_ERR_UNSUPPORTED
    assert _fwd(lib, d=256) == lib.FA_ERR_UNSUPPORTED
    assert _fwd(lib, B=1 << 12, H=1 << 12, N=1 << 12, d=64) == lib.FA_ERR_UNSUPPORTED
    assert _fwd(lib, k=24) == lib.FA_ERR_MISALIGNED
    assert _fwd(lib, lse=20) == lib.FA_ERR_MISALIGNED


def test_bwd_argument_errors(lib):
    P = ctypes.c_void_p
    good = [P(16)] * 10
    args = lambda ptrs, d=128, N=8: (*ptrs, 1, 1, N, d, 0.1, 1, P(0))
    assert lib._lib.fa_bwd(*args(good[:9] + [P(0)])) == lib.FA_ERR_INVALID_ARG
    assert lib._lib.fa_bwd(*args(good, d=32)) == lib.FA_ERR_UNSUPPORTED
    assert lib._lib.fa_bwd(*args(good[:5] + [P(8)] + good[6:])) == lib.FA_ERR_MISALIGNED


def test_f32_argument_errors(lib):
    P = ctypes.c_void_p
    f = lib._lib.fa_fwd_f32
    assert f(P(16), P(16), P(16), P(16), P(16), 1, 1, 8, 129, 0.1, 0, 0, P(0)) == lib.FA_ERR_UNSUPPORTED
    assert f(P(16), P(16), P(16), P(16), P(16), 1, 1, 8, 64, 0.1, 0, 2000, P(0)) == lib.FA_ERR_INVALID_ARG
    assert f(P(16), P(16), P(16), P(16), P(16), 1, 1, 8, 64, 0.1, 0, -1, P(0)) == lib.FA_ERR_INVALID_ARG
    assert f(P(0), P(16), P(16), P(16), P(16), 1, 1, 8, 64, 0.1, 0, 0, P(0)) == lib.FA_ERR_INVALID_ARG


def test_workspace_is_linear_in_sequence_length(lib):
    # two fp32 row vectors per head, padded to 128 rows and 256 bytes: O(N), never O(N^2)
    for B, H, N, d in [(1, 1, 1, 64), (4, 16, 4096, 128), (1, 16, 16384, 128), (2, 3, 300, 64)]:
        rows = B * H * (-(-N // 128) * 128)
        assert lib.bwd_workspace_bytes(B, H, N, d) == 2 * (-(-rows * 4 // 256) * 256) + 256
    assert lib.bwd_workspace_bytes(0, 1, 1, 64) == 0


def test_host_arena_size(lib):
    B, H, N, d = 2, 3, 300, 64
    E, R = B * H * N * d, B * H * N
    up = lambda x: -(-x // 256) * 256
    want = 5 * up(E * 2) + 3 * up(E * 4) + up(R * 4) + up(lib.bwd_workspace_bytes(B, H, N, d))
    assert lib.attention_host_arena_bytes(B, H, N, d) == want


def test_selftest_argument_errors(lib):
    P = ctypes.c_void_p
    f = lib._lib.fa_selftest_umma
    assert f(P(16), P(16), P(16), 64, 64, 64, 0, 0, 0, 0, P(0)) == lib.FA_ERR_UNSUPPORTED
    assert f(P(16), P(16), P(16), 128, 64, 64, 1, 0, 1, 0, P(0)) == lib.FA_ERR_UNSUPPORTED
    assert f(P(0), P(16), P(16), 128, 64, 64, 0, 0, 0, 0, P(0)) == lib.FA_ERR_INVALID_ARG


def test_splitkv_argument_errors(lib):
    f = lib._lib.fa_fwd_splitkv
    P = ctypes.c_void_p
    ptrs = [P(16)] * 6

    def call(B=1, H=1, Nq=1, Nk=256, d=128, scale=0.1, causal=0, n_split=0):
        return f(*ptrs, B, H, Nq, Nk, d, scale, causal, n_split, P(0))

    assert f(P(0), *ptrs[1:], 1, 1, 1, 256, 128, 0.1, 0, 0, P(0)) == lib.FA_ERR_INVALID_ARG
    assert call(Nq=0) == lib.FA_ERR_INVALID_ARG
    assert call(Nk=0) == lib.FA_ERR_INVALID_ARG
    assert call(n_split=-1) == lib.FA_ERR_INVALID_ARG
    assert call(causal=1, Nq=300, Nk=299) == lib.FA_ERR_INVALID_ARG
    assert call(causal=2) == lib.FA_ERR_INVALID_ARG
    assert call(d=96) == lib.FA_ERR_UNSUPPORTED
    assert call(B=300, H=300) == lib.FA_ERR_UNSUPPORTED
    assert f(*ptrs[:5], P(8), 1, 1, 1, 256, 128, 0.1, 0, 0, P(0)) == lib.FA_ERR_MISALIGNED


def test_splitkv_workspace_size(lib):
    ws = lib._lib.fa_fwd_splitkv_workspace_bytes
    # explicit n_split needs no device: ranges are clipped to the 128-key tiles
    assert ws(2, 3, 5, 1000, 128, 4) == ((4 * 2 * 3 * 5 * 128 * 4 + 255) // 256 + (4 * 2 * 3 * 5 * 4 + 255) // 256) * 256
    assert ws(1, 1, 1, 100, 64, 8) == ws(1, 1, 1, 100, 64, 1)  # one tile: one range
    assert ws(1, 1, 0, 100, 64, 1) == 0
    assert ws(1, 1, 1, 100, 64, -1) == 0


def test_blocksparse_argument_errors(lib):
    f = lib._lib.fa_fwd_blocksparse
    P = ctypes.c_void_p

    def call(B=1, H=1, N=256, d=128, scale=0.1, causal=0, stride=0, mask=P(16), q=P(16)):
        return f(q, P(16), P(16), P(16), P(16), mask, stride, B, H, N, d, scale, causal, P(0))

    assert call(q=P(0)) == lib.FA_ERR_INVALID_ARG
    assert call(mask=P(0)) == lib.FA_ERR_INVALID_ARG
    assert call(N=0) == lib.FA_ERR_INVALID_ARG
    assert call(stride=-1) == lib.FA_ERR_INVALID_ARG
    assert call(causal=3) == lib.FA_ERR_INVALID_ARG
    assert call(d=32) == lib.FA_ERR_UNSUPPORTED
    assert call(N=2048 * 128 + 1, d=64) == lib.FA_ERR_UNSUPPORTED   # more than 2048 key tiles
    assert call(q=P(24)) == lib.FA_ERR_MISALIGNED


def test_fp8_argument_errors(lib):
    f = lib._lib.fa_fwd_fp8
    P = ctypes.c_void_p

    def call(B=1, H=1, N=256, d=128, scale=0.1, causal=0, ds=(1.0, 1.0, 1.0), q=P(16)):
        return f(q, P(16), P(16), P(16), P(16), ds[0], ds[1], ds[2], B, H, N, d, scale, causal, P(0))

    assert call(q=P(0)) == lib.FA_ERR_INVALID_ARG
    assert call(N=0) == lib.FA_ERR_INVALID_ARG
    assert call(ds=(0.0, 1.0, 1.0)) == lib.FA_ERR_INVALID_ARG
    assert call(ds=(1.0, float("inf"), 1.0)) == lib.FA_ERR_INVALID_ARG
    assert call(ds=(1.0, 1.0, -2.0)) == lib.FA_ERR_INVALID_ARG
    assert call(ds=(1e30, 1e30, 1.0)) == lib.FA_ERR_INVALID_ARG   # scale * descales overflows
    assert call(d=64) == lib.FA_ERR_UNSUPPORTED
    assert call(q=P(8)) == lib.FA_ERR_MISALIGNED


def test_dropout_argument_errors(lib):
    f = lib._lib.fa_fwd_dropout
    P = ctypes.c_void_p

    def call(B=1, H=1, N=256, d=128, scale=0.1, causal=0, t=230, q=P(16)):
        return f(q, P(16), P(16), P(16), P(16), B, H, N, d, scale, causal, t, 1, 0, P(0))

    assert call(q=P(0)) == lib.FA_ERR_INVALID_ARG
    assert call(t=-1) == lib.FA_ERR_INVALID_ARG
    assert call(t=257) == lib.FA_ERR_INVALID_ARG
    assert call(N=0) == lib.FA_ERR_INVALID_ARG
    assert call(d=80) == lib.FA_ERR_UNSUPPORTED
    assert call(q=P(4)) == lib.FA_ERR_MISALIGNED


def test_blocksparse_mask_layout_is_checked(lib):
    """A mask whose rows are not dense (a transposed view) or of the wrong dtype
    or shape is refused before the library is called."""
    import torch
    m = torch.ones((4, 4), dtype=torch.uint8)
    for bad in (m.t().contiguous().t()[:, :3], m.to(torch.int32), torch.ones((2, 4, 4), dtype=torch.uint8).transpose(1, 2),
                torch.ones((3, 3), dtype=torch.uint8)):
        with pytest.raises(ValueError):
            lib._check_mask(bad, 2, 512, torch.device("cuda", 0))
    with pytest.raises(ValueError):  # not on a GPU
        lib._check_mask(m, 2, 512, torch.device("cuda", 0))


def test_blocksparse_mask_layout_accepts_dense_device_masks(lib):
    """The accepting side of the check, with stand-ins that report a device
    tensor's dtype, shape and strides (no GPU here)."""
    import torch

    class DeviceView:
        def __init__(self, t, index=0):
            self._t, self.dtype, self.is_cuda = t, t.dtype, True
            self.shape = t.shape
            self.device = torch.device("cuda", index)

        def dim(self):
            return self._t.dim()

        def stride(self, i=None):
            return self._t.stride() if i is None else self._t.stride(i)

    T = 4  # N = 512
    dev = torch.device("cuda", 0)
    for good in (torch.ones((T, T), dtype=torch.uint8), torch.ones((1, T, T), dtype=torch.uint8),
                 torch.ones((3, T, T), dtype=torch.uint8), torch.ones((6, T, T), dtype=torch.uint8)[::2]):
        lib._check_mask(DeviceView(good), 3, 512, dev)
    with pytest.raises(ValueError):
        lib._check_mask(DeviceView(torch.ones((2, T, T), dtype=torch.uint8)), 3, 512, dev)  # 2 heads of 3
    with pytest.raises(ValueError):
        lib._check_mask(DeviceView(torch.ones((T, T), dtype=torch.uint8)), 3, 640, dev)    # T = 5
    with pytest.raises(ValueError):  # on another GPU than q
        lib._check_mask(DeviceView(torch.ones((T, T), dtype=torch.uint8), index=1), 3, 512, dev)


def test_dropout_backward_argument_errors(lib):
    f = lib._lib.fa_bwd_dropout
    P = ctypes.c_void_p

    def call(B=1, H=1, N=256, d=128, scale=0.1, causal=0, t=230, q=P(16), ws=P(16)):
        return f(q, P(16), P(16), P(16), P(16), P(16), P(16), P(16), P(16), ws, B, H, N, d, scale, causal, t, 1, 0,
                 P(0))

    assert call(q=P(0)) == lib.FA_ERR_INVALID_ARG
    assert call(ws=P(0)) == lib.FA_ERR_INVALID_ARG
    assert call(t=-1) == lib.FA_ERR_INVALID_ARG
    assert call(t=257) == lib.FA_ERR_INVALID_ARG
    assert call(N=0) == lib.FA_ERR_INVALID_ARG
    assert call(scale=0.0) == lib.FA_ERR_INVALID_ARG
    assert call(d=96) == lib.FA_ERR_UNSUPPORTED
    assert call(B=300, H=300) == lib.FA_ERR_UNSUPPORTED   # more than 65535 heads
    assert call(q=P(4)) == lib.FA_ERR_MISALIGNED
    assert lib.last_launch_count() == 0


def test_fp32_backward_block_size_is_checked(lib):
    f = lib._lib.fa_bwd_f32
    P = ctypes.c_void_p

    def call(block_k):
        return f(P(16), P(16), P(16), P(16), P(16), P(16), P(16), P(16), P(16), P(16), 1, 1, 64, 64, 0.1, 0, block_k,
                 P(0))

    assert call(-1) == lib.FA_ERR_INVALID_ARG
    assert call(1025) == lib.FA_ERR_INVALID_ARG


def test_forward_queue_word_count_is_checked(lib):
    f = lib._lib.fa_set_fwd_queue_words
    assert f(0) == lib.FA_ERR_INVALID_ARG and f(65) == lib.FA_ERR_INVALID_ARG
    assert f(64) == lib.FA_OK


def test_backward_softmax_warp_count_is_checked(lib):
    f = lib._lib.fa_set_bwd_softmax_warps
    assert f(2) == lib.FA_ERR_INVALID_ARG and f(16) == lib.FA_ERR_INVALID_ARG
    assert f(4) == lib.FA_OK and f(8) == lib.FA_OK and f(0) == lib.FA_OK
