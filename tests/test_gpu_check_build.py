"""Race stress: the parity suites' ragged, many-item and multi-path cases run
again on the check build (libfa_sm100_check.so).

The check build is the same source compiled with FA_CHECK_BUILD: one bounded
wait in four sleeps a pseudo-random 0-2 us after it succeeds, so the warps of
a CTA meet at their barriers in orders that ordinary timing does not produce,
and every TMA tile copy tests its coordinates before it is issued.  A barrier
phase taken as complete too early (a waiter two phases ahead of its barrier)
or a buffer rewritten while a copy still reads it then shows up here as a
result outside the oracle's bar, or as an expired wait, instead of staying
hidden.  Both passes' persistent item loops, the forward's staging turns (Q
tiles past N), the host-buffer step and the split-KV, block-sparse, FP8 and
dropout kernels are covered; each case runs twice (different sleeps) and
every call must leave the device error word clear (no bad tile coordinate, no
expired wait).
"""
import pytest

from tests import test_gpu_bf16 as bf16
from tests import test_gpu_blocksparse as bsp
from tests import test_gpu_decode as dec
from tests import test_gpu_dropout as drop
from tests import test_gpu_fp8 as fp8
from tests import test_gpu_host_step as host
from tests import test_gpu_persistent as pers

pytestmark = pytest.mark.gpu

REPEAT = [0, 1]


@pytest.fixture(scope="module")
def fa_check():
    from exact_io_aware_53_b200 import fa
    chk = fa.check_build()
    assert chk.LIB_PATH.endswith("libfa_sm100_check.so")
    chk.check_device_status()  # start from a clear error word
    return chk


@pytest.mark.parametrize("rep", REPEAT)
@pytest.mark.parametrize("warps", [8, 4])
@pytest.mark.parametrize("shape", pers.SHAPES)
def test_backward_many_items_per_cta(fa_check, shape, warps, rep):
    pers.test_persistent_backward_many_items_per_cta(fa_check, shape, warps)


@pytest.mark.parametrize("rep", REPEAT)
@pytest.mark.parametrize("B,H,N,d,causal", [
    (4, 40, 300, 64, False), (4, 40, 300, 128, False), (2, 40, 550, 64, True), (2, 30, 550, 128, True),
    (8, 20, 129, 128, True), (8, 20, 129, 64, False),
])
def test_forward_items_with_a_q_tile_past_n(fa_check, B, H, N, d, causal, rep):
    pers.test_forward_items_with_a_q_tile_past_n(fa_check, B, H, N, d, causal)


@pytest.mark.parametrize("rep", REPEAT)
def test_dropout_backward_many_items_per_cta(fa_check, rep):
    pers.test_persistent_dropout_backward_many_items_per_cta(fa_check)


@pytest.mark.parametrize("B,H,N,d,causal", bf16.SMALL)
def test_small_fwd_bwd(fa_check, B, H, N, d, causal):
    bf16.test_small_fwd_bwd_full_compare(fa_check, B, H, N, d, causal)


@pytest.mark.parametrize("shape", host.SHAPES)
def test_host_step(fa_check, shape):
    host.test_host_step_equals_device_calls(fa_check, shape)


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,n_split", dec.CASES)
def test_splitkv(fa_check, B, H, Nq, Nk, d, causal, n_split):
    dec.test_splitkv_matches_oracle(fa_check, B, H, Nq, Nk, d, causal, n_split)


@pytest.mark.parametrize("B,H,N,d,causal,per_head", bsp.CASES)
def test_blocksparse(fa_check, B, H, N, d, causal, per_head):
    bsp.test_blocksparse_matches_oracle(fa_check, B, H, N, d, causal, per_head)


@pytest.mark.parametrize("B,H,N,causal,gain", [
    (2, 1, 200, False, 1.0), (1, 2, 513, True, 1.0), (2, 2, 400, True, 1.0), (1, 3, 16, False, 1.0),
    (3, 1, 768, False, 1.0),
])
def test_fp8(fa_check, B, H, N, causal, gain):
    fp8.test_fp8_matches_oracle_within_the_derived_bound(fa_check, B, H, N, causal, gain)


@pytest.mark.parametrize("B,H,N,d,causal,keep_t", [
    (1, 2, 200, 128, True, 230), (2, 1, 300, 64, False, 128), (2, 2, 383, 64, True, 250),
])
def test_dropout_fwd_bwd(fa_check, B, H, N, d, causal, keep_t):
    drop.test_dropout_matches_oracle(fa_check, B, H, N, d, causal, keep_t)
    drop.test_dropout_backward_matches_oracle(fa_check, B, H, N, d, causal, keep_t)


def test_error_word_clear_after_the_suite(fa_check):
    assert fa_check.check_device_status() == fa_check.FA_OK
