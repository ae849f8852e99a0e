"""Single-tile tcgen05 GEMMs through the C ABI: the operand encodings the
attention kernels use (K-major / MN-major shared-memory tiles with the 128-byte
swizzle, the TMEM A operand, the software swizzle) against a float64 matmul of
the same bf16 values."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _case(fa, N, K, a_mn, b_mn, a_tmem, b_manual, seed):
    g = torch.Generator().manual_seed(seed)
    M = 128
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)   # logical A [M][K]
    Bm = torch.randn(K, N, generator=g).to(torch.bfloat16)  # logical B [K][N]
    a_store = (A.t() if a_mn else A).contiguous().cuda()
    b_store = (Bm if b_mn else Bm.t()).contiguous().cuda()
    d = fa.selftest_umma(a_store, b_store, M, N, K, a_mn, b_mn, a_tmem, b_manual)
    torch.cuda.synchronize()
    ref = A.double() @ Bm.double()
    err = (d.double().cpu() - ref).abs().max().item()
    # exact bf16 products, fp32 accumulation of K terms
    assert err < 1e-3 * max(1.0, ref.abs().max().item()), err


@pytest.mark.parametrize("N,K", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_umma_smem_operands(fa_lib, N, K, a_mn, b_mn):
    _case(fa_lib, N, K, a_mn, b_mn, 0, 0, seed=N + K + 10 * a_mn + 100 * b_mn)


@pytest.mark.parametrize("N,K", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("b_mn", [0, 1])
def test_umma_tmem_a_operand(fa_lib, N, K, b_mn):
    _case(fa_lib, N, K, 0, b_mn, 1, 0, seed=7 + N + K + b_mn)


@pytest.mark.parametrize("N,K", [(64, 128), (128, 128), (64, 64)])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 1), (1, 1), (0, 0)])
def test_umma_software_swizzled_b(fa_lib, N, K, a_mn, b_mn):
    _case(fa_lib, N, K, a_mn, b_mn, 0, 1, seed=3 + N + K + a_mn + b_mn)


def test_fma_pipe_exp2_within_its_fitted_bound(fa_lib):
    """The polynomial exp2 the kernels use beside ex2.approx: relative error
    against float64 2^x within the Remez fit's bound (exp2_poly.h) plus float32
    evaluation rounding, over the range the kernels feed it."""
    import os
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    hdr = open(os.path.join(root, "exact_io_aware_53_b200", "csrc", "exp2_poly.h")).read()
    bound = float(re.search(r"MAX_REL_ERR = ([0-9.e+-]+)f", hdr).group(1))
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.linspace(-124.0, 64.0, 1 << 20), torch.rand(1 << 20, generator=g) * 20 - 16,
                   torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, 7.999, -124.5])])
    x = x.contiguous().cuda()
    y = fa_lib.selftest_exp2(x, 0)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref) / ref).abs().max().item()
    assert rel <= bound + 8 * 2.0 ** -24, rel
    # below the clamp the result stands for zero
    lo = fa_lib.selftest_exp2(torch.tensor([-200.0, float("-inf"), -126.0, 0, 0, 0, 0, 0]).cuda(), 0)
    assert float(lo[:3].max()) <= 2.0 ** -124
    # the hardware approximation it runs beside, for comparison
    y1 = fa_lib.selftest_exp2(x, 1)
    assert ((y1.double() - ref) / ref).abs().max().item() < 2.0 ** -20
