"""Pins for the fp64 CPU oracle (no GPU).

Every check here compares the oracle against something other than itself:
values the FlashAttention explainer page prints, closed forms, torch's own
softmax / logsumexp / autograd on tiny inputs, central finite differences, and
invariants that follow from rows of P summing to one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(shape, seed, gain=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * gain


def _torch_attention(q, k, v, scale, causal):
    """Library formulation: torch fp64 softmax over the full score matrix."""
    q, k, v = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    s = scale * q @ k.transpose(-1, -2)
    if causal:
        N = s.shape[-1]
        mask = torch.ones(N, N, dtype=torch.bool).triu(1)
        s = s.masked_fill(mask, float("-inf"))
    return (torch.softmax(s, -1) @ v).numpy(), torch.logsumexp(s, -1).numpy()


# ---------------------------------------------------------------- worked row


def test_worked_row_online_trace_matches_page():
    g = _golden("worked_row.json")
    w, m_trace, l_trace = oracle.softmax_online(g["row"], g["block"])
    nd = g["printed_decimals"]
    assert list(m_trace) == g["m_after_block"]
    assert round(l_trace[0], nd) == g["l_after_first_block"]
    assert round(l_trace[-1], nd) == g["l_final"]
    assert [round(x, nd) for x in w] == g["weights"]
    # the same weights from the naive (whole-row) softmax
    assert [round(x, nd) for x in oracle.softmax_naive(g["row"])] == g["weights"]
    # the page's identity: the final sum equals e^-1 + e^-2 + e^0 + e^-3
    assert abs(l_trace[-1] - (math.exp(-1) + math.exp(-2) + 1 + math.exp(-3))) < 1e-15


def test_worked_row_rescale_step_is_exact_not_printed_rounding():
    # the rescaled old sum is (e^0 + e^-1) * e^(2-3); the page prints 0.5033
    # (rounding of a rounded number), exact is 0.503215...
    row = [2.0, 1.0, 3.0, 0.0]
    _, _, lt = oracle.softmax_online(row, 2)
    rescaled = lt[0] * math.exp(2 - 3)
    assert abs(rescaled - 0.5032147244) < 1e-9
    assert abs(lt[1] - (rescaled + 1 + math.exp(-3))) < 1e-15


@pytest.mark.parametrize("n", [1, 2, 5, 64, 257])
@pytest.mark.parametrize("block", [1, 2, 3, 7, 64, None])
def test_online_softmax_equals_naive_and_sums_to_one(n, block):
    row = _rand(n, seed=n * 31 + (block or 0), gain=5.0)
    naive = oracle.softmax_naive(row)
    online, _, _ = oracle.softmax_online(row, block or n)
    assert np.max(np.abs(online - naive)) < 1e-13
    assert abs(online.sum() - 1.0) < 1e-13
    # and both agree with the library softmax
    ref = torch.softmax(torch.from_numpy(row), 0).numpy()
    assert np.max(np.abs(naive - ref)) < 1e-13


# ---------------------------------------------------------------- forward


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (1, 2, 5, 3), (2, 1, 8, 4), (1, 1, 7, 2)])
def test_fwd_matches_library_bruteforce(shape, causal):
    q, k, v = (_rand(shape, seed=s) for s in (1, 2, 3))
    scale = 1 / math.sqrt(shape[-1])
    o, lse = oracle.attn_fwd(q, k, v, scale, causal)
    o_ref, lse_ref = _torch_attention(q, k, v, scale, causal)
    assert np.max(np.abs(o - o_ref)) < 1e-13
    assert np.max(np.abs(lse - lse_ref)) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 2, 3, 7, 64, 100])
def test_block_size_never_changes_the_answer(block, causal):
    shape = (1, 2, 100, 16)
    q, k, v = (_rand(shape, seed=s, gain=2.0) for s in (11, 12, 13))
    scale = 0.25
    o, lse = oracle.attn_fwd(q, k, v, scale, causal)
    ot, lset = oracle.attn_fwd_tiled(q, k, v, scale, causal, block)
    assert np.max(np.abs(ot - o)) < 1e-13
    assert np.max(np.abs(lset - lse)) < 1e-13


def test_page_demo_tiled_equals_standard():
    g = _golden("demo_qkv.json")
    q, k, v = (np.array(g[x], dtype=np.float64)[None, None] for x in ("Q", "K", "V"))
    scale = 1 / math.sqrt(q.shape[-1])
    o, lse = oracle.attn_fwd(q, k, v, scale, False)
    o_ref, lse_ref = _torch_attention(q, k, v, scale, False)
    assert np.max(np.abs(o - o_ref)) <= g["max_abs_diff"]
    for b in g["blocks"]:
        ot, _ = oracle.attn_fwd_tiled(q, k, v, scale, False, b)
        assert np.max(np.abs(ot - o)) <= g["max_abs_diff"]


def test_fwd_rows_matches_full():
    shape = (1, 1, 50, 8)
    q, k, v = (_rand(shape, seed=s) for s in (21, 22, 23))
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, 0.3, causal)
        orow, lrow = oracle.attn_fwd_rows(q[0, 0], k[0, 0], v[0, 0], 17, 33, 0.3, causal)
        assert np.array_equal(orow, o[0, 0, 17:33])
        assert np.array_equal(lrow, lse[0, 0, 17:33])


# closed forms ------------------------------------------------------------


def test_single_key_returns_its_value():
    q, k, v = (_rand((2, 3, 1, 5), seed=s) for s in (31, 32, 33))
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, 0.7, causal)
        assert np.max(np.abs(o - v)) < 1e-15
        assert np.max(np.abs(lse - 0.7 * np.sum(q * k, -1))) < 1e-14


def test_zero_queries_give_uniform_weights():
    N, d = 9, 4
    q = np.zeros((1, 1, N, d))
    k, v = (_rand((1, 1, N, d), seed=s) for s in (41, 42))
    o, lse = oracle.attn_fwd(q, k, v, 1.0, False)
    assert np.max(np.abs(o[0, 0] - v[0, 0].mean(0))) < 1e-14
    assert np.max(np.abs(lse - math.log(N))) < 1e-14
    o, lse = oracle.attn_fwd(q, k, v, 1.0, True)
    prefix_mean = np.cumsum(v[0, 0], 0) / np.arange(1, N + 1)[:, None]
    assert np.max(np.abs(o[0, 0] - prefix_mean)) < 1e-14
    assert np.max(np.abs(lse[0, 0] - np.log(np.arange(1, N + 1)))) < 1e-14


def test_causal_first_row_is_first_value():
    q, k, v = (_rand((1, 2, 6, 3), seed=s, gain=3.0) for s in (51, 52, 53))
    o, _ = oracle.attn_fwd(q, k, v, 1.0, True)
    assert np.max(np.abs(o[:, :, 0] - v[:, :, 0])) < 1e-15


def test_identity_values_expose_the_weights_and_rows_sum_to_one():
    N = 6
    q, k = (_rand((1, 1, N, N), seed=s) for s in (61, 62))
    v = np.eye(N)[None, None]
    for causal in (False, True):
        o, _ = oracle.attn_fwd(q, k, v, 0.5, causal)
        s = 0.5 * q[0, 0] @ k[0, 0].T
        for i in range(N):
            n = i + 1 if causal else N
            w = torch.softmax(torch.from_numpy(s[i, :n]), 0).numpy()
            assert np.max(np.abs(o[0, 0, i, :n] - w)) < 1e-14
            assert np.all(o[0, 0, i, n:] == 0.0)
        assert np.max(np.abs(o.sum(-1) - 1.0)) < 1e-14


def test_worked_row_as_an_attention_problem():
    # q0 = e1, k_j = s_j * e1, scale 1, V = I: row 0 of O is the worked row's weights.
    g = _golden("worked_row.json")
    N = d = 4
    q = np.zeros((1, 1, N, d))
    k = np.zeros((1, 1, N, d))
    q[0, 0, 0, 0] = 1.0
    k[0, 0, :, 0] = g["row"]
    v = np.eye(N)[None, None]
    o, lse = oracle.attn_fwd(q, k, v, 1.0, False)
    assert [round(x, 4) for x in o[0, 0, 0]] == g["weights"]
    assert round(math.exp(lse[0, 0, 0] - 3.0), 4) == g["l_final"]


# ---------------------------------------------------------------- backward


def _loss(q, k, v, g, scale, causal):
    o, _ = oracle.attn_fwd(q, k, v, scale, causal)
    return float(np.sum(o * g))


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_central_finite_differences(causal):
    shape = (1, 2, 5, 3)
    q, k, v, g = (_rand(shape, seed=s) for s in (71, 72, 73, 74))
    scale = 0.6
    dq, dk, dv = oracle.attn_bwd(q, k, v, g, scale, causal)
    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}; args_p[name] = xp
            args_m = {"q": q, "k": k, "v": v}; args_m[name] = xm
            num[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], g, scale, causal)
                        - _loss(args_m["q"], args_m["k"], args_m["v"], g, scale, causal)) / (2 * h)
        err = np.max(np.abs(num - grad)) / max(1.0, np.max(np.abs(grad)))
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_torch_autograd(causal):
    shape = (2, 2, 11, 6)
    q, k, v, g = (_rand(shape, seed=s) for s in (81, 82, 83, 84))
    scale = 1 / math.sqrt(6)
    dq, dk, dv = oracle.attn_bwd(q, k, v, g, scale, causal)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    s = scale * tq @ tk.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.ones(11, 11, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.softmax(s, -1) @ tv
    (o * torch.from_numpy(g)).sum().backward()
    for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.max(np.abs(a - b.numpy())) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_invariants(causal):
    shape = (1, 3, 40, 8)
    q, k, v, g = (_rand(shape, seed=s, gain=1.5) for s in (91, 92, 93, 94))
    dq, dk, dv = oracle.attn_bwd(q, k, v, g, 0.35, causal)
    # rows of dS sum to zero  =>  sum_j dK_j = 0
    assert np.max(np.abs(dk.sum(2))) < 1e-12
    # rows of P sum to one    =>  sum_j dV_j = sum_i dO_i
    assert np.max(np.abs(dv.sum(2) - g.sum(2))) < 1e-12
    if causal:
        # the last key is seen only by the last query: dV_{N-1} = P_{N-1,N-1} dO_{N-1}
        o, lse = oracle.attn_fwd(q, k, v, 0.35, True)
        p_last = np.exp(0.35 * np.sum(q[:, :, -1] * k[:, :, -1], -1) - lse[:, :, -1])
        assert np.max(np.abs(dv[:, :, -1] - p_last[..., None] * g[:, :, -1])) < 1e-13


def test_bwd_dq_rows_matches_full_backward():
    shape = (1, 1, 37, 5)
    q, k, v, g = (_rand(shape, seed=s) for s in (101, 102, 103, 104))
    for causal in (False, True):
        dq, _, _ = oracle.attn_bwd(q, k, v, g, 0.45, causal)
        rows = oracle.attn_bwd_dq_rows(q[0, 0], k[0, 0], v[0, 0], g[0, 0], 5, 29, 0.45, causal)
        assert np.max(np.abs(rows - dq[0, 0, 5:29])) < 1e-14


def test_bwd_kv_rows_matches_full_backward():
    shape = (1, 1, 41, 6)
    q, k, v, g = (_rand(shape, seed=s) for s in (111, 112, 113, 114))
    for causal in (False, True):
        _, dk, dv = oracle.attn_bwd(q, k, v, g, 0.4, causal)
        rk, rv = oracle.attn_bwd_kv_rows(q[0, 0], k[0, 0], v[0, 0], g[0, 0], 9, 30, 0.4, causal)
        assert np.max(np.abs(rk - dk[0, 0, 9:30])) < 1e-14
        assert np.max(np.abs(rv - dv[0, 0, 9:30])) < 1e-14


# ---------------------------------------------------------------- Nq queries against Nk keys
# (the decode / split-KV shape).  Causal reading: the queries are the last Nq
# positions, so query i sees keys j <= Nk - Nq + i.

def _torch_attention_rect(q, k, v, scale, causal):
    """Library brute force: torch fp64 softmax(Q K^T scale + mask) V with the
    mask built by torch.tril on a rectangular matrix."""
    q, k, v = (torch.as_tensor(np.asarray(t, dtype=np.float64)) for t in (q, k, v))
    s = torch.matmul(q, k.transpose(-1, -2)) * scale
    Nq, Nk = s.shape[-2], s.shape[-1]
    if causal:
        keep = torch.tril(torch.ones(Nq, Nk, dtype=torch.bool), diagonal=Nk - Nq)
        s = s.masked_fill(~keep, float("-inf"))
    return torch.matmul(torch.softmax(s, dim=-1), v).numpy(), torch.logsumexp(s, dim=-1).numpy()


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 9), (3, 11), (7, 7), (5, 130)])
@pytest.mark.parametrize("causal", [False, True])
def test_rect_fwd_matches_library_bruteforce(Nq, Nk, causal):
    q = _rand((2, 2, Nq, 6), seed=Nq * 31 + Nk)
    k = _rand((2, 2, Nk, 6), seed=Nq * 37 + Nk)
    v = _rand((2, 2, Nk, 6), seed=Nq * 41 + Nk)
    o, lse = oracle.attn_fwd_rect(q, k, v, 0.4, causal)
    ro, rlse = _torch_attention_rect(q, k, v, 0.4, causal)
    assert np.max(np.abs(o - ro)) < 1e-12
    assert np.max(np.abs(lse - rlse)) < 1e-12


def test_rect_single_query_sees_every_key_even_causal():
    """With one query the causal mask allows all Nk keys (j <= Nk - 1)."""
    q, k, v = _rand((1, 3, 1, 8), 1), _rand((1, 3, 50, 8), 2), _rand((1, 3, 50, 8), 3)
    o_c, lse_c = oracle.attn_fwd_rect(q, k, v, 0.3, True)
    o_n, lse_n = oracle.attn_fwd_rect(q, k, v, 0.3, False)
    assert np.array_equal(o_c, o_n) and np.array_equal(lse_c, lse_n)


def test_rect_zero_queries_give_prefix_means():
    """Q = 0: uniform weights over the allowed keys, so causal row i is the mean
    of v[0 .. Nk - Nq + i] and LSE = ln(Nk - Nq + i + 1)."""
    Nq, Nk = 4, 10
    q = np.zeros((1, 1, Nq, 5))
    k, v = _rand((1, 1, Nk, 5), 7), _rand((1, 1, Nk, 5), 8)
    o, lse = oracle.attn_fwd_rect(q, k, v, 1.0, True)
    for i in range(Nq):
        n = Nk - Nq + i + 1
        assert np.allclose(o[0, 0, i], v[0, 0, :n].mean(axis=0), atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(n)) < 1e-14


def test_rect_with_nq_equal_nk_is_the_square_problem():
    """Nq = Nk reduces the bottom-right mask to the square top-left one."""
    q, k, v = _rand((2, 2, 9, 4), 11), _rand((2, 2, 9, 4), 12), _rand((2, 2, 9, 4), 13)
    for causal in (False, True):
        o, lse = oracle.attn_fwd_rect(q, k, v, 0.5, causal)
        ro, rlse = _torch_attention(q, k, v, 0.5, causal)
        assert np.max(np.abs(o - ro)) < 1e-12 and np.max(np.abs(lse - rlse)) < 1e-12


def test_rect_key_splits_combine_by_the_rescale_rule():
    """Attention over disjoint key ranges, each with its own (O_s, LSE_s),
    recombines exactly: LSE = ln sum_s e^{LSE_s}, O = sum_s e^{LSE_s - LSE} O_s
    (the online-softmax update applied to whole blocks)."""
    q, k, v = _rand((1, 2, 3, 6), 21), _rand((1, 2, 40, 6), 22), _rand((1, 2, 40, 6), 23)
    o, lse = oracle.attn_fwd_rect(q, k, v, 0.7, False)
    parts = [oracle.attn_fwd_rect(q, k[:, :, a:b], v[:, :, a:b], 0.7, False) for a, b in ((0, 13), (13, 14), (14, 40))]
    L = np.log(sum(np.exp(p[1]) for p in parts))
    O = sum(np.exp(p[1] - L)[..., None] * p[0] for p in parts)
    assert np.max(np.abs(L - lse)) < 1e-12 and np.max(np.abs(O - o)) < 1e-12


# ---------------------------------------------------------------- block-sparse
# Square attention restricted to the (query block, key block) pairs a block
# mask allows; rows with no allowed key give O = 0, LSE = -inf.

def _torch_attention_blockmask(q, k, v, scale, causal, mask, br, bc):
    """Library brute force: the block mask expanded to an element mask with
    torch.repeat_interleave, then fp64 softmax(Q K^T scale + mask) V."""
    q, k, v = (torch.as_tensor(np.asarray(t, dtype=np.float64)) for t in (q, k, v))
    N = q.shape[-2]
    m = torch.as_tensor(np.asarray(mask) != 0)
    if m.dim() == 2:
        m = m[None]
    keep = m.repeat_interleave(br, dim=1)[:, :N].repeat_interleave(bc, dim=2)[:, :, :N]  # [Hm, N, N]
    if causal:
        keep = keep & torch.tril(torch.ones(N, N, dtype=torch.bool))
    s = (torch.matmul(q, k.transpose(-1, -2)) * scale).masked_fill(~keep, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    p = torch.softmax(s, dim=-1).nan_to_num(0.0)  # a row with no allowed key: all -inf
    return torch.matmul(p, v).numpy(), lse.numpy()


@pytest.mark.parametrize("N,br,bc", [(7, 2, 3), (12, 4, 4), (13, 5, 2), (9, 9, 1)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("per_head", [False, True])
def test_blockmask_matches_library_bruteforce(N, br, bc, causal, per_head):
    H = 3
    q, k, v = (_rand((2, H, N, 5), seed=N * 7 + br + 10 * s) for s in range(3))
    nqb, nkb = -(-N // br), -(-N // bc)
    rng = np.random.default_rng(N * 13 + bc)
    mask = (rng.random((H if per_head else 1, nqb, nkb)) < 0.5).astype(np.uint8)
    mask[0, 0, :] = 0  # the first query block of head 0 sees nothing
    o, lse = oracle.attn_fwd_blockmask(q, k, v, 0.6, causal, mask, br, bc)
    ro, rlse = _torch_attention_blockmask(q, k, v, 0.6, causal, mask, br, bc)
    assert np.max(np.abs(o - ro)) < 1e-12
    assert np.array_equal(np.isinf(lse), np.isinf(rlse))
    fin = np.isfinite(rlse)
    assert np.max(np.abs(lse[fin] - rlse[fin]), initial=0.0) < 1e-12
    assert np.all(o[0, 0, :br] == 0.0) and np.all(lse[0, 0, :br] == -np.inf)


def test_blockmask_zero_queries_give_the_mean_of_the_chosen_key_block():
    """Q = 0 and one key block per query block: uniform weights over that
    block's keys, so O_i is their mean and LSE_i = ln(block size)."""
    N, br, bc = 20, 4, 6
    q = np.zeros((1, 1, N, 3))
    k, v = _rand((1, 1, N, 3), 31), _rand((1, 1, N, 3), 32)
    nqb, nkb = N // br, -(-N // bc)
    mask = np.zeros((1, nqb, nkb), dtype=np.uint8)
    for qb in range(nqb):
        mask[0, qb, (3 * qb + 1) % nkb] = 1
    o, lse = oracle.attn_fwd_blockmask(q, k, v, 1.0, False, mask, br, bc)
    for i in range(N):
        kb = (3 * (i // br) + 1) % nkb
        keys = v[0, 0, kb * bc:min(N, (kb + 1) * bc)]
        assert np.allclose(o[0, 0, i], keys.mean(axis=0), atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(len(keys))) < 1e-14


def test_blockmask_all_ones_and_lower_triangle_reduce_to_dense():
    q, k, v = (_rand((1, 2, 23, 4), 40 + s) for s in range(3))
    ones = np.ones((1, 3, 3), dtype=np.uint8)
    lower = np.tril(ones[0])[None]
    for causal, mask in ((False, ones), (True, ones), (True, lower)):
        o, lse = oracle.attn_fwd_blockmask(q, k, v, 0.5, causal, mask, 8, 8)
        ro, rlse = _torch_attention(q, k, v, 0.5, causal)
        assert np.max(np.abs(o - ro)) < 1e-12 and np.max(np.abs(lse - rlse)) < 1e-12


def test_blockmask_block_diagonal_is_independent_blocks():
    """A block-diagonal mask splits the problem into independent attentions,
    one per block (computed here by slicing the inputs)."""
    N, b = 18, 6
    q, k, v = (_rand((1, 1, N, 4), 50 + s) for s in range(3))
    mask = np.eye(N // b, dtype=np.uint8)[None]
    o, lse = oracle.attn_fwd_blockmask(q, k, v, 0.8, False, mask, b, b)
    for t in range(N // b):
        sl = slice(t * b, (t + 1) * b)
        ro, rlse = _torch_attention(q[:, :, sl], k[:, :, sl], v[:, :, sl], 0.8, False)
        assert np.max(np.abs(o[:, :, sl] - ro)) < 1e-12 and np.max(np.abs(lse[:, :, sl] - rlse)) < 1e-12


# ---------------------------------------------------------------- dropout
# Keep decisions from Philox4x64-10 (counter (j // 32, i, bh, 0), key (seed,
# offset), byte j % 32 of the 32 output bytes < t), weights scaled by 256 / t.

def test_philox_matches_numpy_bit_generator():
    """numpy.random.Philox is Philox4x64-10; it advances its counter before each
    block, so its first block under counter c is the function at c + 1."""
    rng = np.random.default_rng(0)
    for _ in range(20):
        c = rng.integers(0, 2 ** 63, size=4, dtype=np.uint64)
        c[0] = c[0] // 2  # no carry out of word 0
        k = rng.integers(0, 2 ** 63, size=2, dtype=np.uint64) * np.uint64(2) + np.uint64(1)
        ref = np.random.Philox(counter=c, key=k).random_raw(4)
        c1 = c.copy()
        c1[0] += np.uint64(1)
        assert np.array_equal(oracle.philox4x64_10(c1, k), ref)


def _numpy_block(counter, key):
    """The Philox4x64-10 block at `counter` from numpy's bit generator, which
    advances its 256-bit counter by one before each block: start one below."""
    value = sum(int(w) << (64 * n) for n, w in enumerate(counter))
    value = (value - 1) % (1 << 256)
    below = np.array([(value >> (64 * n)) & (2 ** 64 - 1) for n in range(4)], dtype=np.uint64)
    return np.random.Philox(counter=below, key=np.asarray(key, dtype=np.uint64)).random_raw(4)


def _numpy_keep_mask(bh, N, t, seed, offset):
    """The keep mask derived from numpy's Philox outputs directly."""
    z = np.zeros((N, N), dtype=np.uint8)
    for i in range(N):
        for jb in range((N + 31) // 32):
            w = _numpy_block([jb, i, bh, 0], [seed, offset])
            b = np.frombuffer(np.asarray(w, dtype="<u8").tobytes(), dtype=np.uint8)
            for jj in range(min(32, N - jb * 32)):
                z[i, jb * 32 + jj] = b[jj] < t
    return z


@pytest.mark.parametrize("bh,N,t,seed,offset", [(0, 40, 230, 7, 0), (3, 70, 128, 2 ** 40 + 5, 9), (1, 33, 1, 1, 1)])
def test_dropout_mask_matches_numpy_philox_bytes(bh, N, t, seed, offset):
    assert np.array_equal(oracle.dropout_mask(bh, N, t, seed, offset), _numpy_keep_mask(bh, N, t, seed, offset))


def test_dropout_keep_rate_is_t_over_256():
    for t in (26, 128, 230):
        z = oracle.dropout_mask(2, 300, t, 1234, 5)
        p = t / 256
        n = z.size
        assert abs(z.mean() - p) <= 5 * math.sqrt(p * (1 - p) / n)


def _torch_dropout_reference(q, k, v, do, scale, causal, z, t):
    """torch fp64: O = (256/t) (softmax(S) o Z) V and its autograd gradients."""
    q, k, v, do = (torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True) for x in (q, k, v, do))
    s = torch.matmul(q, k.transpose(-1, -2)) * scale
    if causal:
        N = s.shape[-1]
        s = s.masked_fill(~torch.tril(torch.ones(N, N, dtype=torch.bool)), float("-inf"))
    p = torch.softmax(s, dim=-1)
    o = torch.matmul(p * torch.as_tensor(z, dtype=torch.float64) * (256.0 / t), v)
    (o * do).sum().backward()
    return o.detach().numpy(), torch.logsumexp(s, dim=-1).detach().numpy(), q.grad.numpy(), k.grad.numpy(), \
        v.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("t", [230, 100])
def test_dropout_forward_and_backward_match_torch_with_the_mask(causal, t):
    B, H, N, d = 1, 2, 37, 5
    q, k, v, do = (_rand((B, H, N, d), seed=60 + s) for s in range(4))
    seed, offset = 99, 3
    z = np.stack([oracle.dropout_mask(h, N, t, seed, offset) for h in range(H)])[None]
    o, lse = oracle.attn_fwd_dropout(q, k, v, 0.5, causal, t, seed, offset)
    dq, dk, dv = oracle.attn_bwd_dropout(q, k, v, do, 0.5, causal, t, seed, offset)
    ro, rlse, rdq, rdk, rdv = _torch_dropout_reference(q, k, v, do, 0.5, causal, z, t)
    for a, b in ((o, ro), (lse, rlse), (dq, rdq), (dk, rdk), (dv, rdv)):
        assert np.max(np.abs(a - b)) < 1e-12


def test_dropout_with_t256_is_plain_attention_and_t0_is_zero():
    q, k, v, do = (_rand((1, 2, 29, 4), seed=70 + s) for s in range(4))
    for causal in (False, True):
        o, lse = oracle.attn_fwd_dropout(q, k, v, 0.7, causal, 256, 5, 6)
        ro, rlse = oracle.attn_fwd(q, k, v, 0.7, causal)
        assert np.array_equal(o, ro) and np.array_equal(lse, rlse)
        g = oracle.attn_bwd_dropout(q, k, v, do, 0.7, causal, 256, 5, 6)
        rg = oracle.attn_bwd(q, k, v, do, 0.7, causal)
        for a, b in zip(g, rg):
            assert np.max(np.abs(a - b)) < 1e-14
        o0, lse0 = oracle.attn_fwd_dropout(q, k, v, 0.7, causal, 0, 5, 6)
        assert np.all(o0 == 0) and np.array_equal(lse0, rlse)
        assert all(np.all(x == 0) for x in oracle.attn_bwd_dropout(q, k, v, do, 0.7, causal, 0, 5, 6))


def test_dropout_head_offset_selects_the_heads_generator_stream():
    """Heads given alone with bh0 = their index reproduce the whole problem's rows."""
    q, k, v = (_rand((2, 3, 40, 4), seed=80 + s) for s in range(3))
    o, lse = oracle.attn_fwd_dropout(q, k, v, 0.6, True, 200, 11, 2)
    for b, h in ((0, 2), (1, 0), (1, 2)):
        oh, lh = oracle.attn_fwd_dropout(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], 0.6, True,
                                         200, 11, 2, bh0=b * 3 + h)
        assert np.array_equal(oh[0, 0], o[b, h]) and np.array_equal(lh[0, 0], lse[b, h])


# ---------------------------------------------------------------- per-head threaded backward


def _torch_grads(q, k, v, g, scale, causal, z=None, t=256):
    """torch fp64 autograd of L = sum(O * G), O = (256/t) (softmax(S) o Z) V (Z = 1: plain)."""
    tq, tk, tv = (torch.from_numpy(np.asarray(x, dtype=np.float64)).requires_grad_(True) for x in (q, k, v))
    s = scale * tq @ tk.transpose(-1, -2)
    N = s.shape[-1]
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    p = torch.softmax(s, -1)
    if z is not None:
        p = p * torch.as_tensor(z, dtype=torch.float64) * (256.0 / t)
    ((p @ tv) * torch.from_numpy(np.asarray(g, dtype=np.float64))).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 3), (23, 5), (70, 8)])
def test_head_backward_matches_torch_autograd(N, d, causal):
    q, k, v, g = (_rand((N, d), seed=s, gain=1.3) for s in (121, 122, 123, 124))
    dq, dk, dv = oracle.attn_bwd_head(q, k, v, g, 0.55, causal)
    for a, b in zip((dq, dk, dv), _torch_grads(q, k, v, g, 0.55, causal)):
        assert np.max(np.abs(a - b)) < 1e-12
    # the same definition as the per-head-threaded backward
    for a, b in zip((dq, dk, dv), oracle.attn_bwd(q[None, None], k[None, None], v[None, None], g[None, None],
                                                  0.55, causal)):
        assert np.max(np.abs(a - b[0, 0])) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_head_backward_invariants(causal):
    N, d = 90, 6
    q, k, v, g = (_rand((N, d), seed=s, gain=1.5) for s in (131, 132, 133, 134))
    dq, dk, dv = oracle.attn_bwd_head(q, k, v, g, 0.4, causal)
    assert np.max(np.abs(dk.sum(0))) < 1e-12          # rows of dS sum to zero
    assert np.max(np.abs(dv.sum(0) - g.sum(0))) < 1e-12  # rows of P sum to one
    if causal:
        # key 0 is seen by every query and the first query sees only key 0
        o, lse = oracle.attn_fwd(q[None, None], k[None, None], v[None, None], 0.4, True)
        assert np.max(np.abs(dq[0])) < 1e-15          # P_00 = 1, dS_00 = dP_00 - D_0 = 0


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bh,t", [(0, 200), (5, 77)])
def test_head_backward_with_dropout_matches_torch_with_numpy_mask(bh, t, causal):
    N, d = 45, 4
    q, k, v, g = (_rand((N, d), seed=s) for s in (141, 142, 143, 144))
    seed, offset = 2 ** 33 + 17, 4
    z = _numpy_keep_mask(bh, N, t, seed, offset)
    dq, dk, dv = oracle.attn_bwd_head(q, k, v, g, 0.5, causal, keep_t=t, seed=seed, offset=offset, bh=bh)
    for a, b in zip((dq, dk, dv), _torch_grads(q, k, v, g, 0.5, causal, z, t)):
        assert np.max(np.abs(a - b)) < 1e-12


def test_dropout_backward_head_offset_selects_the_heads_generator_stream():
    """Heads given alone with bh0 = their index reproduce the whole problem's gradients."""
    q, k, v, g = (_rand((2, 3, 33, 4), seed=150 + s) for s in range(4))
    full = oracle.attn_bwd_dropout(q, k, v, g, 0.6, True, 190, 8, 1)
    for b, h in ((0, 1), (1, 2)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        part = oracle.attn_bwd_dropout(q[sl], k[sl], v[sl], g[sl], 0.6, True, 190, 8, 1, bh0=b * 3 + h)
        head = oracle.attn_bwd_head(q[b, h], k[b, h], v[b, h], g[b, h], 0.6, True, keep_t=190, seed=8, offset=1,
                                    bh=b * 3 + h)
        for a, p, hh in zip(full, part, head):
            assert np.array_equal(p[0, 0], a[b, h])
            assert np.max(np.abs(hh - a[b, h])) < 1e-13
