"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check is a value printed
on the pages (the worked example of the FlashAttention-2 tutorial, 2.1.9), a
closed form, an invariant of softmax attention, a special case that reduces to
a simpler problem, brute force over block splits, central finite differences,
or an independent library witness (torch fp64).
"""

import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "online_softmax_worked_example.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        k, v = [t.strip() for t in line.split("=")]
        nums = [float(x) for x in v.split()]
        vals[k] = nums if len(nums) > 1 else nums[0]
    return vals


def _rand(seed, shape):
    return synth.bf16_bits_to_f64(synth.normal_bf16(seed, shape))


def _worked_qkv(scores, d=None):
    """One query whose scaled scores against n = len(scores) keys are exactly
    ``scores`` (scale 1, q = e_0, k_j = scores[j] e_0), head dimension d
    (default n) and, when d == n, V = identity so that O = P."""
    n = len(scores)
    d = n if d is None else d
    Q = np.zeros((1, 1, 1, d))
    Q[0, 0, 0, 0] = 1.0
    K = np.zeros((1, 1, n, d))
    K[0, 0, :, 0] = scores
    V = np.eye(n, d)[None, None]
    return Q, K, V


# ---------------------------------------------------------------- worked example


def test_worked_example_one_pass():
    g = _golden()
    Q, K, V = _worked_qkv(g["scores"])
    O, L = oracle.fwd(Q, K, V, scale=1.0)
    p = O[0, 0, 0]
    assert np.all(np.abs(p - np.array(g["probs"])) <= g["tol"])
    # LSE = max + ln(sum of shifted exponentials), from the printed max and sum
    assert abs(L[0, 0, 0] - (g["max"] + math.log(g["sum"]))) <= g["tol_sum"] / g["sum"] + 1e-12
    # the exponentials relative to the max and their sum
    P, lse = oracle.probs(Q[0, 0], K[0, 0], 1.0)
    e = P[0] * math.exp(lse[0] - g["max"])
    assert np.all(np.abs(e - np.array(g["exps"])) <= g["tol"])
    assert abs(e.sum() - g["sum"]) <= g["tol_sum"]
    assert abs(P[0].sum() - 1.0) <= 1e-15


def test_worked_example_two_blocks_unnormalised():
    g = _golden()
    n = len(g["scores"])
    O, m, l, mt, lt = oracle.online_row(g["scores"], np.eye(n), [int(x) for x in g["block_ends"]])
    assert np.all(np.abs(O - np.array(g["probs"])) <= g["tol"])
    assert mt[0] == g["blockA_max"] and m == g["max"]
    assert abs(lt[0] - g["blockA_sum"]) <= g["tol"]
    assert abs(lt[1] - g["sum"]) <= g["tol_sum"]
    assert abs((lt[1] - lt[0]) - g["blockB_sum"]) <= g["tol"]


def test_worked_example_two_blocks_normalised_merge():
    g = _golden()
    s = np.array(g["scores"])
    n = len(s)
    # each block on its own: (m, l, O) with O normalised inside the block
    Oa, ma, la, _, _ = oracle.online_row(s[:2], np.eye(n)[:2], [2])
    Ob, mb, lb, _, _ = oracle.online_row(s[2:], np.eye(n)[2:], [2])
    assert np.all(np.abs(Oa[:2] - np.array(g["blockA_probs"])) <= g["tol"])
    m, l, O = oracle.merge(ma, la, Oa, mb, lb, Ob)
    assert np.all(np.abs(O - np.array(g["probs"])) <= g["tol"])
    # weight that carries the block-A probabilities into the merged row
    ratio = math.exp(ma - m) * la / l
    assert abs(ratio - g["old_over_new"]) <= g["tol_ratio"]
    # block B's unnormalised weights relative to the running max 5
    wb = np.exp(s[2:] - m)
    assert np.all(np.abs(wb - np.array(g["blockB_weights"])) <= g["tol"])


def test_worked_example_block_c_rescale():
    """A third block [10] raises the max from 5 to 10: the history is scaled by e^-5."""
    g = _golden()
    s = np.array(list(g["scores"]) + [g["blockC"]])
    n = len(s)
    O, m, l, mt, lt = oracle.online_row(s, np.eye(n), [2, 4, 5])
    assert mt[1] == g["max"] and mt[2] == g["blockC"] and m == g["blockC"]
    factor = math.exp(g["blockC_factor_exponent"])
    assert abs(lt[2] - (lt[1] * factor + 1.0)) <= 1e-15
    # and the result is the one-pass softmax of all five scores
    Q, K, V = _worked_qkv(s)
    O1, _ = oracle.fwd(Q, K, V, scale=1.0)
    assert np.max(np.abs(O - O1[0, 0, 0])) <= 1e-15


# ---------------------------------------------------------------- invariants


@pytest.mark.parametrize("causal", [False, True])
def test_rows_sum_to_one_and_masked_zero(causal):
    Q = _rand(11, (37, 16))
    K = _rand(12, (53, 16))
    P, lse = oracle.probs(Q, K, 0.25, causal=causal, kv_len=41)
    vis = P > 0
    assert np.all(np.abs(P.sum(axis=1) - 1.0) <= 1e-14)
    i = np.arange(37)[:, None]
    j = np.arange(53)[None, :]
    allowed = (j < 41) & ((~np.bool_(causal)) | (j <= i + (53 - 37)))
    assert not np.any(vis & ~allowed)


def test_constant_v_gives_v():
    Q = _rand(21, (1, 2, 19, 8))
    K = _rand(22, (1, 2, 23, 8))
    v = _rand(23, (8,))
    V = np.broadcast_to(v, (1, 2, 23, 8)).copy()
    for causal in (False, True):
        O, _ = oracle.fwd(Q, K, V, 0.3, causal=causal)
        assert np.max(np.abs(O - v)) <= 1e-14 * max(1.0, np.max(np.abs(v)))


def test_key_permutation_invariance_non_causal():
    Q = _rand(31, (1, 1, 9, 8))
    K = _rand(32, (1, 1, 14, 8))
    V = _rand(33, (1, 1, 14, 8))
    perm = np.random.default_rng(0).permutation(14)
    O1, L1 = oracle.fwd(Q, K, V, 0.35)
    O2, L2 = oracle.fwd(Q, K[:, :, perm], V[:, :, perm], 0.35)
    assert np.max(np.abs(O1 - O2)) <= 1e-13
    assert np.max(np.abs(L1 - L2)) <= 1e-13


def test_causal_row_zero_is_v0():
    Q = _rand(41, (1, 1, 12, 16))
    K = _rand(42, (1, 1, 12, 16))
    V = _rand(43, (1, 1, 12, 16))
    O, L = oracle.fwd(Q, K, V, 0.25, causal=True)
    assert np.array_equal(O[0, 0, 0], V[0, 0, 0])
    s00 = float(np.dot(Q[0, 0, 0], K[0, 0, 0])) * 0.25
    assert abs(L[0, 0, 0] - s00) <= 1e-13


def test_single_key_closed_form():
    Q = _rand(51, (2, 2, 7, 8))
    K = _rand(52, (2, 2, 1, 8))
    V = _rand(53, (2, 2, 1, 8))
    O, L = oracle.fwd(Q, K, V, 0.5)
    assert np.array_equal(O, np.broadcast_to(V, O.shape))
    s = np.einsum("bhid,bhjd->bhi", Q, K) * 0.5
    assert np.max(np.abs(L - s)) <= 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_visible(causal):
    Lq, Lk, kl = 6, 10, 8
    Q = np.zeros((1, 1, Lq, 4))
    K = _rand(61, (1, 1, Lk, 4))
    V = _rand(62, (1, 1, Lk, 4))
    O, L = oracle.fwd(Q, K, V, 1.0, causal=causal, k_lens=[kl])
    for i in range(Lq):
        hi = min(kl, i + (Lk - Lq) + 1) if causal else kl
        assert np.max(np.abs(O[0, 0, i] - V[0, 0, :hi].mean(axis=0))) <= 1e-14
        assert abs(L[0, 0, i] - math.log(hi)) <= 1e-14


def test_fully_masked_rows():
    Q = _rand(71, (2, 1, 5, 4))
    K = _rand(72, (2, 1, 3, 4))
    V = _rand(73, (2, 1, 3, 4))
    # k_len = 0 masks every key of sequence 0
    O, L = oracle.fwd(Q, K, V, 1.0, k_lens=[0, 3])
    assert np.all(O[0] == 0.0) and np.all(L[0] == -np.inf)
    assert np.all(np.isfinite(L[1]))
    # bottom-right causal with Lq > Lk: row i sees keys j <= i - 2
    O, L = oracle.fwd(Q, K, V, 1.0, causal=True, k_lens=[3, 3])
    assert np.all(O[:, :, :2] == 0.0) and np.all(L[:, :, :2] == -np.inf)
    assert np.array_equal(O[:, :, 2], V[:, :, 0])


def test_padding_equals_truncated_problem():
    """A key length k reduces to the unmasked problem on the first k keys."""
    Q = _rand(81, (1, 2, 11, 8))
    K = _rand(82, (1, 2, 17, 8))
    V = _rand(83, (1, 2, 17, 8))
    O1, L1 = oracle.fwd(Q, K, V, 0.3, k_lens=[9])
    O2, L2 = oracle.fwd(Q, K[:, :, :9], V[:, :, :9], 0.3)
    assert np.max(np.abs(O1 - O2)) <= 1e-15 and np.max(np.abs(L1 - L2)) <= 1e-15
    # causal + padding: bottom-right causality is defined against the full Lk
    O3, _ = oracle.fwd(Q, K, V, 0.3, causal=True, k_lens=[9])
    for i in range(11):
        hi = min(9, i + (17 - 11) + 1)
        Oi, _ = oracle.fwd(Q[:, :, i:i + 1], K[:, :, :hi], V[:, :, :hi], 0.3)
        assert np.max(np.abs(O3[:, :, i] - Oi[:, :, 0])) <= 1e-14


def test_gqa_reads_shared_head():
    Q = _rand(91, (1, 4, 5, 8))
    K = _rand(92, (1, 2, 6, 8))
    V = _rand(93, (1, 2, 6, 8))
    O, L = oracle.fwd(Q, K, V, 0.3)
    Ke = np.repeat(K, 2, axis=1)
    Ve = np.repeat(V, 2, axis=1)
    O2, L2 = oracle.fwd(Q, Ke, Ve, 0.3)
    assert np.array_equal(O, O2) and np.array_equal(L, L2)


def test_rows_subset_matches_full():
    Q = _rand(95, (1, 1, 40, 8))
    K = _rand(96, (1, 1, 40, 8))
    V = _rand(97, (1, 1, 40, 8))
    O, L = oracle.fwd(Q, K, V, 0.3, causal=True)
    rows = [0, 7, 39, 21]
    Os, Ls = oracle.fwd(Q, K, V, 0.3, causal=True, rows=rows)
    assert np.array_equal(Os[0, 0], O[0, 0, rows]) and np.array_equal(Ls[0, 0], L[0, 0, rows])


# ---------------------------------------------------------------- blockwise == one pass


def _compositions(n):
    """Every split of range(n) into consecutive non-empty blocks, as block right ends."""
    for cuts in itertools.product([0, 1], repeat=n - 1):
        ends = [i + 1 for i, c in enumerate(cuts) if c] + [n]
        yield ends


@pytest.mark.parametrize("n,d,seed", [(1, 2, 1), (3, 2, 2), (5, 3, 3), (8, 4, 4)])
def test_online_equals_one_pass_every_split(n, d, seed):
    s = _rand(100 + seed, (n,)) * 3.0
    V = _rand(200 + seed, (n, d))
    Q, K, _ = _worked_qkv(s, d)
    O1, L1 = oracle.fwd(Q, K, V[None, None], 1.0)
    for ends in _compositions(n):
        O, m, l, _, _ = oracle.online_row(s, V, ends)
        assert np.max(np.abs(O - O1[0, 0, 0])) <= 1e-12
        assert abs(m + math.log(l) - L1[0, 0, 0]) <= 1e-12
        # normalised merge applied block by block gives the same row
        mm, ll, OO = -np.inf, 0.0, np.zeros(d)
        start = 0
        for e in ends:
            Ob, mb, lb, _, _ = oracle.online_row(s[start:e], V[start:e], [e - start])
            mm, ll, OO = oracle.merge(mm, ll, OO, mb, lb, Ob)
            start = e
        assert np.max(np.abs(OO - O1[0, 0, 0])) <= 1e-12


def test_online_with_masked_entries():
    s = np.array([-np.inf, 1.0, -np.inf, 2.5, 0.5, -np.inf])
    V = _rand(301, (6, 3))
    ends_all = list(_compositions(6))
    ref = None
    for ends in ends_all:
        O, m, l, _, _ = oracle.online_row(s, V, ends)
        ref = O if ref is None else ref
        assert np.max(np.abs(O - ref)) <= 1e-14
    w = np.exp(np.array([1.0, 2.5, 0.5]) - 2.5)
    exp_O = (w[:, None] * V[[1, 3, 4]]).sum(0) / w.sum()
    assert np.max(np.abs(ref - exp_O)) <= 1e-14


# ---------------------------------------------------------------- library witness


@pytest.mark.parametrize("causal,klen", [(False, None), (True, None), (True, 19), (False, 5)])
def test_torch_fp64_witness_forward(causal, klen):
    import torch

    Q = _rand(401, (2, 4, 13, 16))
    K = _rand(402, (2, 2, 23, 16))
    V = _rand(403, (2, 2, 23, 16))
    kl = None if klen is None else [klen, 23]
    O, L = oracle.fwd(Q, K, V, 0.25, causal=causal, k_lens=kl)
    q = torch.from_numpy(Q)
    k = torch.from_numpy(np.repeat(K, 2, axis=1))
    v = torch.from_numpy(np.repeat(V, 2, axis=1))
    s = q @ k.transpose(-1, -2) * 0.25
    i = torch.arange(13)[:, None]
    j = torch.arange(23)[None, :]
    for b in range(2):
        keep = torch.ones(13, 23, dtype=torch.bool)
        if causal:
            keep &= j <= i + 10
        if kl is not None:
            keep &= j < kl[b]
        s[b] = s[b].masked_fill(~keep, float("-inf"))
    ref_L = torch.logsumexp(s, dim=-1)
    ref_O = torch.softmax(s, dim=-1) @ v
    assert np.max(np.abs(O - ref_O.numpy())) <= 1e-13
    assert np.max(np.abs(L - ref_L.numpy())) <= 1e-13


# ---------------------------------------------------------------- backward


def _loss(Q, K, V, dO, scale, causal, k_lens):
    O, _ = oracle.fwd(Q, K, V, scale, causal=causal, k_lens=k_lens)
    return float(np.sum(O * dO))


@pytest.mark.parametrize("causal,k_lens,Hq,Hkv", [(False, None, 1, 1), (True, None, 1, 1),
                                                   (True, [4], 2, 1), (False, [2], 2, 2)])
def test_backward_central_differences(causal, k_lens, Hq, Hkv):
    rng = np.random.default_rng(7)
    Lq, Lk, d = 3, 5, 2
    Q = rng.standard_normal((1, Hq, Lq, d))
    K = rng.standard_normal((1, Hkv, Lk, d))
    V = rng.standard_normal((1, Hkv, Lk, d))
    dO = rng.standard_normal((1, Hq, Lq, d))
    scale = 0.7
    dQ, dK, dV = oracle.bwd(Q, K, V, dO, scale, causal=causal, k_lens=k_lens)
    h = 1e-5
    for X, G in ((Q, dQ), (K, dK), (V, dV)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            old = X[idx]
            X[idx] = old + h
            fp = _loss(Q, K, V, dO, scale, causal, k_lens)
            X[idx] = old - h
            fm = _loss(Q, K, V, dO, scale, causal, k_lens)
            X[idx] = old
            num[idx] = (fp - fm) / (2 * h)
        err = np.max(np.abs(num - G)) / max(1e-12, np.max(np.abs(G)))
        assert err <= 1e-6, err


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    Q = _rand(501, (1, 2, 17, 8))
    K = _rand(502, (1, 2, 21, 8))
    V = _rand(503, (1, 2, 21, 8))
    dO = _rand(504, (1, 2, 17, 8))
    dQ, dK, dV = oracle.bwd(Q, K, V, dO, 0.3, causal=causal)
    # every row of dS sums to zero, so the key gradients sum to zero
    assert np.max(np.abs(dK.sum(axis=2))) <= 1e-12
    # every visible row of P sums to one, so sum_j dV_j = sum_i dO_i
    assert np.max(np.abs(dV.sum(axis=2) - dO.sum(axis=2))) <= 1e-12


def test_backward_gqa_is_sum_of_heads():
    Q = _rand(511, (1, 4, 9, 8))
    K = _rand(512, (1, 2, 11, 8))
    V = _rand(513, (1, 2, 11, 8))
    dO = _rand(514, (1, 4, 9, 8))
    dQ, dK, dV = oracle.bwd(Q, K, V, dO, 0.3, causal=True)
    Ke = np.repeat(K, 2, axis=1)
    Ve = np.repeat(V, 2, axis=1)
    dQe, dKe, dVe = oracle.bwd(Q, Ke, Ve, dO, 0.3, causal=True)
    assert np.max(np.abs(dQ - dQe)) <= 1e-13
    assert np.max(np.abs(dK - dKe.reshape(1, 2, 2, 11, 8).sum(2))) <= 1e-13
    assert np.max(np.abs(dV - dVe.reshape(1, 2, 2, 11, 8).sum(2))) <= 1e-13


def test_backward_sampled_matches_full():
    Q = _rand(521, (1, 4, 33, 8))
    K = _rand(522, (1, 2, 40, 8))
    V = _rand(523, (1, 2, 40, 8))
    dO = _rand(524, (1, 4, 33, 8))
    dQ, dK, dV = oracle.bwd(Q, K, V, dO, 0.3, causal=True, k_lens=[37])
    qr = [0, 5, 32, 17]
    kc = [0, 36, 39, 12]
    dQs, dKs, dVs = oracle.bwd_sampled(Q, K, V, dO, 0.3, True, [37], 0, 1, qr, kc)
    assert np.max(np.abs(dQs - dQ[0, 2:4][:, qr])) <= 1e-13
    assert np.max(np.abs(dKs - dK[0, 1, kc])) <= 1e-13
    assert np.max(np.abs(dVs - dV[0, 1, kc])) <= 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_torch_fp64_autograd_witness_backward(causal):
    import torch

    Q = _rand(531, (1, 2, 12, 8))
    K = _rand(532, (1, 2, 15, 8))
    V = _rand(533, (1, 2, 15, 8))
    dO = _rand(534, (1, 2, 12, 8))
    dQ, dK, dV = oracle.bwd(Q, K, V, dO, 0.3, causal=causal)
    q = torch.tensor(Q, requires_grad=True)
    k = torch.tensor(K, requires_grad=True)
    v = torch.tensor(V, requires_grad=True)
    s = q @ k.transpose(-1, -2) * 0.3
    if causal:
        i = torch.arange(12)[:, None]
        j = torch.arange(15)[None, :]
        s = s.masked_fill(~(j <= i + 3), float("-inf"))
    o = torch.softmax(s, dim=-1) @ v
    o.backward(torch.from_numpy(dO))
    assert np.max(np.abs(dQ - q.grad.numpy())) <= 1e-12
    assert np.max(np.abs(dK - k.grad.numpy())) <= 1e-12
    assert np.max(np.abs(dV - v.grad.numpy())) <= 1e-12


# ---------------------------------------------------------------- sliding window


@pytest.mark.parametrize("Lq,Lk", [(12, 12), (7, 12)])
def test_window_wider_than_the_sequence_is_causal(Lq, Lk):
    Q, K, V, dO = (_rand(900 + i, s) for i, s in enumerate(
        [(1, 2, Lq, 16), (1, 1, Lk, 16), (1, 1, Lk, 16), (1, 2, Lq, 16)]))
    O1, L1 = oracle.fwd(Q, K, V, 0.3, causal=True)
    O2, L2 = oracle.fwd(Q, K, V, 0.3, causal=True, window=Lk + 1)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)
    g1 = oracle.bwd(Q, K, V, dO, 0.3, causal=True)
    g2 = oracle.bwd(Q, K, V, dO, 0.3, causal=True, window=Lk + 1)
    for a, b in zip(g1, g2):  # dK, dV sum over threads in any order: equal to rounding
        assert np.allclose(a, b, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("Lq,Lk", [(9, 9), (6, 10)])
def test_window_one_sees_only_the_diagonal_key(Lq, Lk):
    """W = 1: each row's softmax has one term, so O_i = V_{i+off} and
    LSE_i = scale * q_i . k_{i+off}; then P is one-hot, dS = P (dP - D) = 0, so
    dQ = dK = 0 and dV_j gathers dO of the row that sees key j."""
    off = Lk - Lq
    Q, K, V, dO = (_rand(920 + i, s) for i, s in enumerate(
        [(1, 1, Lq, 8), (1, 1, Lk, 8), (1, 1, Lk, 8), (1, 1, Lq, 8)]))
    O, L = oracle.fwd(Q, K, V, 0.25, causal=True, window=1)
    for i in range(Lq):
        j = i + off
        assert np.allclose(O[0, 0, i], V[0, 0, j], rtol=0, atol=1e-15)
        assert math.isclose(L[0, 0, i], 0.25 * float(Q[0, 0, i] @ K[0, 0, j]), rel_tol=1e-13)
    dQ, dK, dV = oracle.bwd(Q, K, V, dO, 0.25, causal=True, window=1)
    assert np.allclose(dQ, 0.0, atol=1e-13) and np.allclose(dK, 0.0, atol=1e-13)
    want = np.zeros_like(dV)
    for i in range(Lq):
        want[0, 0, i + off] = dO[0, 0, i]
    assert np.allclose(dV, want, rtol=0, atol=1e-13)


def test_window_two_is_a_two_term_softmax():
    Lq = Lk = 10
    Q, K, V = (_rand(940 + i, (1, 1, Lq, 8)) for i in range(3))
    O, _ = oracle.fwd(Q, K, V, 0.5, causal=True, window=2)
    for i in range(1, Lq):
        a = 0.5 * float(Q[0, 0, i] @ K[0, 0, i - 1])
        b = 0.5 * float(Q[0, 0, i] @ K[0, 0, i])
        wa, wb = 1.0 / (1.0 + math.exp(b - a)), 1.0 / (1.0 + math.exp(a - b))
        assert np.allclose(O[0, 0, i], wa * V[0, 0, i - 1] + wb * V[0, 0, i], rtol=1e-12,
                           atol=1e-14)
    assert np.allclose(O[0, 0, 0], V[0, 0, 0], rtol=0, atol=1e-15)


@pytest.mark.parametrize("W", [1, 3, 5])
def test_window_visible_set_per_row(W):
    """Brute force on the probability matrix: row i has exactly the keys
    (i + off - W, i + off] that exist, each with positive probability."""
    Lq, Lk = 7, 11
    off = Lk - Lq
    Q, K = _rand(960, (Lq, 8)), _rand(961, (Lk, 8))
    P, _ = oracle.probs(Q, K, 0.4, causal=True, window=W)
    for i in range(Lq):
        want = {j for j in range(Lk) if i + off - W < j <= i + off}
        assert {j for j in range(Lk) if P[i, j] > 0} == want
        assert math.isclose(P[i].sum(), 1.0, rel_tol=1e-13)


def test_window_requires_causal():
    with pytest.raises(ValueError):
        oracle.fwd(_rand(1, (1, 1, 4, 8)), _rand(2, (1, 1, 4, 8)), _rand(3, (1, 1, 4, 8)), 1.0,
                   causal=False, window=2)


# ---------------------------------------------------------------- 8-bit (E4M3) inputs


def test_e4m3_decode_matches_torch_on_every_code():
    """Library witness: torch's float8_e4m3fn widening of all 256 codes."""
    import torch

    c = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_to_f64(c)
    ref = torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_landmark_values():
    """The format's fixed points: zero, smallest subnormal and normal, one, the
    largest finite value, the sign bit."""
    v = oracle.e4m3_to_f64(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0x3F, 0x7E, 0xFE, 0xC0],
                                    dtype=np.uint8))
    assert list(v) == [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.875, 448.0, -448.0, -2.0]
    assert np.signbit(oracle.e4m3_to_f64(np.array([0x80], dtype=np.uint8)))[0]


@pytest.mark.parametrize("L", [1, 128, 129, 300])
def test_dequant_assigns_each_row_its_tile_scale(L):
    """Constant codes 0x38 (= 1.0): every dequantised row equals the scale of
    tile i // 128, including the ragged last tile."""
    nt = (L + 127) // 128
    codes = np.full((2, 3, L, 8), 0x38, dtype=np.uint8)
    scales = (np.arange(2 * 3 * nt, dtype=np.float32).reshape(2, 3, nt) + 1.0) * 0.125
    x = oracle.dequant_tiles(codes, scales)
    for i in range(L):
        assert np.all(x[:, :, i, :] == scales[:, :, i // 128][..., None])
    with pytest.raises(ValueError):
        oracle.dequant_tiles(codes, scales[..., :nt - 1] if nt > 1 else np.zeros((2, 3, 2)))


def _fp8_case(seed, B=1, Hq=2, Hkv=1, Lq=200, Lk=300, d=16):
    Q8, qs = synth.normal_e4m3(seed, (B, Hq, Lq, d))
    K8, ks = synth.normal_e4m3(seed + 1, (B, Hkv, Lk, d))
    V8, vs = synth.normal_e4m3(seed + 2, (B, Hkv, Lk, d))
    return Q8, K8, V8, qs, ks, vs


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_scale_invariances(causal):
    """A factor c on every V scale multiplies O by c and leaves LSE; a factor on
    the Q scales traded against the softmax scale changes nothing; a per-tile
    power of two moved from K's codes into K's scales changes nothing (catches a
    Q/K/V scale mix-up or a wrong tile index)."""
    Q8, K8, V8, qs, ks, vs = _fp8_case(931)
    sc = 0.25
    O, L = oracle.fwd_fp8(Q8, K8, V8, qs, ks, vs, sc, causal=causal)
    O2, L2 = oracle.fwd_fp8(Q8, K8, V8, qs, ks, vs.astype(np.float64) * 3.0, sc, causal=causal)
    assert np.allclose(O2, 3.0 * O, rtol=1e-13, atol=1e-14) and np.allclose(L2, L, atol=1e-13)
    O3, L3 = oracle.fwd_fp8(Q8, K8, V8, qs.astype(np.float64) * 3.0, ks, vs, sc / 3.0, causal=causal)
    assert np.allclose(O3, O, atol=1e-13) and np.allclose(L3, L, atol=1e-13)
    # halve the codes of K tile 1 (exponent field - 1 on normal codes) and double its scale
    K8b, ksb = K8.copy(), ks.copy()
    t1 = K8b[:, :, 128:256, :]
    e = (t1 >> 3) & 0xF
    assert np.all((e >= 2) | (t1 & 0x7F == 0)), "test codes must stay normal when halved"
    t1[...] = np.where(t1 & 0x7F == 0, t1, t1 - 8)
    ksb[:, :, 1] *= 2.0
    O4, L4 = oracle.fwd_fp8(Q8, K8b, V8, qs, ksb, vs, sc, causal=causal)
    assert np.allclose(O4, O, atol=1e-13) and np.allclose(L4, L, atol=1e-13)


def test_fp8_brute_force_against_torch():
    """Tiny case: decode with torch, assign tile scales row by row, softmax in
    torch fp64 -- against the oracle."""
    import torch

    Q8, K8, V8, qs, ks, vs = _fp8_case(977, B=2, Hq=2, Hkv=2, Lq=140, Lk=260, d=8)

    def deq(c, s):
        x = torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64)
        out = torch.empty_like(x)
        for i in range(x.shape[2]):
            out[:, :, i, :] = x[:, :, i, :] * torch.from_numpy(s[:, :, i // 128].astype(np.float64))[..., None]
        return out

    q, k, v = deq(Q8, qs), deq(K8, ks), deq(V8, vs)
    s = q @ k.transpose(-1, -2) * 0.3
    i = torch.arange(140)[:, None]
    j = torch.arange(260)[None, :]
    s = s.masked_fill(~(j <= i + 120), float("-inf"))
    O, L = oracle.fwd_fp8(Q8, K8, V8, qs, ks, vs, 0.3, causal=True)
    assert np.max(np.abs(O - (torch.softmax(s, -1) @ v).numpy())) <= 1e-12
    assert np.max(np.abs(L - torch.logsumexp(s, -1).numpy())) <= 1e-12

