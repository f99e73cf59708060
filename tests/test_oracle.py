"""Pins for the fp64 oracle: each check fixes the oracle to something other than itself.

* brute force (independent pure-Python loops) on tiny shapes;
* central finite differences of L = sum(dO * O) for the backward;
* a library softmax / logsumexp (scipy) on the masked scaled scores;
* closed forms: identical keys, Q = 0, causal row 0, N = 1, key shift;
* invariants: rows of P sum to 1, permutation invariance, sum_j dK_j = 0,
  sum_j dV_j = sum_i dO_i;
* a 60-digit Decimal evaluation of the peaked (|s| ~ 100) stress case.
"""
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest
import scipy.special

import oracle
from oracle import attention_fp64 as A

RNG = np.random.default_rng(1234)


def _rand(shape, scale=1.0):
    return scale * RNG.standard_normal(shape)


def _lists(x):
    return x.tolist()


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 1), (3, 2), (7, 4), (16, 8)])
@pytest.mark.parametrize("scale", [None, 0.37, -0.5])
def test_ref_fwd_matches_brute_force(causal, N, d, scale):
    q, k, v = _rand((1, 2, N, d)), _rand((1, 2, N, d)), _rand((1, 2, N, d))
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    o, lse = oracle.ref_fwd(q, k, v, causal, sc)
    ob, lb = oracle.brute_fwd(_lists(q), _lists(k), _lists(v), causal, sc)
    np.testing.assert_allclose(o, np.array(ob), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(lb), rtol=1e-12, atol=1e-12)


def test_row_blocking_does_not_change_result():
    q, k, v = _rand((2, 1, 37, 5)), _rand((2, 1, 37, 5)), _rand((2, 1, 37, 5))
    for causal in (False, True):
        o1, l1 = oracle.ref_fwd(q, k, v, causal, 0.4)
        o2, l2 = oracle.ref_fwd(q, k, v, causal, 0.4, row_block=4)
        np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(l1, l2, rtol=1e-13, atol=1e-14)


# -------------------------------------------------------- finite differences
@pytest.mark.parametrize("causal", [False, True])
def test_ref_bwd_matches_finite_differences(causal):
    B, H, N, d = 1, 1, 5, 3
    q, k, v, do = (_rand((B, H, N, d)) for _ in range(4))
    dq, dk, dv = oracle.ref_bwd(q, k, v, do, causal, 0.7)
    fq, fk, fv = oracle.finite_diff_grads(q, k, v, do, causal, 0.7)
    for g, f in ((dq, fq), (dk, fk), (dv, fv)):
        np.testing.assert_allclose(g, f, rtol=1e-7, atol=1e-8)


def test_ref_bwd_row_blocking_and_sampled_rows():
    N, d = 40, 6
    q, k, v, do = (_rand((N, d)) for _ in range(4))
    for causal in (False, True):
        a = oracle.ref_bwd_head(q, k, v, do, causal, 0.3)
        b = oracle.ref_bwd_head(q, k, v, do, causal, 0.3, row_block=7)
        for x, y in zip(a, b):
            np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-13)
        rows = [0, 5, 39]
        np.testing.assert_allclose(oracle.ref_dq_rows(q, k, v, do, rows, causal, 0.3),
                                   a[0][rows], rtol=1e-12, atol=1e-13)
        o_r, l_r = oracle.ref_fwd_rows(q, k, v, rows, causal, 0.3)
        o, lse = oracle.ref_fwd(q[None, None], k[None, None], v[None, None], causal, 0.3)
        np.testing.assert_allclose(o_r, o[0, 0, rows], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(l_r, lse[0, 0, rows], rtol=1e-12, atol=1e-13)


# ------------------------------------------------------ library softmax pin
@pytest.mark.parametrize("causal", [False, True])
def test_probs_match_scipy_softmax(causal):
    N, d = 33, 8
    q, k = _rand((1, 1, N, d)), _rand((1, 1, N, d))
    sc = 1 / math.sqrt(d)
    p = oracle.ref_probs(q, k, causal, sc)[0, 0]
    s = np.einsum("id,jd->ij", q[0, 0], k[0, 0]) * sc
    if causal:
        s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
    np.testing.assert_allclose(p, scipy.special.softmax(s, axis=1), rtol=1e-12, atol=1e-15)
    _, lse = oracle.ref_fwd(q, k, _rand((1, 1, N, d)), causal, sc)
    np.testing.assert_allclose(lse[0, 0], scipy.special.logsumexp(s, axis=1), rtol=1e-13)


def test_probs_rows_sum_to_one_and_mask_is_exact_zero():
    q, k = _rand((1, 2, 29, 4)), _rand((1, 2, 29, 4))
    for causal in (False, True):
        p = oracle.ref_probs(q, k, causal, 0.9)
        np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
        assert (p >= 0).all()
        if causal:
            assert np.all(p[..., np.triu_indices(29, 1)[0], np.triu_indices(29, 1)[1]] == 0.0)


# ------------------------------------------------------------ closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_values(causal):
    N, d = 24, 5
    q = _rand((1, 1, N, d))
    key = _rand((d,))
    k = np.broadcast_to(key, (1, 1, N, d)).copy()
    v = _rand((1, 1, N, d))
    o, lse = oracle.ref_fwd(q, k, v, causal, 0.6)
    counts = np.arange(1, N + 1) if causal else np.full(N, N)
    mean = np.cumsum(v[0, 0], axis=0) / counts[:, None] if causal else np.broadcast_to(
        v[0, 0].mean(0), (N, d))
    np.testing.assert_allclose(o[0, 0], mean, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], 0.6 * q[0, 0] @ key + np.log(counts), rtol=1e-12)


def test_zero_queries_give_uniform_attention():
    N, d = 19, 3
    q = np.zeros((1, 1, N, d))
    k, v = _rand((1, 1, N, d)), _rand((1, 1, N, d))
    o, lse = oracle.ref_fwd(q, k, v, False, 0.5)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(0), (N, d)), atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.log(N), atol=1e-14)
    o, lse = oracle.ref_fwd(q, k, v, True, 0.5)
    np.testing.assert_allclose(o[0, 0], np.cumsum(v[0, 0], 0) / np.arange(1, N + 1)[:, None],
                               atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.log(np.arange(1, N + 1)), atol=1e-14)


def test_causal_row_zero_is_first_value():
    q, k, v = _rand((2, 3, 11, 4)), _rand((2, 3, 11, 4)), _rand((2, 3, 11, 4))
    o, lse = oracle.ref_fwd(q, k, v, True, 0.8)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-15)
    np.testing.assert_allclose(lse[:, :, 0], 0.8 * np.sum(q[:, :, 0] * k[:, :, 0], -1), rtol=1e-13)


def test_single_key_returns_value():
    q, k, v = _rand((1, 2, 1, 7)), _rand((1, 2, 1, 7)), _rand((1, 2, 1, 7))
    for causal in (False, True):
        o, _ = oracle.ref_fwd(q, k, v, causal, 1.3)
        np.testing.assert_allclose(o, v, atol=1e-15)


def test_key_shift_leaves_output_and_shifts_lse():
    N, d = 21, 6
    q, k, v = _rand((1, 1, N, d)), _rand((1, 1, N, d)), _rand((1, 1, N, d))
    c = _rand((d,))
    for causal in (False, True):
        o1, l1 = oracle.ref_fwd(q, k, v, causal, 0.45)
        o2, l2 = oracle.ref_fwd(q, k + c, v, causal, 0.45)
        np.testing.assert_allclose(o1, o2, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(l2 - l1, 0.45 * (q @ c), rtol=1e-10, atol=1e-12)


def test_permuting_keys_and_values_together_is_invariant():
    N, d = 26, 4
    q, k, v = _rand((1, 1, N, d)), _rand((1, 1, N, d)), _rand((1, 1, N, d))
    perm = RNG.permutation(N)
    o1, l1 = oracle.ref_fwd(q, k, v, False, 0.5)
    o2, l2 = oracle.ref_fwd(q, k[:, :, perm], v[:, :, perm], False, 0.5)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-13)


# ------------------------------------------------------ backward invariants
@pytest.mark.parametrize("causal", [False, True])
def test_backward_column_sums(causal):
    N, d = 30, 5
    q, k, v, do = (_rand((N, d)) for _ in range(4))
    dq, dk, dv = oracle.ref_bwd_head(q, k, v, do, causal, 0.55)
    # sum_j ds_ij = 0 for every row  =>  sum_j dK_j = 0
    np.testing.assert_allclose(dk.sum(0), 0.0, atol=1e-12)
    # sum_j P_ij = 1 for every row   =>  sum_j dV_j = sum_i dO_i
    np.testing.assert_allclose(dv.sum(0), do.sum(0), atol=1e-12)


def test_backward_dv_is_probs_transpose_times_dout():
    N, d = 17, 3
    q, k, v, do = (_rand((1, 1, N, d)) for _ in range(4))
    sc = 0.9
    s = np.einsum("id,jd->ij", q[0, 0], k[0, 0]) * sc
    p = scipy.special.softmax(s, axis=1)
    _, _, dv = oracle.ref_bwd(q, k, v, do, False, sc)
    np.testing.assert_allclose(dv[0, 0], p.T @ do[0, 0], rtol=1e-12, atol=1e-13)


# ------------------------------------------------------ peaked stress case
def _decimal_attention_row(qi, k, v, scale, visible):
    getcontext().prec = 60
    logits = [Decimal(scale) * sum(Decimal(float(a)) * Decimal(float(b)) for a, b in zip(qi, k[j]))
              for j in visible]
    w = [x.exp() for x in logits]  # no max subtraction: Decimal has the range
    total = sum(w)
    out = [float(sum(wj * Decimal(float(v[j][c])) for wj, j in zip(w, visible)) / total)
           for c in range(len(v[0]))]
    return out, float(total.ln())


@pytest.mark.parametrize("causal", [False, True])
def test_peaked_scores_against_high_precision(causal):
    N, d = 12, 16
    q, k = _rand((1, 1, N, d), 4.0), _rand((1, 1, N, d), 4.0)
    v = RNG.uniform(-1, 1, (1, 1, N, d))
    sc = 1 / math.sqrt(d) * 4  # push |s| to ~100
    s = sc * np.einsum("id,jd->ij", q[0, 0], k[0, 0])
    assert np.abs(s).max() > 60
    o, lse = oracle.ref_fwd(q, k, v, causal, sc)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    for i in range(N):
        vis = list(range(i + 1)) if causal else list(range(N))
        ref_o, ref_l = _decimal_attention_row(q[0, 0, i], k[0, 0], v[0, 0], sc, vis)
        np.testing.assert_allclose(o[0, 0, i], ref_o, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[0, 0, i], ref_l, rtol=1e-13)
