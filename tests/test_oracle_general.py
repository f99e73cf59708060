"""Pins for the oracle's general form: N_q queries against N_k keys with the causal
mask aligned at the bottom right, grouped key/value heads, and dropout drawn from
Philox4x32-10.

* Philox4x32-10 against the published known-answer vectors of its authors
  (Salmon et al., SC'11, Random123 distribution);
* the dropout mask's layout tied to those vectors, its keep rate against the
  binomial law, and the expectation of the dropped output (1 / (1 - p)
  rescaling) against the undropped one;
* brute force (independent pure-Python loops) on tiny shapes;
* central finite differences of L = sum(dO * O) for the backward;
* special cases that reduce to the square form pinned in test_oracle.py:
  N_q = N_k, H_kv = H, p = 0; and H_kv < H equal to H_kv = H with each key/value
  head repeated over its group.
"""
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(4321)


def _rand(shape, scale=1.0):
    return scale * RNG.standard_normal(shape)


# ----------------------------------------------------------------- Philox
KAT = [  # (counter, key, output) for Philox4x32-10, published with the generator
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF, 0xFFFFFFFF), (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


@pytest.mark.parametrize("ctr,key,out", KAT)
def test_philox_known_answers(ctr, key, out):
    got = oracle.philox4x32_10(tuple(np.array([c], dtype=np.uint64) for c in ctr), key)
    assert tuple(int(w[0]) for w in got) == out


def test_dropout_layout_follows_the_counter_definition():
    # head 0, row 0, keys 0..3 with seed 0, offset 0 use counter (0, 0, 0, 0), key (0, 0):
    # the first known-answer vector
    p = 0.5
    t = oracle.dropout_threshold(p)
    assert t == 1 << 31
    z = oracle.dropout_multiplier(0, [0], 8, p, seed=0, offset=0)
    words = KAT[0][2]
    np.testing.assert_array_equal(z[0, :4], [2.0 if w >= t else 0.0 for w in words])
    # counter (2^32-1, 2^32-1, 2^32-1, 2^32-1), key (2^32-1, 2^32-1): row 2^32-1, keys
    # 4(2^32-1) .. +3, head 2^32-1, offset 2^32-1, seed 2^64-1
    words = KAT[1][2]
    big = 0xFFFFFFFF
    zz = _mult_at(big, big, 4 * big, p, (1 << 64) - 1, big)
    np.testing.assert_array_equal(zz, [2.0 if w >= t else 0.0 for w in words])


def _mult_at(bh, row, col0, p, seed, offset):
    """dropout_multiplier restricted to keys col0..col0+3 without building all columns."""
    cols = np.arange(col0, col0 + 4, dtype=np.int64)
    ctr = (np.full(4, row), cols >> 2, np.full(4, bh), np.full(4, offset))
    words = oracle.philox4x32_10(ctr, (seed & 0xFFFFFFFF, seed >> 32))
    r = np.array([int(words[c & 3][i]) for i, c in enumerate(cols)])
    # the same decision dropout_multiplier takes, from the published words
    full = oracle.dropout_multiplier(bh, [row], 4, p, seed, offset) if col0 == 0 else None
    keep = r >= oracle.dropout_threshold(p)
    out = np.where(keep, 1.0 / (1.0 - p), 0.0)
    if full is not None:
        np.testing.assert_array_equal(full[0], out)
    return out


def test_dropout_threshold_edges():
    assert oracle.dropout_threshold(0.0) == 0
    assert oracle.dropout_threshold(0.25) == 1 << 30
    assert oracle.dropout_threshold(np.float32(0.1)) == math.floor(float(np.float32(0.1)) * 2 ** 32)
    assert oracle.dropout_threshold(1.0 - 2 ** -40) == 2 ** 32 - 1


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
def test_dropout_keep_rate_is_binomial(p):
    z = oracle.dropout_multiplier(3, np.arange(256), 512, p, seed=1234, offset=7)
    n = z.size
    kept = int((z > 0).sum())
    mean = n * (1 - p)
    sd = math.sqrt(n * p * (1 - p))
    assert abs(kept - mean) < 5 * sd
    np.testing.assert_allclose(z[z > 0], 1.0 / (1.0 - p))


def test_dropout_masks_differ_across_heads_offsets_and_seeds():
    base = oracle.dropout_multiplier(0, np.arange(16), 64, 0.5, 1, 0)
    for other in (oracle.dropout_multiplier(1, np.arange(16), 64, 0.5, 1, 0),
                  oracle.dropout_multiplier(0, np.arange(16), 64, 0.5, 1, 1),
                  oracle.dropout_multiplier(0, np.arange(16), 64, 0.5, 2, 0),
                  oracle.dropout_multiplier(0, np.arange(16), 64, 0.5, 1 << 32, 0)):
        assert (other != base).mean() > 0.3


def test_dropped_output_is_unbiased():
    """E[O] over the dropout mask is the undropped O (the kept weights are divided by 1 - p)."""
    B, H, N, d, p = 1, 1, 6, 3, 0.4
    q, k, v = _rand((B, H, N, d)), _rand((B, H, N, d)), _rand((B, H, N, d))
    o0, _ = oracle.ref_fwd_general(q, k, v, False, 0.7)
    acc = np.zeros_like(o0)
    n = 4000
    for s in range(n):
        o, _ = oracle.ref_fwd_general(q, k, v, False, 0.7, dropout_p=p, seed=s)
        acc += o
    # per-element standard error is below sqrt(p/(1-p)) max|V| / sqrt(n)
    np.testing.assert_allclose(acc / n, o0, atol=6 * math.sqrt(p / (1 - p)) * np.abs(v).max() / math.sqrt(n))


# ---------------------------------------------------------------- brute force
GEN_SHAPES = [  # B, H, H_kv, N_q, N_k, d
    (1, 2, 2, 3, 7, 4),   # fewer queries than keys
    (1, 4, 2, 7, 3, 3),   # more queries than keys: causal rows 0..3 see nothing
    (2, 4, 1, 1, 5, 2),   # one query (decode), one key/value head for all
    (1, 3, 3, 5, 5, 4),   # square, no grouping
    (1, 6, 2, 4, 9, 2),   # groups of 3
]


@pytest.mark.parametrize("p", [0.0, 0.3])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d", GEN_SHAPES)
def test_general_fwd_matches_brute_force(B, H, H_kv, N_q, N_k, d, causal, p):
    q, k, v = _rand((B, H, N_q, d)), _rand((B, H_kv, N_k, d)), _rand((B, H_kv, N_k, d))
    sc, seed, off = 0.6, 99, 5
    o, lse = oracle.ref_fwd_general(q, k, v, causal, sc, p, seed, off)
    mult = np.stack([np.stack([oracle.dropout_multiplier(b * H + h, np.arange(N_q), N_k, p, seed, off)
                               for h in range(H)]) for b in range(B)])
    ob, lb = oracle.brute_fwd_general(q.tolist(), k.tolist(), v.tolist(), causal, sc, mult.tolist())
    np.testing.assert_allclose(o, np.array(ob), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(lb), rtol=1e-12, atol=1e-12)
    if causal and N_q > N_k:
        empty = N_q - N_k
        assert np.all(np.isneginf(lse[:, :, :empty])) and np.all(o[:, :, :empty] == 0)
    # sampled rows agree with the whole-head evaluation
    rows = [0, N_q - 1]
    o_r, l_r = oracle.ref_fwd_general_rows(q, k, v, B - 1, H - 1, rows, causal, sc, p, seed, off)
    np.testing.assert_allclose(o_r, o[B - 1, H - 1, rows], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l_r, lse[B - 1, H - 1, rows], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("p", [0.0, 0.3])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d", [(1, 2, 1, 3, 4, 2), (1, 2, 2, 4, 2, 2)])
def test_general_bwd_matches_finite_differences(B, H, H_kv, N_q, N_k, d, causal, p):
    q, k, v, do = _rand((B, H, N_q, d)), _rand((B, H_kv, N_k, d)), _rand((B, H_kv, N_k, d)), \
        _rand((B, H, N_q, d))
    sc, seed, off = 0.8, 5, 2
    got = oracle.ref_bwd_general(q, k, v, do, causal, sc, p, seed, off)
    fd = oracle.finite_diff_grads_general(q, k, v, do, causal, sc, p, seed, off)
    for g, f in zip(got, fd):
        np.testing.assert_allclose(g, f, rtol=1e-7, atol=1e-8)
    rows = [0, N_q - 1]
    np.testing.assert_allclose(oracle.ref_dq_general_rows(q, k, v, do, 0, H - 1, rows, causal, sc, p, seed, off),
                               got[0][0, H - 1, rows], rtol=1e-12, atol=1e-13)


# ------------------------------------------------------ reductions to the square form
@pytest.mark.parametrize("causal", [False, True])
def test_square_case_reduces_to_ref_fwd(causal):
    q, k, v, do = (_rand((2, 3, 9, 4)) for _ in range(4))
    o, lse = oracle.ref_fwd_general(q, k, v, causal, 0.4)
    o2, l2 = oracle.ref_fwd(q, k, v, causal, 0.4)
    np.testing.assert_allclose(o, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, l2, rtol=1e-13, atol=1e-14)
    for a, b in zip(oracle.ref_bwd_general(q, k, v, do, causal, 0.4), oracle.ref_bwd(q, k, v, do, causal, 0.4)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_grouped_heads_equal_repeated_heads(causal):
    B, H, H_kv, N_q, N_k, d = 2, 6, 2, 5, 8, 3
    q, do = _rand((B, H, N_q, d)), _rand((B, H, N_q, d))
    k, v = _rand((B, H_kv, N_k, d)), _rand((B, H_kv, N_k, d))
    rep = lambda t: np.repeat(t, H // H_kv, axis=1)  # noqa: E731
    o, lse = oracle.ref_fwd_general(q, k, v, causal, 0.5)
    o2, l2 = oracle.ref_fwd_general(q, rep(k), rep(v), causal, 0.5)
    np.testing.assert_allclose(o, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, l2, rtol=1e-13, atol=1e-14)
    dq, dk, dv = oracle.ref_bwd_general(q, k, v, do, causal, 0.5)
    dq2, dk2, dv2 = oracle.ref_bwd_general(q, rep(k), rep(v), do, causal, 0.5)
    np.testing.assert_allclose(dq, dq2, rtol=1e-12, atol=1e-13)
    # a shared head's gradient is the sum over the query heads of its group
    np.testing.assert_allclose(dk, dk2.reshape(B, H_kv, H // H_kv, N_k, d).sum(2), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, H_kv, H // H_kv, N_k, d).sum(2), rtol=1e-12, atol=1e-13)


def test_bottom_right_alignment_equals_the_tail_of_a_square_problem():
    """Causal with N_q < N_k: the queries act as the last N_q positions of an N_k-long
    sequence, so their rows equal those rows of the square causal problem."""
    N_q, N_k, d = 4, 11, 3
    k, v = _rand((1, 1, N_k, d)), _rand((1, 1, N_k, d))
    q_full = _rand((1, 1, N_k, d))
    o_full, l_full = oracle.ref_fwd(q_full, k, v, True, 0.9)
    o, lse = oracle.ref_fwd_general(q_full[:, :, N_k - N_q:], k, v, True, 0.9)
    np.testing.assert_allclose(o, o_full[:, :, N_k - N_q:], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, l_full[:, :, N_k - N_q:], rtol=1e-13, atol=1e-14)
