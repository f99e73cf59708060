"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each.

Every mutation replaces one step of ``oracle.attention_fp64`` for the duration of
one test; the named pin from ``test_oracle`` must then fail.
"""
import numpy as np
import pytest

from oracle import attention_fp64 as A
import test_oracle as pins
import test_oracle_general as gpins


def _softmax_no_norm(s):
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    return e, (m + np.log(e.sum(1, keepdims=True)))[:, 0]


def _softmax_lse_without_max(s):
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(1, keepdims=True)
    return e / z, np.log(z)[:, 0]


MUTATIONS = [
    # (name, attribute, replacement, pin that must fail)
    ("scale dropped", "scores", lambda q, k, scale: q @ k.T,
     lambda: pins.test_ref_fwd_matches_brute_force(False, 7, 4, 0.37)),
    ("scores transposed", "scores",
     lambda q, k, scale: scale * (k @ q.T) if q.shape[0] == k.shape[0] else scale * (q @ k.T),
     lambda: pins.test_ref_fwd_matches_brute_force(False, 7, 4, 0.37)),
    ("mask excludes diagonal", "causal_keep",
     lambda rows, n: np.arange(n)[None, :] < rows[:, None],
     lambda: pins.test_causal_row_zero_is_first_value()),
    ("mask one past diagonal", "causal_keep",
     lambda rows, n: np.arange(n)[None, :] <= rows[:, None] + 1,
     lambda: pins.test_ref_fwd_matches_brute_force(True, 7, 4, None)),
    ("softmax not normalised", "softmax_rows", _softmax_no_norm,
     lambda: pins.test_probs_rows_sum_to_one_and_mask_is_exact_zero()),
    ("LSE misses the max", "softmax_rows", _softmax_lse_without_max,
     lambda: pins.test_probs_match_scipy_softmax(False)),
    ("softmax gradient sign", "softmax_grad",
     lambda p, dp: p * (np.sum(p * dp, 1, keepdims=True) - dp),
     lambda: pins.test_ref_bwd_matches_finite_differences(False)),
    ("softmax gradient row term dropped", "softmax_grad", lambda p, dp: p * dp,
     lambda: pins.test_backward_column_sums(True)),
    ("causal mask aligned top-left", "causal_keep",
     lambda rows, n, offset=0: np.arange(n)[None, :] <= np.asarray(rows)[:, None],
     lambda: gpins.test_general_fwd_matches_brute_force(1, 2, 2, 3, 7, 4, True, 0.0)),
    ("key/value head by modulo", "kv_head_of", lambda h, H, H_kv: h % H_kv,
     lambda: gpins.test_general_fwd_matches_brute_force(1, 4, 2, 7, 3, 3, False, 0.0)),
    ("dropout kept weights not rescaled", "dropout_multiplier",
     lambda bh, rows, n_k, p, seed, offset: (_orig_mult(bh, rows, n_k, p, seed, offset) > 0).astype(float),
     lambda: gpins.test_dropped_output_is_unbiased()),
    ("rows with no visible key left undefined", "softmax_rows_masked", A.softmax_rows,
     lambda: gpins.test_general_fwd_matches_brute_force(1, 4, 2, 7, 3, 3, True, 0.0)),
]
_orig_mult = A.dropout_multiplier


@pytest.mark.parametrize("name,attr,repl,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pin_catches_planted_mistake(monkeypatch, name, attr, repl, pin):
    monkeypatch.setattr(A, attr, repl)
    with np.errstate(all="ignore"):
        with pytest.raises(AssertionError):
            pin()
