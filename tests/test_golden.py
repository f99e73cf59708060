"""The oracle reproduces its committed golden record (tests/golden/tiny_oracle_case.json).

The record was written by tests/golden/make_golden.py, which calls only the
oracle; it guards against unintended changes to the oracle's arithmetic.
"""
import json
import os

import numpy as np
import pytest

import oracle

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("mode", ["full", "causal"])
def test_oracle_matches_golden_record(mode):
    with open(os.path.join(HERE, "tiny_oracle_case.json")) as f:
        case = json.load(f)
    q, k, v, do = (np.array(case[n]) for n in ("q", "k", "v", "do"))
    causal = mode == "causal"
    o, lse = oracle.ref_fwd(q, k, v, causal, case["scale"])
    dq, dk, dv = oracle.ref_bwd(q, k, v, do, causal, case["scale"])
    exp = case[mode]
    for name, got in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(got, np.array(exp[name]), rtol=1e-12, atol=1e-13, err_msg=name)
