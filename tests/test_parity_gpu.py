"""GPU parity: libfattn forward and backward against the fp64 oracle, element by
element, on seeded inputs small enough for the oracle to finish in seconds but
spanning several 128-row tiles."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_108_b200 import binding
from exact_attention_108_b200.workloads import WORKLOADS, to_f64
from gpu_common import assert_device_ok, check_grad, check_lse, check_o, gpu_inputs

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, H, N, d, seed, dist
    (1, 1, 128, 64, 0, "normal"),     # the tiny workload: one tile
    (2, 2, 384, 64, 11, "normal"),    # three tiles, several heads
    (1, 3, 512, 128, 12, "normal"),   # four tiles, d = 128
    (2, 1, 256, 128, 13, "peaked"),   # |s| ~ 100 stress at small size
    (1, 2, 1024, 64, 14, "normal"),   # eight tiles (ring wraps several times)
    (1, 1, 1152, 128, 15, "normal"),  # nine tiles: odd tile count
]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("B,H,N,d,seed,dist", SHAPES)
def test_fwd_bwd_match_oracle(B, H, N, d, seed, dist, causal):
    (q, k, v, do), (qg, kg, vg, dog) = gpu_inputs(B, H, N, d, seed, dist)
    scale = 1.0 / math.sqrt(d)
    o, lse = binding.fwd(qg, kg, vg, causal=causal, scale=scale)
    dq, dk, dv = binding.bwd(qg, kg, vg, o, lse, dog, causal=causal, scale=scale)
    assert_device_ok()
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.ref_fwd(qf, kf, vf, causal, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)
    dq_ref, dk_ref, dv_ref = oracle.ref_bwd(qf, kf, vf, dof, causal, scale)
    check_grad(dq, dq_ref, "dQ")
    check_grad(dk, dk_ref, "dK")
    check_grad(dv, dv_ref, "dV")


def test_tiny_workload_forward_backward():
    w = WORKLOADS["tiny"]
    (q, k, v, do), (qg, kg, vg, dog) = gpu_inputs(w.B, w.H, w.N, w.d, w.seed, w.dist)
    o, lse = binding.fwd(qg, kg, vg, causal=w.causal, scale=w.scale)
    dq, dk, dv = binding.bwd(qg, kg, vg, o, lse, dog, causal=w.causal, scale=w.scale)
    assert_device_ok()
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.ref_fwd(qf, kf, vf, w.causal, w.scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)
    for g, r, n in zip((dq, dk, dv), oracle.ref_bwd(qf, kf, vf, dof, w.causal, w.scale), "QKV"):
        check_grad(g, r, "d" + n)


def _check_o_derived(o, o_ref, v_ref):
    """Off-workload scales: the bound the arithmetic itself gives.  P is rounded
    to bf16 before the PV product (unit roundoff 2^-8 per weight, so at most
    2^-8 * max|V| on a row) and O is rounded to bf16 on output (<= 2^-8 |O|).
    The fp32 exponentials and accumulation add errors near 2^-20 relative per
    term, covered by a 2^-14 * max|V| allowance."""
    err = np.abs(to_f64(o) - o_ref)
    bound = 2.0 ** -8 * (np.abs(v_ref).max() + np.abs(o_ref)) + 2.0 ** -14 * np.abs(v_ref).max()
    assert (err <= bound).all(), f"O error {err.max():.3e} exceeds the bf16 rounding bound"
    assert err.mean() <= 1e-3


@pytest.mark.parametrize("scale", [0.0, -0.2, 0.5])
def test_unusual_scales(scale):
    (q, k, v, do), (qg, kg, vg, dog) = gpu_inputs(1, 2, 256, 64, 21)
    for causal in (False, True):
        o, lse = binding.fwd(qg, kg, vg, causal=causal, scale=scale)
        dq, dk, dv = binding.bwd(qg, kg, vg, o, lse, dog, causal=causal, scale=scale)
        assert_device_ok()
        qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
        o_ref, lse_ref = oracle.ref_fwd(qf, kf, vf, causal, scale)
        _check_o_derived(o, o_ref, vf)
        check_lse(lse, lse_ref)
        for g, r, n in zip((dq, dk, dv), oracle.ref_bwd(qf, kf, vf, dof, causal, scale), "QKV"):
            if n == "V" or scale != 0.0:
                check_grad(g, r, "d" + n)
            else:  # scale 0: dQ = dK = 0 exactly
                assert torch.count_nonzero(g).item() == 0


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("N", [100, 200, 1000])
@pytest.mark.parametrize("scale", [0.0, -0.2])
def test_unusual_scales_ragged(scale, N, causal):
    """Zero and negative scales on sequence lengths with a ragged last tile: the
    keys past N must get weight 0 even where scale * (masked score) is 0 * inf."""
    (q, k, v, do), (qg, kg, vg, dog) = gpu_inputs(1, 2, N, 64, 24)
    o, lse = binding.fwd(qg, kg, vg, causal=causal, scale=scale)
    dq, dk, dv = binding.bwd(qg, kg, vg, o, lse, dog, causal=causal, scale=scale)
    assert_device_ok()
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.ref_fwd(qf, kf, vf, causal, scale)
    _check_o_derived(o, o_ref, vf)
    check_lse(lse, lse_ref)
    for g, r, n in zip((dq, dk, dv), oracle.ref_bwd(qf, kf, vf, dof, causal, scale), "QKV"):
        if n == "V" or scale != 0.0:
            check_grad(g, r, "d" + n)
        else:  # scale 0: dQ = dK = 0 exactly
            assert torch.count_nonzero(g).item() == 0


def test_repeated_calls_are_identical():
    _, (qg, kg, vg, dog) = gpu_inputs(2, 2, 512, 128, 22)
    o1, l1 = binding.fwd(qg, kg, vg, causal=True)
    o2, l2 = binding.fwd(qg, kg, vg, causal=True)
    assert_device_ok()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    dq1, dk1, dv1 = binding.bwd(qg, kg, vg, o1, l1, dog, causal=True)
    dq2, dk2, dv2 = binding.bwd(qg, kg, vg, o1, l1, dog, causal=True)
    assert_device_ok()
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    # dQ goes through fp32 atomics: equal up to the order of additions
    assert (dq1.float() - dq2.float()).abs().max().item() <= 1e-2 * dq1.float().abs().max().item()


def test_runs_on_a_side_stream():
    (q, k, v, _), (qg, kg, vg, _) = gpu_inputs(1, 2, 256, 64, 23, with_do=False)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, lse = binding.fwd(qg, kg, vg, causal=False, stream=s)
    s.synchronize()
    assert_device_ok()
    qf, kf, vf = (to_f64(t) for t in (q, k, v))
    o_ref, lse_ref = oracle.ref_fwd(qf, kf, vf, False, 1 / 8)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)
