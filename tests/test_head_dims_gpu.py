"""Head dims 32 and 96 (page 3 section 3 states Q, K, V as N x d with d general):
their tiles are 32-column blocks with 64-byte swizzle, so these shapes exercise
a second shared-memory layout in every kernel.  Parity with the fp64 oracle for
the forward, both backwards and decoding, on several tiles with ragged ends."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_108_b200 import binding
from exact_attention_108_b200.workloads import make_inputs, to_f64
from gpu_common import assert_device_ok, check_grad, check_lse, check_o, gpu_inputs

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, H, N, seed
    (1, 2, 384, 70),    # three whole tiles
    (2, 1, 300, 71),    # ragged last tile
    (1, 3, 1000, 72),   # eight tiles, odd pair count
]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("B,H,N,seed", SHAPES)
@pytest.mark.parametrize("d", [32, 96])
def test_head_dim_fwd_bwd_match_oracle(d, B, H, N, seed, causal):
    (q, k, v, do), (qg, kg, vg, dog) = gpu_inputs(B, H, N, d, seed)
    scale = 1.0 / math.sqrt(d)
    o, lse = binding.fwd(qg, kg, vg, causal=causal, scale=scale)
    g_red = binding.bwd(qg, kg, vg, o, lse, dog, causal=causal, scale=scale)
    g_det = binding.bwd_ex(qg, kg, vg, o, lse, dog, causal=causal, scale=scale, deterministic=True)
    assert_device_ok()
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.ref_fwd(qf, kf, vf, causal, scale)
    check_o(o, o_ref, f"d={d}")
    check_lse(lse, lse_ref, f"d={d}")
    refs = oracle.ref_bwd(qf, kf, vf, dof, causal, scale)
    for gs, what in ((g_red, "reduce-add"), (g_det, "deterministic")):
        for g, r, n in zip(gs, refs, ("dQ", "dK", "dV")):
            check_grad(g, r, n, f"d={d} {what}")


@pytest.mark.parametrize("d", [32, 96])
def test_head_dim_grouped_uneven_lengths(d):
    g = torch.Generator("cpu").manual_seed(73)
    q = torch.randn((1, 4, 200, d), generator=g).to(torch.bfloat16)
    k = torch.randn((1, 2, 333, d), generator=g).to(torch.bfloat16)
    v = torch.randn((1, 2, 333, d), generator=g).to(torch.bfloat16)
    do = torch.randn((1, 4, 200, d), generator=g).to(torch.bfloat16)
    qg, kg, vg, dog = (t.cuda() for t in (q, k, v, do))
    o, lse = binding.fwd_ex(qg, kg, vg, causal=True)
    grads = binding.bwd_ex(qg, kg, vg, o, lse, dog, causal=True)
    od, ld = binding.decode(qg[:, :, -3:].contiguous(), kg, vg, causal=True, num_splits=2)
    assert_device_ok()
    scale = 1.0 / math.sqrt(d)
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.ref_fwd_general(qf, kf, vf, True, scale)
    check_o(o, o_ref, f"d={d} grouped")
    check_lse(lse, lse_ref, f"d={d} grouped")
    for gr, r, n in zip(grads, oracle.ref_bwd_general(qf, kf, vf, dof, True, scale), ("dQ", "dK", "dV")):
        check_grad(gr, r, n, f"d={d} grouped")
    od_ref, ld_ref = oracle.ref_fwd_general(qf[:, :, -3:], kf, vf, True, scale)
    check_o(od, od_ref, f"d={d} decode")
    check_lse(ld, ld_ref, f"d={d} decode")


D256_CASES = [
    # B, H, H_kv, N_q, N_k, causal
    (1, 2, 2, 384, 384, False),
    (1, 2, 2, 384, 384, True),
    (2, 4, 2, 300, 1000, True),    # grouped heads, N_q < N_k, ragged
    (1, 2, 1, 500, 200, True),     # N_q > N_k: rows 0..299 see no key
    (1, 3, 3, 1000, 1000, False),
]


@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,causal", D256_CASES)
def test_head_dim_256_forward(B, H, H_kv, N_q, N_k, causal):
    """d = 256: the forward runs the one-query-tile-per-CTA kernel of the decoding path
    (two query tiles with their 256-column accumulators would not fit in TMEM)."""
    d = 256
    g = torch.Generator("cpu").manual_seed(80 + N_q)
    q = torch.randn((B, H, N_q, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, H_kv, N_k, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, H_kv, N_k, d), generator=g).to(torch.bfloat16)
    qg, kg, vg = (t.cuda() for t in (q, k, v))
    scale = 1.0 / math.sqrt(d)
    o, lse = binding.fwd_ex(qg, kg, vg, causal=causal, scale=scale)
    od, ld = binding.decode(qg[:, :, -4:].contiguous(), kg, vg, causal=causal, num_splits=3)
    assert_device_ok()
    qf, kf, vf = (to_f64(t) for t in (q, k, v))
    o_ref, lse_ref = oracle.ref_fwd_general(qf, kf, vf, causal, scale)
    check_o(o, o_ref, "d=256")
    g_lse = lse.double().cpu().numpy()
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(g_lse), empty)
    assert np.abs(g_lse[~empty] - lse_ref[~empty]).max() <= 1e-3
    od_ref, ld_ref = oracle.ref_fwd_general(qf[:, :, -4:], kf, vf, causal, scale)
    check_o(od, od_ref, "d=256 decode")
    check_lse(ld, ld_ref, "d=256 decode")
    if B * H == 2 and N_q == N_k:  # the plain entry point takes the same path
        o2, l2 = binding.fwd(qg, kg, vg, causal=causal, scale=scale)
        assert_device_ok()
        assert torch.equal(o, o2) and torch.equal(lse, l2)
