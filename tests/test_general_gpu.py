"""GPU parity of the general entry points (fattn_fwd_ex, fattn_bwd_ex) with the fp64
oracle: separate query and key lengths with the causal mask aligned at the bottom
right, grouped key/value heads, dropout regenerated from (seed, offset), and the
deterministic backward (dQ by its own pass)."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_108_b200 import binding
from exact_attention_108_b200.workloads import to_f64
from gpu_common import assert_device_ok, check_grad, check_o, gpu_inputs, o_max_abs_bound

pytestmark = pytest.mark.gpu


def _inputs(B, H, H_kv, N_q, N_k, d, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, H, N_q, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, H_kv, N_k, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, H_kv, N_k, d), generator=g).to(torch.bfloat16)
    do = torch.randn((B, H, N_q, d), generator=g).to(torch.bfloat16)
    return (q, k, v, do), tuple(t.cuda() for t in (q, k, v, do))


def _check_lse_general(lse, ref, what=""):
    """LSE max-abs <= 1e-3 where the row sees a key; exactly -inf where it sees none."""
    g = lse.double().cpu().numpy()
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(g), empty), f"{what} rows with no visible key differ"
    err = np.abs(g[~empty] - ref[~empty])
    assert np.isfinite(err).all() and (err.size == 0 or err.max() <= 1e-3), f"{what} LSE max-abs {err.max():.3e}"


CASES = [
    # B, H, H_kv, N_q, N_k, d
    (1, 2, 2, 128, 512, 128),   # fewer queries than keys, whole tiles
    (2, 4, 1, 1, 4096, 64),     # one query row against many keys, one shared key/value head
    (1, 4, 2, 300, 1000, 128),  # ragged on both sides, groups of two
    (1, 2, 1, 512, 128, 64),    # more queries than keys: causal rows 0..383 see nothing
    (1, 6, 3, 200, 200, 64),    # square, ragged, grouped
    (2, 2, 2, 77, 333, 128),    # causal offset not a multiple of the tile
    (1, 16, 1, 384, 384, 128),  # sixteen query heads share one key/value head
    (1, 4, 2, 130, 700, 32),    # d = 32: grouped, ragged, fewer queries than keys
    (1, 6, 3, 700, 130, 96),    # d = 96: grouped, ragged, more queries than keys
]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d", CASES)
def test_general_shapes_match_oracle(B, H, H_kv, N_q, N_k, d, causal):
    (q, k, v, do), (qg, kg, vg, dog) = _inputs(B, H, H_kv, N_q, N_k, d, 100 + N_q + N_k + H_kv)
    scale = 1.0 / math.sqrt(d)
    o, lse = binding.fwd_ex(qg, kg, vg, causal=causal, scale=scale)
    grads = {det: binding.bwd_ex(qg, kg, vg, o, lse, dog, causal=causal, scale=scale, deterministic=det)
             for det in (False, True)}
    assert_device_ok()
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.ref_fwd_general(qf, kf, vf, causal, scale)
    check_o(o, o_ref)
    _check_lse_general(lse, lse_ref)
    refs = oracle.ref_bwd_general(qf, kf, vf, dof, causal, scale)
    for det, gs in grads.items():
        for g, r, n in zip(gs, refs, ("dQ", "dK", "dV")):
            check_grad(g, r, n, "deterministic" if det else "reduce-add")


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("p", [0.1, 0.5])
@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d", [(1, 2, 1, 256, 384, 64), (1, 2, 2, 200, 200, 128),
                                             (1, 4, 2, 200, 333, 32), (1, 4, 2, 333, 200, 96)])
def test_dropout_matches_oracle(B, H, H_kv, N_q, N_k, d, p, causal):
    (q, k, v, do), (qg, kg, vg, dog) = _inputs(B, H, H_kv, N_q, N_k, d, 7)
    scale, seed, offset = 1.0 / math.sqrt(d), 0x1234_5678_9ABC, 17
    o, lse = binding.fwd_ex(qg, kg, vg, causal=causal, scale=scale, dropout_p=p, seed=seed, offset=offset)
    grads = {det: binding.bwd_ex(qg, kg, vg, o, lse, dog, causal=causal, scale=scale, dropout_p=p, seed=seed,
                                 offset=offset, deterministic=det) for det in (False, True)}
    assert_device_ok()
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    pf = float(np.float32(p))  # the library takes dropout_p as fp32
    o_ref, lse_ref = oracle.ref_fwd_general(qf, kf, vf, causal, scale, pf, seed, offset)
    # dropped weights are up to 1/(1-p) times larger, and so is the bf16 rounding of P;
    # the bf16 rounding of O itself comes on top where |O| >= 2
    err = np.abs(to_f64(o) - o_ref)
    assert (err <= o_max_abs_bound(o_ref, 1e-2 / (1 - p))).all() and err.mean() <= 1e-3 / (1 - p), \
        (err.max(), err.mean())
    _check_lse_general(lse, lse_ref)
    refs = oracle.ref_bwd_general(qf, kf, vf, dof, causal, scale, pf, seed, offset)
    for det, gs in grads.items():
        for g, r, n in zip(gs, refs, ("dQ", "dK", "dV")):
            check_grad(g, r, n, f"p={p} " + ("deterministic" if det else "reduce-add"))


def test_dropout_depends_on_seed_and_offset_only():
    _, (qg, kg, vg, _) = _inputs(1, 2, 2, 256, 256, 64, 8)
    a, _ = binding.fwd_ex(qg, kg, vg, dropout_p=0.3, seed=5, offset=0)
    b, _ = binding.fwd_ex(qg, kg, vg, dropout_p=0.3, seed=5, offset=0)
    c, _ = binding.fwd_ex(qg, kg, vg, dropout_p=0.3, seed=5, offset=1)
    d, _ = binding.fwd_ex(qg, kg, vg, dropout_p=0.3, seed=6, offset=0)
    assert_device_ok()
    assert torch.equal(a, b)
    assert not torch.equal(a, c) and not torch.equal(a, d)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_deterministic_backward_is_bit_identical(causal):
    _, (qg, kg, vg, dog) = _inputs(2, 4, 2, 640, 640, 128, 9)
    o, lse = binding.fwd_ex(qg, kg, vg, causal=causal)
    runs = [binding.bwd_ex(qg, kg, vg, o, lse, dog, causal=causal, deterministic=True) for _ in range(3)]
    assert_device_ok()
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a, b)


def test_square_general_call_equals_the_plain_entry_points():
    _, (qg, kg, vg, dog) = _inputs(1, 3, 3, 384, 384, 64, 10)
    o1, l1 = binding.fwd(qg, kg, vg, causal=True)
    o2, l2 = binding.fwd_ex(qg, kg, vg, causal=True)
    g1 = binding.bwd(qg, kg, vg, o1, l1, dog, causal=True)
    g2 = binding.bwd_ex(qg, kg, vg, o1, l1, dog, causal=True, deterministic=False)
    assert_device_ok()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])  # dK, dV: same kernel, fixed order


@pytest.mark.parametrize("p", [0.1, 0.5])
def test_dropout_tiny_workload(p):
    """The tiny workload (B=1, H=1, N=128, d=64, non-causal, seed 0) with dropout:
    forward and both backwards element by element against the oracle."""
    from exact_attention_108_b200.workloads import WORKLOADS
    w = WORKLOADS["tiny"]
    (q, k, v, do), (qg, kg, vg, dog) = gpu_inputs(w.B, w.H, w.N, w.d, w.seed, w.dist)
    seed, offset = 99, 5
    o, lse = binding.fwd_ex(qg, kg, vg, causal=w.causal, scale=w.scale, dropout_p=p, seed=seed, offset=offset)
    grads = {det: binding.bwd_ex(qg, kg, vg, o, lse, dog, causal=w.causal, scale=w.scale, dropout_p=p, seed=seed,
                                 offset=offset, deterministic=det) for det in (False, True)}
    assert_device_ok()
    pf = float(np.float32(p))
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    o_ref, lse_ref = oracle.ref_fwd_general(qf, kf, vf, w.causal, w.scale, pf, seed, offset)
    err = np.abs(to_f64(o) - o_ref)
    assert (err <= o_max_abs_bound(o_ref, 1e-2 / (1 - p))).all() and err.mean() <= 1e-3 / (1 - p)
    _check_lse_general(lse, lse_ref)
    refs = oracle.ref_bwd_general(qf, kf, vf, dof, w.causal, w.scale, pf, seed, offset)
    for det, gs in grads.items():
        for g, r, n in zip(gs, refs, ("dQ", "dK", "dV")):
            check_grad(g, r, n, f"tiny p={p}")


@pytest.mark.parametrize("p", [0.1, 0.5])
def test_dropout_training_shape_sampled_heads(p):
    """The training shape (B=4, H=32, N=4096, d=128, causal, seed 2) with dropout: O and
    LSE of sampled rows on every head, and whole labelled heads (fwd and bwd) against
    the oracle with the same Philox draws."""
    from exact_attention_108_b200.workloads import WORKLOADS
    w = WORKLOADS["train_d128_causal"]
    (q, k, v, do), (qg, kg, vg, dog) = gpu_inputs(w.B, w.H, w.N, w.d, w.seed, w.dist)
    seed, offset = 31337, 1
    o, lse = binding.fwd_ex(qg, kg, vg, causal=True, scale=w.scale, dropout_p=p, seed=seed, offset=offset)
    dq, dk, dv = binding.bwd_ex(qg, kg, vg, o, lse, dog, causal=True, scale=w.scale, dropout_p=p, seed=seed,
                                offset=offset)
    assert_device_ok()
    pf = float(np.float32(p))
    rng = np.random.default_rng(5)
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    for b in range(w.B):
        for h in range(w.H):
            rows = sorted({0, 1, 127, 128, w.N - 1} | set(rng.integers(0, w.N, 4).tolist()))
            o_r, l_r = oracle.ref_fwd_general_rows(qf, kf, vf, b, h, rows, True, w.scale, pf, seed, offset)
            err = np.abs(to_f64(o[b, h, rows]) - o_r)
            assert (err <= o_max_abs_bound(o_r, 1e-2 / (1 - p))).all(), (b, h, err.max())
            assert np.abs(lse[b, h, rows].double().cpu().numpy() - l_r).max() <= 1e-3
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1)]:
        # whole heads through ref_fwd_general_rows: a sliced [1, 1] call would renumber the
        # flattened head index b*H + h that the dropout draws depend on
        o_full, _ = oracle.ref_fwd_general_rows(qf, kf, vf, b, h, np.arange(w.N), True, w.scale, pf, seed, offset)
        err = np.abs(to_f64(o[b, h]) - o_full)
        assert (err <= o_max_abs_bound(o_full, 1e-2 / (1 - p))).all() and err.mean() <= 1e-3 / (1 - p)
        dq_r = oracle.ref_dq_general_rows(qf, kf, vf, dof, b, h, np.arange(w.N), True, w.scale, pf, seed, offset)
        check_grad(to_f64(dq[b, h]), dq_r, "dQ", f"train p={p} head ({b},{h})")


def test_graph_capture_of_the_general_forms_matches_eager_bitwise():
    """The grouped-head forward with dropout, the deterministic backward and split-KV
    decoding captured in one CUDA graph and replayed: every output bit-equal to the
    eager calls (all buffers, workspaces included, allocated before the capture)."""
    _, (qg, kg, vg, dog) = _inputs(2, 8, 2, 512, 700, 128, 11)
    kw = dict(causal=True, dropout_p=0.2, seed=7, offset=2)
    o_e, l_e = binding.fwd_ex(qg, kg, vg, **kw)
    g_e = binding.bwd_ex(qg, kg, vg, o_e, l_e, dog, deterministic=True, **kw)
    qd = qg[:, :, -2:].contiguous()
    od_e, ld_e = binding.decode(qd, kg, vg, causal=True, num_splits=3)
    assert_device_ok()
    o, l = torch.empty_like(o_e), torch.empty_like(l_e)
    dq, dk, dv = (torch.empty_like(t) for t in g_e)
    od, ld = torch.empty_like(od_e), torch.empty_like(ld_e)
    ws_b = torch.empty(64 << 20, device="cuda", dtype=torch.uint8)
    ws_d = torch.empty(16 << 20, device="cuda", dtype=torch.uint8)

    def step():
        binding.fwd_ex(qg, kg, vg, out=o, lse=l, **kw)
        binding.bwd_ex(qg, kg, vg, o, l, dog, deterministic=True, dq=dq, dk=dk, dv=dv, workspace=ws_b, **kw)
        binding.decode(qd, kg, vg, causal=True, num_splits=3, out=od, lse=ld, workspace=ws_d)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture
        step()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(2):
        for t in (o, l, dq, dk, dv, od, ld):
            t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_e) and torch.equal(l, l_e)
        assert torch.equal(dq, g_e[0]) and torch.equal(dk, g_e[1]) and torch.equal(dv, g_e[2])
        assert torch.equal(od, od_e) and torch.equal(ld, ld_e)
    del graph
    assert_device_ok()


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_negative_scale_grouped_dropout(causal):
    """A negative scale flips which key a row favours (the row max becomes a min of
    the raw scores); with grouped heads, a ragged bottom-right mask and dropout."""
    (q, k, v, do), (qg, kg, vg, dog) = _inputs(1, 4, 2, 200, 300, 64, 21)
    scale, p, seed, offset = -0.1, 0.2, 99, 5
    o, lse = binding.fwd_ex(qg, kg, vg, causal=causal, scale=scale, dropout_p=p, seed=seed, offset=offset)
    grads = {det: binding.bwd_ex(qg, kg, vg, o, lse, dog, causal=causal, scale=scale, dropout_p=p, seed=seed,
                                 offset=offset, deterministic=det) for det in (False, True)}
    assert_device_ok()
    qf, kf, vf, dof = (to_f64(t) for t in (q, k, v, do))
    pf = float(np.float32(p))
    o_ref, lse_ref = oracle.ref_fwd_general(qf, kf, vf, causal, np.float32(scale).item(), pf, seed, offset)
    err = np.abs(to_f64(o) - o_ref)
    assert (err <= o_max_abs_bound(o_ref, 1e-2 / (1 - p))).all() and err.mean() <= 1e-3 / (1 - p), \
        (err.max(), err.mean())
    _check_lse_general(lse, lse_ref)
    refs = oracle.ref_bwd_general(qf, kf, vf, dof, causal, np.float32(scale).item(), pf, seed, offset)
    for det, gs in grads.items():
        for g, r, n in zip(gs, refs, ("dQ", "dK", "dV")):
            check_grad(g, r, n, "negative scale " + ("deterministic" if det else "reduce-add"))
