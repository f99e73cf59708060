"""Full-size GPU parity on the five workloads, in the launch configuration bench.py
times (fattn_fwd then the three backward stages).

At full size the oracle runs on what it can compute one by one:
* whole (batch, head) slices (fwd + bwd) for two labelled heads per workload;
* sampled query rows of O, LSE and dQ on every head (each needs only its own row);
and properties that hold at any size check the rest on every head:
* Q = 0 gives uniform (prefix-mean) attention, exactly representable on the GPU;
* sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i per head.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_attention_108_b200 import binding
from exact_attention_108_b200.workloads import WORKLOADS, to_f64
from gpu_common import assert_device_ok, check_grad, check_lse, check_o, gpu_inputs, o_max_abs_bound

pytestmark = pytest.mark.gpu

ROWS_PER_HEAD = 6


def _run(w):
    cpu, (q, k, v, do) = gpu_inputs(w.B, w.H, w.N, w.d, w.seed, w.dist, with_do=w.backward)
    o, lse = binding.fwd(q, k, v, causal=w.causal, scale=w.scale)
    grads = None
    if w.backward:
        ws = torch.empty(binding.workspace_size(w.B, w.H, w.N, w.d), device=q.device, dtype=torch.uint8)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        binding.bwd_preprocess(o, lse, do, ws)
        binding.bwd_dkdv(q, k, v, do, dk, dv, ws, causal=w.causal, scale=w.scale)
        binding.bwd_dq(dq, ws, scale=w.scale)
        grads = (dq, dk, dv)
    assert_device_ok()
    return cpu, (q, k, v, do), o, lse, grads


def _sampled_rows(N, rng):
    rows = {0, 1, 127, 128, N - 1}
    rows.update(rng.integers(0, N, ROWS_PER_HEAD).tolist())
    return sorted(rows)


def _check_workload(w, full_heads):
    cpu, gpu, o, lse, grads = _run(w)
    q, k, v, do = cpu
    # labelled heads: everything.  Their reference maxima also give a lower bound
    # on the tensor-wide max|dQ| that the gradient tolerance is relative to.
    dq_max_ref = 0.0
    for (b, h) in full_heads:
        qh, kh, vh = (to_f64(t[b, h]) for t in (q, k, v))
        o_ref, lse_ref = oracle.ref_fwd(qh[None, None], kh[None, None], vh[None, None], w.causal, w.scale)
        check_o(to_f64(o[b, h]), o_ref[0, 0], f"{w.name} head ({b},{h})")
        check_lse(lse[b, h], lse_ref[0, 0], f"{w.name} head ({b},{h})")
        if grads is not None:
            doh = to_f64(do[b, h])
            refs = oracle.ref_bwd_head(qh, kh, vh, doh, w.causal, w.scale)
            dq_max_ref = max(dq_max_ref, float(np.abs(refs[0]).max()))
            for g, r, n in zip(grads, refs, ("dQ", "dK", "dV")):
                check_grad(to_f64(g[b, h]), r, n, f"{w.name} head ({b},{h})")
    rng = np.random.default_rng(w.seed)
    o_max, o_sum, o_cnt, lse_max, dq_rel = 0.0, 0.0, 0, 0.0, 0.0
    # every head: sampled rows of O, LSE (and dQ)
    for b in range(w.B):
        for h in range(w.H):
            rows = _sampled_rows(w.N, rng)
            qh, kh, vh = (to_f64(t[b, h]) for t in (q, k, v))
            o_r, l_r = oracle.ref_fwd_rows(qh, kh, vh, rows, w.causal, w.scale)
            emax, emean = check_o(to_f64(o[b, h, rows]), o_r, f"head ({b},{h}) rows", quiet=True)
            o_max, o_sum, o_cnt = max(o_max, emax), o_sum + emean * o_r.size, o_cnt + o_r.size
            lse_max = max(lse_max, check_lse(lse[b, h, rows], l_r, f"head ({b},{h}) rows", quiet=True))
            if grads is not None:
                doh = to_f64(do[b, h])
                dq_r = oracle.ref_dq_rows(qh, kh, vh, doh, rows, w.causal, w.scale)
                err = np.abs(to_f64(grads[0][b, h, rows]) - dq_r).max()
                bound = 2e-2 * max(dq_max_ref, float(np.abs(dq_r).max()))
                assert err <= bound, f"dQ rows head ({b},{h}): {err:.3e} > {bound:.3e}"
                dq_rel = max(dq_rel, err / bound * 2e-2)
    print(f"[parity] {w.name} sampled rows of all {w.B * w.H} heads: O max-abs {o_max:.3e} mean-abs "
          f"{o_sum / o_cnt:.3e}, LSE max-abs {lse_max:.3e}" +
          (f", dQ max-abs {dq_rel:.2e} of the max|ref| bound" if grads is not None else ""))
    # every head: column-sum invariants of the backward.  bf16 rounding of the
    # individual rows makes the sums inexact, so they are bounded relative to the
    # sum of magnitudes (a gross error -- a dropped term, a wrong mask -- breaks this).
    if grads is not None:
        dq, dk, dv = grads
        dkd, dvd, dod = dk.double(), dv.double(), gpu[3].double()
        rel_k = dkd.sum(dim=2).abs() / dkd.abs().sum(dim=2).clamp_min(1e-30)
        assert rel_k.max().item() <= 1e-2, f"sum_j dK_j != 0 (rel {rel_k.max().item():.2e})"
        rel_v = (dvd.sum(dim=2) - dod.sum(dim=2)).abs() / dvd.abs().sum(dim=2).clamp_min(1e-30)
        assert rel_v.max().item() <= 1e-2, f"sum_j dV_j != sum_i dO_i (rel {rel_v.max().item():.2e})"


def test_fwd_d64_full_size():
    _check_workload(WORKLOADS["fwd_d64"], [(0, 0), (7, 15)])


def test_fwd_d64_causal_full_size():
    _check_workload(WORKLOADS["fwd_d64_causal"], [(0, 0), (7, 15)])


def test_train_d128_causal_full_size():
    _check_workload(WORKLOADS["train_d128_causal"], [(0, 0), (3, 31)])


def test_peaked_n8192_full_size():
    _check_workload(WORKLOADS["peaked_n8192"], [(0, 0), (1, 15)])


@pytest.mark.slow
def test_long_n32768_causal_full_size():
    _check_workload(WORKLOADS["long_n32768_causal"], [(0, 0), (0, 7)])


@pytest.mark.parametrize("name", ["train_d128_causal", "long_n32768_causal", "fwd_d64"])
def test_zero_queries_closed_form_full_size(name):
    """Q = 0: every weight is exp(0) = 1, so O is the (prefix) mean of V and LSE
    = ln(count) on every head, at full size."""
    w = WORKLOADS[name]
    _, (q, k, v, _) = gpu_inputs(w.B, w.H, w.N, w.d, w.seed, w.dist, with_do=False)
    q.zero_()
    o, lse = binding.fwd(q, k, v, causal=w.causal, scale=w.scale)
    assert_device_ok()
    counts = torch.arange(1, w.N + 1, device=v.device, dtype=torch.float64) if w.causal else \
        torch.full((w.N,), float(w.N), device=v.device, dtype=torch.float64)
    vd = v.double()
    mean = (vd.cumsum(dim=2) if w.causal else vd.sum(dim=2, keepdim=True).expand_as(vd)) / counts[:, None]
    err = (o.double() - mean).abs()
    assert err.max().item() <= 1e-2 and err.mean().item() <= 1e-3
    assert (lse.double() - counts.log()).abs().max().item() <= 1e-3


@pytest.mark.parametrize("name", ["train_d128_causal", "peaked_n8192"])
def test_deterministic_backward_full_size(name):
    """The deterministic backward at full size: dK and dV are bit-equal to the default
    backward's (the same products in the same order, without the dQ product); dQ
    matches the oracle on sampled rows of every head and is the same on a second run."""
    w = WORKLOADS[name]
    cpu, (q, k, v, do) = gpu_inputs(w.B, w.H, w.N, w.d, w.seed, w.dist, with_do=True)
    o, lse = binding.fwd(q, k, v, causal=w.causal, scale=w.scale)
    ref = binding.bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.scale)
    det = binding.bwd_ex(q, k, v, o, lse, do, causal=w.causal, scale=w.scale, deterministic=True)
    det2 = binding.bwd_ex(q, k, v, o, lse, do, causal=w.causal, scale=w.scale, deterministic=True)
    assert_device_ok()
    assert torch.equal(det[1], ref[1]) and torch.equal(det[2], ref[2])
    assert torch.equal(det[0], det2[0])
    qc, kc, vc, doc = cpu
    rng = np.random.default_rng(w.seed + 100)
    worst = 0.0
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 2)]:
        rows = _sampled_rows(w.N, rng)
        qh, kh, vh, doh = (to_f64(t[b, h]) for t in (qc, kc, vc, doc))
        dq_r = oracle.ref_dq_rows(qh, kh, vh, doh, rows, w.causal, w.scale)
        err = np.abs(to_f64(det[0][b, h, rows]) - dq_r).max()
        worst = max(worst, err / np.abs(dq_r).max())
        assert err <= 2e-2 * np.abs(dq_r).max(), f"dQ rows head ({b},{h}): {err:.3e}"
    print(f"[parity] {name} deterministic dQ sampled rows: max-abs {worst:.2e} of the rows' max|ref|")


def test_grouped_heads_dropout_training_shape():
    """B=4, H=32 query heads over H_kv=8 key/value heads, N=4096, d=128, causal, dropout
    0.1: O and LSE on sampled rows of every query head, dQ on sampled rows of labelled
    heads, against the oracle's general form with the same Philox draws."""
    B, H, H_kv, N, d, p, seed, offset = 4, 32, 8, 4096, 128, 0.1, 2024, 3
    g = torch.Generator("cpu").manual_seed(12)
    qc = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
    kc = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16)
    vc = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16)
    doc = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
    q, k, v, do = (t.cuda() for t in (qc, kc, vc, doc))
    scale = 1.0 / np.sqrt(d)
    o, lse = binding.fwd_ex(q, k, v, causal=True, scale=scale, dropout_p=p, seed=seed, offset=offset)
    dq, dk, dv = binding.bwd_ex(q, k, v, o, lse, do, causal=True, scale=scale, dropout_p=p, seed=seed,
                                offset=offset)
    assert_device_ok()
    pf = float(np.float32(p))
    qd, kd, vd, dod = (to_f64(t) for t in (qc, kc, vc, doc))
    rng = np.random.default_rng(13)
    o_max = 0.0
    for b in range(B):
        for h in range(H):
            rows = _sampled_rows(N, rng)
            o_r, l_r = oracle.ref_fwd_general_rows(qd, kd, vd, b, h, rows, True, scale, pf, seed, offset)
            err = np.abs(to_f64(o[b, h, rows]) - o_r)
            o_max = max(o_max, float(err.max()))
            # 1e-2 / (1 - p) (kept weights, and their bf16 rounding, grow by 1 / (1 - p)) plus
            # the bf16 rounding of O itself where |O| >= 2:
            # the first causal rows average few, rescaled values and reach |O| of 2 to 8
            excess = err - o_max_abs_bound(o_r, 1e-2 / (1 - p))
            assert excess.max() <= 0, f"O rows head ({b},{h}): {err.max():.3e} (over by {excess.max():.3e})"
            check_lse(lse[b, h, rows], l_r, f"head ({b},{h}) rows", quiet=True)
            if (b, h) in ((0, 0), (B - 1, H - 1)):
                dq_r = oracle.ref_dq_general_rows(qd, kd, vd, dod, b, h, rows, True, scale, pf, seed, offset)
                e = np.abs(to_f64(dq[b, h, rows]) - dq_r).max()
                assert e <= 2e-2 * np.abs(dq_r).max(), f"dQ rows head ({b},{h}): {e:.3e}"
    print(f"[parity] grouped heads + dropout, training shape: O sampled rows max-abs {o_max:.3e}")
