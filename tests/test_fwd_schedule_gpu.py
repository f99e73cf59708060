"""The persistent forward's work distribution.

One CTA per SM loops over units of two query tiles; causal launches claim units
from a device counter (one of a small pool of counter slots; with every slot
busy a launch reuses the least recently handed-out one behind a stream wait on
its event), while launches under CUDA-graph capture take units round-robin.
Which CTA computes a unit does not change its arithmetic, so every schedule
must give bit-identical O and LSE; the oracle pins one of them.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_attention_108_b200 import binding
from exact_attention_108_b200.workloads import to_f64
from gpu_common import assert_device_ok, check_lse, check_o, gpu_inputs

pytestmark = pytest.mark.gpu


# 160 heads, so every CTA runs several units; odd tile counts (3, 5) give units
# with a single query tile.
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(384, 64), (384, 128), (640, 128)])
def test_many_units_per_cta_match_oracle(N, d, causal):
    B, H = 2, 80
    (q, k, v, _), (qg, kg, vg, _) = gpu_inputs(B, H, N, d, 31 + N + d, with_do=False)
    scale = 1.0 / np.sqrt(d)
    o, lse = binding.fwd(qg, kg, vg, causal=causal, scale=scale)
    assert_device_ok()
    heads = [(b, h) for b in range(B) for h in range(H)][:: (1 if N <= 384 else 7)]
    for (b, h) in heads:
        qh, kh, vh = (to_f64(t[b, h])[None, None] for t in (q, k, v))
        o_ref, lse_ref = oracle.ref_fwd(qh, kh, vh, causal, scale)
        check_o(to_f64(o[b, h]), o_ref[0, 0], f"head ({b},{h})")
        check_lse(lse[b, h], lse_ref[0, 0], f"head ({b},{h})")


def test_graph_capture_matches_eager_bitwise():
    """A captured causal forward schedules statically; an eager one claims units
    dynamically.  Both must give the same bits."""
    _, (qg, kg, vg, _) = gpu_inputs(4, 16, 1024, 128, 41, with_do=False)
    o_e, l_e = binding.fwd(qg, kg, vg, causal=True)
    assert_device_ok()
    o_g = torch.empty_like(o_e)
    l_g = torch.empty_like(l_e)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture
        binding.fwd(qg, kg, vg, causal=True, out=o_g, lse=l_g)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        binding.fwd(qg, kg, vg, causal=True, out=o_g, lse=l_g)
    for _ in range(3):
        o_g.zero_()
        l_g.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o_g, o_e) and torch.equal(l_g, l_e)
    del g
    assert_device_ok()


def test_concurrent_streams_reuse_counter_slots_bitwise():
    """More causal launches than counter slots, spread over three streams with no
    synchronisation between them: each output must equal its sequential run."""
    inputs = [gpu_inputs(4, 16, 1024, 64, 50 + i, with_do=False)[1][:3] for i in range(6)]
    ref = []
    for (q, k, v) in inputs:
        ref.append(binding.fwd(q, k, v, causal=True))
    assert_device_ok()
    streams = [torch.cuda.Stream() for _ in range(3)]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    outs = []
    for rep in range(4):  # 24 launches
        for i, (q, k, v) in enumerate(inputs):
            s = streams[(i + rep) % 3]
            with torch.cuda.stream(s):
                o = torch.empty_like(q)
                lse = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)
                binding.fwd(q, k, v, causal=True, out=o, lse=lse, stream=s)
            outs.append((i, o, lse, s))
    torch.cuda.synchronize()
    assert_device_ok()
    for (i, o, lse, s) in outs:
        o.record_stream(s)
        assert torch.equal(o, ref[i][0]) and torch.equal(lse, ref[i][1]), f"launch of input {i} differs"


def test_launches_queued_ahead_of_the_gpu_bitwise():
    """Forty causal launches on one stream queued behind a long sleep, so that the
    host runs ahead and every counter slot is still busy when most of them are
    issued: each must reuse a slot behind its event and match its sequential run."""
    inputs = [gpu_inputs(2, 16, 768, 128, 70 + i, with_do=False)[1][:3] for i in range(5)]
    ref = [binding.fwd(q, k, v, causal=True) for (q, k, v) in inputs]
    torch.cuda.synchronize()
    assert_device_ok()
    outs = []
    torch.cuda._sleep(200_000_000)  # about 0.1 s of GPU time ahead of the launches
    for rep in range(8):
        for i, (q, k, v) in enumerate(inputs):
            o = torch.empty_like(q)
            lse = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)
            binding.fwd(q, k, v, causal=True, out=o, lse=lse)
            outs.append((i, o, lse))
    torch.cuda.synchronize()
    assert_device_ok()
    for (i, o, lse) in outs:
        assert torch.equal(o, ref[i][0]) and torch.equal(lse, ref[i][1]), f"launch of input {i} differs"
