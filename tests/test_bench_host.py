"""Host-side logic of bench.py on the CPU: the multi-rank reduction (world size 2
over gloo), the whole-job throughput formula, the clock-record parser and the
traffic record's staleness check."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_rank_ms = [4.0, 5.5][rank]
        m = bench.max_over_ranks(per_rank_ms, world)
        out[rank] = (m, bench.whole_job_tflops(world, 1e12, m), bench.rank_seed(2, rank))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_world2_gloo():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 5.5
    assert res[0][1] == pytest.approx(2 * 1e12 / 5.5e-3 / 1e12)
    assert {res[0][2], res[1][2]} == {2, 3}


def test_whole_job_tflops_single():
    assert bench.whole_job_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
    assert bench.max_over_ranks(3.0, 1) == 3.0


def test_clock_parser():
    cs = bench.ClockSampler("0")
    cs.proc = None
    cs.lines = ["1965, 1965, 700.1, Not Active, Not Active, Not Active, Not Active",
                "1800, 1965, 990.0, Not Active, Not Active, Not Active, Active",
                "1890, 1965, 995.0, Not Active, Not Active, Not Active, Active"]

    class _P:
        def terminate(self): pass
        def wait(self, timeout=None): return 0
    cs.proc = _P()
    rec = cs.stop()
    assert rec["sm_mhz"] == 1890 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]


def test_traffic_record_goes_null_when_sources_change(tmp_path, monkeypatch):
    import hashlib
    src = tmp_path / "k.cuh"
    src.write_text("kernel v1")
    prof = tmp_path / "profiles"
    prof.mkdir()
    sha = hashlib.sha256(b"kernel v1").hexdigest()
    (prof / "traffic.json").write_text(json.dumps({
        "sources": ["k.cuh"],
        "kernels": {"kern": {"wl": {"sources_sha256": sha, "dram_bytes_per_launch": 123.0}}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.dominant_kernel_traffic("kern", "wl") == 123.0
    src.write_text("kernel v2")
    assert bench.dominant_kernel_traffic("kern", "wl") is None
