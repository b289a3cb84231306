"""The multi-rank host logic of bench.py, run as two gloo ranks on the CPU.

On GPUs bench.py runs one replica of the MoE layer per GPU (tokens are independent, so the layer
shards by token batches with no exchange); the only cross-rank steps are the barriers around the
timed region and the max of the ranks' device times. These tests run exactly those steps with
world size 2 over gloo, plus the reference arm's rule that only rank 0 does work under torchrun.
"""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    try:
        w, r, _ = bench.dist_setup("gloo")
        bench.barrier(w)
        local_ms = 10.0 + 5.0 * r          # rank 1 is the slow one
        ms_max = bench.max_over_ranks(local_ms, w)
        value = bench.whole_job_throughput(4, 100, w, ms_max)
        bench.barrier(w)
        # the reference arm: ranks other than 0 return without work and print nothing
        buf = io.StringIO()
        ref = None
        if r != 0:
            with contextlib.redirect_stdout(buf):
                ref = bench.run_reference(type("A", (), dict(workload="decode1", steps=1, warmup=1))(), w, r)
        q.put((r, w, ms_max, value, ref, buf.getvalue()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_tokens():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=5) for _ in range(world))
    for (r, w, ms_max, value, ref, out) in res:
        assert w == 2
        assert ms_max == 15.0                                  # max over ranks, seen by every rank
        assert value == pytest.approx(4 * 100 * 2 / 0.015)     # all ranks' tokens / slowest time
        if r == 1:
            assert ref is None and out == ""


def test_single_process_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_throughput(1, 1000, 1, 500.0) == pytest.approx(2000.0)


def test_replicas_draw_distinct_tokens():
    sys.path.insert(0, ROOT)
    import bench
    import synth
    streams = {bench.replica_x_stream(r, i) for r in range(8) for i in range(64)}
    assert len(streams) == 8 * 64
    a = synth.make_x(0, 1, 256, stream=bench.replica_x_stream(0, 0))
    b = synth.make_x(0, 1, 256, stream=bench.replica_x_stream(1, 0))
    assert not torch.equal(a, b)


def test_traffic_figure_follows_source_hash_and_launch_shape(tmp_path, monkeypatch):
    # a committed DRAM-traffic figure is reported only for the launch shape it was captured on
    # and only while the captured kernel source is unchanged
    sys.path.insert(0, ROOT)
    import hashlib
    import bench
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC", {("k", ("shape_a",)): (["k.cu"], sha, 1234)})
    assert bench.traffic_for("k", "shape_a") == 1234
    assert bench.traffic_for("k", "shape_b") is None      # another launch shape
    assert bench.traffic_for("other", "shape_a") is None  # no capture of that kernel
    src.write_text("kernel v2\n")
    assert bench.traffic_for("k", "shape_a") is None      # the source changed since the capture
    (tmp_path / "k.cu").unlink()
    assert bench.traffic_for("k", "shape_a") is None      # source missing
