"""Multi-rank host logic of bench.py on CPU: two gloo ranks, max-over-ranks timing and the
whole-job throughput (replicas, no data exchange)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        per_rank_ms = [12.5, 20.0][rank]
        e2e_ms = [30.0, 25.0][rank]
        mx = bench.max_over_ranks([per_rank_ms, e2e_ms])
        thr = bench.aggregate_throughput(32, 10, world, mx[0])
        q.put((rank, mx, thr))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, thr in res:
        assert mx == [20.0, 30.0], "every rank sees the slowest rank's times"
        assert thr == pytest.approx(2 * 32 * 10 / 0.020)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.aggregate_throughput(32, 4, 1, 8.0) == pytest.approx(16000.0)


def test_clock_record_counts_only_loaded_samples():
    """The clock summary takes the median over the load window and the timed steps, ignores
    samples taken before the load started, and reports every throttle reason seen under load."""
    import bench
    c = bench.ClockSampler(0)
    c.source, c.sm_max = "test", 1965.0
    c.samples = [(0.0, 345.0, set()), (1.0, 1965.0, set()), (1.1, 1900.0, {"sw_power_cap"}),
                 (1.2, 1965.0, set()), (1.3, 1950.0, set()), (9.0, 300.0, {"hw_slowdown"})]
    c.marks = {"load": 0.5, "timed0": 1.15, "timed1": 1.35}
    r = c.stop()
    assert r["samples"] == 4 and r["samples_timed"] == 2
    assert r["sm_mhz"] == pytest.approx(1957.5)
    assert r["reasons"] == ["sw_power_cap"]
    assert r["sm_max_mhz"] == 1965.0
