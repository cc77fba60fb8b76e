"""Host logic of bench.py, on CPU: the paths for more than one rank (gloo
backend) and the clock record.

The GPU runs of this build have one GPU, so the N > 1 paths of the benchmark
(max-over-ranks timing, barriers, the whole-job rate, the reference arm's
non-zero ranks) are exercised here by two real processes.
"""
import datetime
import os
import socket
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, local_ms, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench as b
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, lr, w = b.env_rank()
        b.barrier(world)
        m = b.max_over_ranks(local_ms[rank], world)
        rate = b.aggregate_rate(world, 32, 100, m)
        b.barrier(world)
        q.put((rank, r, lr, w, m, rate))
    finally:
        dist.destroy_process_group()


def _run_ranks(world, local_ms):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_max_over_ranks_two_gloo_ranks():
    out = _run_ranks(2, [3.25, 5.5])
    for rank, r, lr, w, m, rate in out:
        assert (r, lr, w) == (rank, rank, 2)
        assert m == 5.5                       # the slowest rank's time, on every rank
        assert rate == pytest.approx(2 * 32 * 100 / 5.5e-3)


def test_max_over_ranks_slow_rank_zero():
    out = _run_ranks(2, [9.0, 1.0])
    assert [o[4] for o in out] == [9.0, 9.0]


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.0, 1) == 7.0
    bench.barrier(1)
    assert bench.aggregate_rate(1, 8, 10, 2.0) == pytest.approx(8 * 10 / 2e-3)


def test_reference_arm_other_ranks_exit_quietly(monkeypatch, capsys):
    # under torchrun every rank but 0 returns 0 at once and prints nothing
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")

    class Args:
        steps, warmup, gpus = 3, 3, 2
    assert bench.reference_arm(Args()) == 0
    assert capsys.readouterr().out == ""


def test_recorded_traffic_follows_the_source_digest(tmp_path, monkeypatch):
    """bench.py reports DRAM traffic only for the kernel sources it was measured on."""
    csrc = tmp_path / "covariance_corrected_softmax_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "a.cu").write_text("kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d1 = bench.source_digest(["a.cu"])
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# header\nk1  w1  12345  %s  capture\n" % d1)
    assert bench.recorded_traffic("k1", "w1", ["a.cu"]) == 12345.0
    assert bench.recorded_traffic("k1", "other", ["a.cu"]) is None
    (csrc / "a.cu").write_text("kernel v2\n")  # the kernel changed since the capture
    assert bench.recorded_traffic("k1", "w1", ["a.cu"]) is None


def test_clock_summary_keeps_the_timed_window():
    """The clock record is the median of the samples taken inside the timed
    region: pre-roll and tail samples at idle clocks are left out."""
    clk = bench.ClockSampler(0)
    t0 = datetime.datetime(2026, 1, 2, 3, 4, 5).timestamp()

    def row(dt, mhz, power, cap):
        stamp = datetime.datetime.fromtimestamp(t0 + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return (f"{stamp}, 0, {mhz}, 1965, {power}, 0x0, Not Active, Not Active, Not Active, "
                f"{'Active' if cap else 'Not Active'}\n")

    fd, clk.path = tempfile.mkstemp(suffix=".csv")
    with os.fdopen(fd, "w") as f:
        for k in range(15):  # pre-roll at idle
            f.write(row(-0.3 + 0.02 * k, 1965, 100.0, False))
        for k in range(5):  # the timed region, under the power cap
            f.write(row(0.005 + 0.02 * k, 1700 + k, 900.0, True))
        f.write(row(0.3, 1965, 120.0, False))  # tail
    clk.t0, clk.t1 = t0, t0 + 0.1
    s = clk.summary()
    assert s["samples"] == 5 and s["sm_mhz"] == 1702.0
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 900.0
    assert s["sm_max_mhz"] == 1965.0 and s["window_ms"] == 100.0
