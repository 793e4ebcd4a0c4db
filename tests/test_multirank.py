"""Host-side logic of the multi-rank benchmark, run as two gloo ranks on CPU.

Every rank runs its own replica of the workload (the path shards by head and
has no data exchange); the only collective is the timing reduction, whose
maximum over ranks sets the whole-job throughput.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (world, rank, rank)
        local_ms = [100.0, 125.0][rank]
        t_max = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        value = bench.weak_scaling_tflops(world, 5.0e12, 10, t_max)
        out[rank] = (t_max, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        t_max, value = out[rank]
        assert t_max == 125.0
        assert value == pytest.approx(2 * 5.0e12 * 10 / 0.125 / 1e12)


def test_single_rank_helpers_without_process_group():
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.weak_scaling_tflops(1, 1e12, 1, 1000.0) == pytest.approx(1.0)


def test_reference_arm_other_ranks_do_nothing(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(bench, "oracle_inputs", lambda w: (_ for _ in ()).throw(AssertionError("rank 1 worked")))

    class A:
        steps, warmup, heads, workload = 3, 3, None, "wan480_25"

    bench.main_reference(A())
    assert capsys.readouterr().out == ""


def _gather_worker(rank, world, port, out):
    from block_sparse_attention_cross_b200.sharded import gather_in_order
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r holds inputs with ids; rank 0 two, rank 1 one, rank 2 three
        counts = [2, 1, 3][:world]
        first = sum(counts[:rank])
        local = [torch.full((2, 3, 4), float(first + i)) + torch.arange(24.0).view(2, 3, 4) * 1e-3
                 for i in range(counts[rank])]
        got = gather_in_order(local)
        out[rank] = [float(t[0, 0, 0]) for t in got] + [tuple(got[0].shape)]
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_calibration_gathers_inputs_in_global_order_gloo(world):
    # The cross-rank step of calibration sharded by input: every rank must see
    # every input's energies in global input order (rank-major), whatever the
    # per-rank counts, so that selection, votes and the float32 energy sums
    # replay the single-GPU order exactly.
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_gather_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    n = sum([2, 1, 3][:world])
    for rank in range(world):
        assert out[rank][:-1] == [float(i) for i in range(n)]
        assert out[rank][-1] == (2, 3, 4)


def test_bench_workload_helpers():
    # FLOPs per kept block follow the block shape; the _k64 workload is the
    # 480p call with 64-key blocks.
    assert bench.kept_flops(1, 128, 1) == 4.0 * 128 * 128 * 128
    assert bench.kept_flops(2, 128, 1, block_k=64) == bench.kept_flops(1, 128, 1)
    assert bench.key_block("wan480_25_k64") == 64 and bench.key_block("wan480_25") == 128
    w = bench.workload(None, "wan480_25_k64")
    assert (w.name, w.N, w.H) == ("wan480_25", 32760, 40)
    assert bench.workload(8, "sweep").H == 8


def test_linear_fit():
    # an exact line: slope, intercept and R^2 = 1 recovered
    x = [1.0, 0.8, 0.6, 0.4, 0.25, 0.2, 0.1]
    sl, ic, r2 = bench.linear_fit(x, [21.5 * d - 0.1 for d in x])
    assert sl == pytest.approx(21.5) and ic == pytest.approx(-0.1) and r2 == pytest.approx(1.0)
    # a hand case: y = 1, 0, 3, 2 at x = 0 .. 3 -> slope 0.6, intercept 0.6, residual sum 3.2 of a
    # total 5, R^2 = 0.36
    sl, ic, r2 = bench.linear_fit([0, 1, 2, 3], [1, 0, 3, 2])
    assert sl == pytest.approx(0.6) and ic == pytest.approx(0.6) and r2 == pytest.approx(0.36)
    # constant y: the line is flat and fits exactly
    assert bench.linear_fit([0.1, 0.2, 0.3], [2.0, 2.0, 2.0]) == pytest.approx((0.0, 2.0, 1.0))


def _replica_probe(path):
    # one replica of the harness on CPU: the torchrun-style environment set by
    # launch_replicas, a gloo group, the max-over-ranks timing and the line
    import json
    world, rank, local = bench.dist_env()
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t_max = bench.max_over_ranks([100.0, 125.0][rank], dist, torch.device("cpu"))
        line = bench.contract_line(world, 10, 3, t_max, 5.0e12, {"workload": "probe"})
        with open(f"{path}.{rank}", "w") as f:
            f.write(json.dumps({"line": line, "local": local, "addr": os.environ["MASTER_ADDR"]}))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gpus_2_launches_two_replica_ranks_gloo(tmp_path):
    import json
    codes = bench.launch_replicas(2, _replica_probe, (str(tmp_path / "out"),))
    assert codes == [0, 0]
    for rank in range(2):
        rec = json.loads((tmp_path / f"out.{rank}").read_text())
        line = rec["line"]
        assert rec["local"] == rank and rec["addr"] == "127.0.0.1"
        assert line["n_gpus"] == 2 and line["scaling"] == "weak" and line["steps"] == 10
        assert line["ms_per_step"] == 12.5                         # the slower rank's 125 ms over 10 steps
        assert line["value"] == pytest.approx(2 * 5.0e12 * 10 / 0.125 / 1e12, rel=1e-3)
        assert line["config"]["parallelism"].startswith("replicas x2")


def test_main_spawns_replicas_without_a_launcher(monkeypatch):
    calls = []
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench, "launch_replicas", lambda n, target, args=(): calls.append((n, target, args)) or [0] * n)
    monkeypatch.setattr(bench.sys, "argv", ["bench.py", "--gpus", "2", "--steps", "4"])
    bench.main()
    assert calls and calls[0][0] == 2 and calls[0][1] is bench._replica_main
    assert calls[0][2] == (["--gpus", "2", "--steps", "4"],)


def test_main_refuses_a_world_size_other_than_gpus(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(bench.sys, "argv", ["bench.py", "--gpus", "4"])
    with pytest.raises(SystemExit, match="WORLD_SIZE=2"):
        bench.main()


def test_clock_sampler_keeps_the_timed_window(tmp_path):
    # nvidia-smi rows (timestamped) before, inside and after the timed region:
    # only the rows inside it count; a region shorter than the sampling period
    # falls back to the samples nearest to it.
    from datetime import datetime

    def fake_rows(cs, now, offsets, clocks, cap):
        lines = []
        for dt, mhz in zip(offsets, clocks):
            ts = datetime.fromtimestamp(now + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
            lines.append(f"{ts}, 0, {mhz}, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, {cap}")
        cs.path.write_text("\n".join(lines) + "\n")

    class Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            pass

    now = 1_800_000_000.0
    cs = bench.ClockSampler(0)
    cs.path = tmp_path / "clocks.csv"
    fake_rows(cs, now, (-1.0, 0.02, 0.04, 1.0), (1200, 1800, 1810, 1300), "Active")
    cs.proc, cs.fh = Proc(), open(os.devnull, "w")
    cs.mark_window(now, now + 0.05)
    rec = cs.stop()
    assert rec["samples"] == 2 and rec["sm_mhz"] == 1805.0 and rec["reasons"] == ["sw_power_cap"]

    cs = bench.ClockSampler(0)
    cs.path = tmp_path / "clocks2.csv"
    fake_rows(cs, now, (-0.2, -0.03, 0.5), (1500, 1900, 1600), "Not Active")
    cs.proc, cs.fh = Proc(), open(os.devnull, "w")
    cs.mark_window(now, now + 0.01)
    rec = cs.stop()
    assert rec["samples"] == 2 and rec["sm_mhz"] == 1700.0 and rec["reasons"] == []
