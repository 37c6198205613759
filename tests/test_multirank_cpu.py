"""The multi-GPU host logic of bench.py on CPU: two `gloo` ranks (processes,
127.0.0.1) agree on the slowest rank's time and on the whole-job throughput;
the reference arm runs on rank 0 only.  (Replicas: the decode path has no
data-path collective.)"""
import argparse
import datetime
import importlib.util
import json
import multiprocessing as mp
import os
import socket

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rank_worker(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench = _load_bench()
        ms = bench.max_over_ranks(times[rank], dist, "cpu")
        value = bench.whole_job_tokens_per_s(world, 64, 10, ms)
        dist.barrier()
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [3.0, 5.0]
    port = _free_port()
    procs = [ctx.Process(target=_rank_worker, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in procs)
    for rank, ms, value in got:
        assert ms == 5.0                       # max over ranks, on every rank
        assert value == 2 * 64 * 10 / 5e-3     # all ranks' tokens over the slowest time


def test_single_rank_keeps_its_time():
    bench = _load_bench()
    assert bench.max_over_ranks(4.5, None, "cpu") == 4.5
    assert bench.whole_job_tokens_per_s(1, 1, 200, 10.0) == 20000.0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    bench = _load_bench()
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(steps=1, warmup=0, gpus=2)
    cfg = bench.WL.TINY_F32
    assert bench.run_reference(args, cfg) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_contract_line(monkeypatch, capsys):
    """Rank 0 of the reference arm times the oracle and prints the bench
    contract's JSON line, with its CPU baseline and a zero-copy e2e."""
    bench = _load_bench()
    monkeypatch.setenv("RANK", "0")
    args = argparse.Namespace(steps=1, warmup=1, gpus=1)
    cfg = bench.WL.TINY_F32
    bench.run_reference(args, cfg)
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == cfg.name
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
