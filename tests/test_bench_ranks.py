"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the
device time is taken as the maximum over ranks, every rank sees the same
value, the whole-job rate counts all ranks' units, and the reference arm does
its work on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * rank                   # rank 1 is the slower one
        slowest = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        rate = bench.whole_job_rate(world, 1000, 4, slowest)
        dist.barrier()
        out.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[0] for g in got] == [0, 1]
    for _, slowest, rate in got:
        assert slowest == 15.0                     # max over ranks, on every rank
        assert rate == pytest.approx(2 * 1000 * 4 / 0.015)


def test_single_process_aggregation_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.whole_job_rate(1, 100, 10, 1000.0) == pytest.approx(1000.0)


def test_reference_arm_other_ranks_do_no_work(capsys):
    sys.path.insert(0, ROOT)
    import bench
    bench.run_reference(None, 1, 2)                # args unused on rank != 0: returns at once
    assert capsys.readouterr().out == ""


def test_oracle_baseline_of_a_secondary_line():
    """The oracle leg beside a secondary bench line runs on the host alone and
    returns a positive rate with its unit, core count and sample."""
    import bench
    out = bench.oracle_extra_baselines({"tiny_d128_t1024"})
    b = out["tiny_d128_t1024"]
    assert b["kind"] == "oracle" and b["value"] > 0 and b["cores"] >= 1
    assert b["unit"] == "decode us" and "1024 keys" in b["sample"]


def test_reference_arm_json_line_contract():
    """`bench.py --impl reference` (the oracle on host cores, no GPU) prints
    one JSON line with the contract's keys: the headline metric on the same
    workload, impl "reference", a cpu_baseline describing the run and an e2e
    object with no host-device copies."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    run = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=root)
    assert run.returncode == 0, run.stderr[-2000:]
    lines = [ln for ln in run.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "llama31_8b_gqa_decode"
    assert d["value"] > 0 and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
