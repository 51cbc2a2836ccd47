"""Host-side logic of bench.py: argument handling, the max/sum over ranks used for
multi-GPU timing (gloo, world size 2, on CPU), the reference arm's JSON line on
a small workload, and the committed-traffic lookup."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    w, r, l = bench.dist_env()
    assert (w, r, l) == (world, rank, rank)
    dist = bench.init_group(world, "gloo")
    dev = torch.device("cpu")
    # rank r "took" 1 + r seconds and processed 10 * (r + 1) bytes
    t = bench.max_over_ranks(1.0 + rank, dist, dev)
    b = bench.sum_over_ranks(10.0 * (rank + 1), dist, dev)
    bench.barrier(dist, dev)
    q.put((rank, t, b))
    dist.destroy_process_group()


def test_max_and_sum_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, b in got:
        assert t == 2.0  # the slowest rank's time
        assert b == 30.0  # bytes of all ranks


def _reps_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist = bench.init_group(world, "gloo")
    dev = torch.device("cpu")
    calls = [0]

    def run():  # rank 1 is twice as slow, and its first (untimed) region looks very long
        calls[0] += 1
        return (5.0 if calls[0] == 1 and rank == 1 else 0.01 * (rank + 1))

    times = bench.timed_reps(run, dist, dev, min_seconds=0.05)
    q.put((rank, times))
    dist.destroy_process_group()


def test_timed_repetitions_agree_over_two_gloo_ranks():
    """Every rank runs the same number of repetitions (the most any rank asked for) and each
    repetition's time is the max over ranks."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_reps_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got[0] == got[1]
    assert len(got[0]) == 5  # rank 0: 0.05 s / 0.01 s per region
    assert all(t == 0.02 for t in got[0])


def test_timing_summary():
    s = bench.timing_summary([0.004, 0.002, 0.003], 20)
    assert s["reps"] == 3 and s["steps_per_rep"] == 20
    assert abs(s["median_us_per_call"] - 150.0) < 1e-9
    assert abs(s["min_us_per_call"] - 100.0) < 1e-9 and abs(s["max_us_per_call"] - 200.0) < 1e-9


def test_single_process_reductions_are_identity():
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    assert bench.sum_over_ranks(7.0, None, torch.device("cpu")) == 7.0


def test_args_defaults_and_warmup_floor():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.workload == "llama8b" and a.steps == bench.DEFAULT_STEPS["llama8b"]
    assert a.warmup >= 3 and a.impl == "ours"
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])


def test_instances_differ_per_rank_and_instance():
    a0, a1 = bench.make_instances("tiny", 0, 2)
    b0, = bench.make_instances("tiny", 1, 1)
    assert not torch.equal(a0.q, a1.q) and not torch.equal(a0.q, b0.q)
    assert a0.q.shape == b0.q.shape and a0.algorithmic_bytes() == b0.algorithmic_bytes()
    r0, r1 = bench.make_instances("ragged", 0, 2)
    assert torch.equal(r0.seq_lens, r1.seq_lens) and torch.equal(r0.page_table, r1.page_table)
    assert r0.algorithmic_bytes() == r1.algorithmic_bytes() and not torch.equal(r0.q, r1.q)


def test_every_named_workload_has_a_bench_seed_and_a_parser_choice():
    # make_instances looks the workload's seed up before generating anything
    for name in bench.workloads.NAMED:
        assert bench.make_instances(name, 0, 0) == []
        assert bench.parse_args(["--workload", name]).workload == name


def test_committed_traffic_records_are_well_formed():
    # one record per decode workload, each naming its kernel and command, with read + write
    # bytes that add up; a stale record (older device code) is reported as null by the bench
    with open(bench.TRAFFIC_FILE) as f:
        recs = json.load(f)
    names = [r["workload"] for r in recs]
    assert len(names) == len(set(names)) and set(names) <= set(bench.workloads.NAMED)
    for r in recs:
        assert r["dram_bytes_per_launch"] == r["dram_bytes_read"] + r["dram_bytes_write"]
        assert r["command"].startswith("ncu ") and "--clock-control none" in r["command"]
        assert r["kernel"].startswith("apd::") and len(r["kernel_source_sha"]) == 16


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "4", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "tiny_b1_h4x1_d64_l256"


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "3", "--warmup", "3", "--gpus", "2"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_traffic_lookup_is_tied_to_the_kernel_source(tmp_path, monkeypatch):
    f = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.committed_traffic("llama8b") is None
    f.write_text(json.dumps({"kernel_source_sha": bench.kernel_source_sha(), "workload": "llama8b",
                             "dram_bytes_per_launch": 123}))
    assert bench.committed_traffic("llama8b") == 123
    assert bench.committed_traffic("long") is None
    f.write_text(json.dumps({"kernel_source_sha": "0" * 16, "workload": "llama8b", "dram_bytes_per_launch": 123}))
    assert bench.committed_traffic("llama8b") is None
    # one record per workload in a list
    sha = bench.kernel_source_sha()
    f.write_text(json.dumps([{"kernel_source_sha": sha, "workload": "llama8b", "dram_bytes_per_launch": 5},
                             {"kernel_source_sha": "0" * 16, "workload": "gqa32", "dram_bytes_per_launch": 6},
                             {"kernel_source_sha": sha, "workload": "long", "dram_bytes_per_launch": 7}]))
    assert bench.committed_traffic("llama8b") == 5 and bench.committed_traffic("long") == 7
    assert bench.committed_traffic("gqa32") is None and bench.committed_traffic("ragged") is None
