"""Host-side logic of bench.py on CPU: the multi-rank reductions over gloo
(world size 2), per-rank seeding, clock-sample parsing, and the reference
(oracle) arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.max_over_ranks(10.0 + rank)
        sm = bench.sum_over_ranks(1.5 * (rank + 1))
        out[rank] = (mx, sm, bench.rank_seed(3, rank))
    finally:
        dist.destroy_process_group()


def test_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 11.0          # max over ranks
    assert out[0][1] == out[1][1] == 4.5           # sum over ranks
    assert out[0][2] == 3 and out[1][2] != 3       # rank 0 keeps the workload seed


def test_single_process_reductions_are_identity():
    assert bench.max_over_ranks(2.5) == 2.5
    assert bench.sum_over_ranks(2.5) == 2.5


def test_clock_summary_parsing():
    c = bench.ClockSampler(0)
    c.lines = [(100.0, "2026/12/02 10:00:00.000, 0, 1800, 1965, 900.5, 0x4, Not Active, "
                       "Not Active, Not Active, Active"),
               (100.2, "2026/12/02 10:00:00.200, 0, 1850, 1965, 950.0, 0x0, Not Active, "
                       "Not Active, Not Active, Not Active"),
               (150.0, "2026/12/02 10:00:50.000, 0, 345, 1965, 100.0, 0x0, Not Active, "
                       "Not Active, Not Active, Not Active")]
    c.mark(99.9, 100.3)
    s = c.summary()
    assert s["sm_mhz"] == 1825.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples_in_timed_region"] == 2


@pytest.mark.slow
def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "b2_t128_hq4_hkv2_d64", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_non_zero_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_every_traffic_record_matches_the_current_kernel_sources():
    # bench.py reports a leg's DRAM traffic only while the record's source sha
    # matches the kernel headers it was captured from; a stale record would
    # silently turn into a null.
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        records = json.load(f)["records"]
    assert set(records) == set(bench.LEG_SOURCES)
    for leg, rec in records.items():
        assert rec["kernel_source_sha"] == bench.kernel_source_sha(leg), leg
        assert rec["bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"], leg
        assert bench.traffic_bytes(leg, rec["workload"]) == rec["bytes_per_launch"], leg


def test_nominal_roofline_of_the_headline_workload():
    from causal_gqa_attention_03_b200 import inputs
    w = inputs.WORKLOADS[inputs.LARGEST]
    r = bench.nominal_roofline(1350.0, w)
    # tensor-bound: the I/O bytes over 8 TB/s allow far more than 2.25 PFLOP/s
    assert r["nominal_peak"] == 2250.0
    assert r["frac_nominal"] == 0.6 and r["target_met"]
    assert not bench.nominal_roofline(1349.0, w)["target_met"]
