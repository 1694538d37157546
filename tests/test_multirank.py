"""The N > 1 host path of bench.py, on CPU with the gloo backend (world size 2).

The attention path has no exchange step: ranks run independent batches and only
the timing is reduced (max over ranks).  These tests cover that reduction, the
whole-job throughput formula, and a two-rank launch of the reference arm, where
rank 0 alone works and prints one line.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.init_ranks(world, rank, "gloo")
    got = bench.max_over_ranks(dist, 1.0 + 3.0 * rank)
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert dict(out) == {0: 4.0, 1: 4.0}


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 1e9 bytes in 10 ms (the slowest rank) = 200 GB/s
    assert bench.job_throughput(1e9, 2, 10.0, 1e9) == pytest.approx(200.0)
    assert bench.max_over_ranks(None, 3.5) == 3.5


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--workload", "decode_tiny", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
    # the same workload object as this arm's line (one rank per GPU: parallelism replicas x1)
    sys.path.insert(0, ROOT)
    import bench
    import workloads as wl
    spec = wl.SPECS["decode_tiny"]
    assert d["config"] == bench.workload_config("decode_tiny", spec, wl.make_batch(spec, "cpu").num_slots, 1)


def test_clock_summary_keeps_the_timed_region():
    """The clocks reported beside a number are the samples taken while it was timed."""
    sys.path.insert(0, ROOT)
    import bench
    idle = (1000.0, 1965.0, set())
    busy = (1965.0, 1965.0, {"sw_power_cap"})
    hot = (1500.0, 1965.0, {"sw_thermal_slowdown"})
    c = bench.ClockSampler(0)
    c.samples = [(t,) + x for t, x in [(0.9, idle), (1.1, busy), (1.3, hot), (1.5, busy), (1.9, idle)]]
    c.t0, c.t1 = 1.0, 1.6
    got = c.summary()
    assert got["samples"] == 3 and got["sm_mhz"] == 1965.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"] and got["window"] == "in_region"
    # no sample inside the region: the first one after its start stands for it, marked as such
    c.t0, c.t1 = 1.12, 1.2
    got = c.summary()
    assert got["samples"] == 1 and got["sm_mhz"] == 1500.0 and got["reasons"] == ["sw_thermal_slowdown"]
    assert got["window"] == "post_region"
    c.samples = []
    assert c.summary()["reasons"] == ["unsampled"]


def test_every_bench_workload_is_a_named_spec():
    sys.path.insert(0, ROOT)
    import bench
    import workloads as wl
    assert set(bench.WORKLOADS) <= set(wl.SPECS)
    for name in bench.WORKLOADS:
        assert wl.SPECS[name].name == name
    # the seed ids are distinct, so no two workloads draw the same inputs
    ids = [s.cfg for s in wl.SPECS.values()]
    assert len(ids) == len(set(ids))
    # the step class matches the workload's mode
    modes = {"DecodeWorkload": "decode", "ExtendWorkload": "extend", "SageExtendWorkload": "extend",
             "SageWorkload": "sage", "SageSparseWorkload": "sage", "Fp8DecodeWorkload": "fp8"}
    for name, cls in bench.WORKLOADS.items():
        assert wl.SPECS[name].mode == modes[cls.__name__], name
