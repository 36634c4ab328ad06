"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

Each rank runs an independent batch (no data-path collective); only the report is reduced:
the max over ranks of the timings and the sum of the work. The reference arm runs on rank 0
only; other ranks return without work."""
import multiprocessing as mp
import os
import socket


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times, work = bench.reduce_over_ranks([1.0 + rank, 10.0 * (rank + 1)], 100.0 * (rank + 1), "cpu")
        seed_notes = bench.workload(2, rank).notes
        q.put((rank, times, work, seed_notes))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_independent_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, times, work, _ in res:
        assert times == [2.0, 20.0]          # max over ranks
        assert work == 300.0                 # sum over ranks
    assert res[0][3] != res[1][3]            # every rank draws its own batch


def test_reference_arm_runs_on_rank0_only(capsys):
    import argparse
    import bench
    bench.run_reference(argparse.Namespace(config=2, steps=1, warmup=0), rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_single_process_reduction_is_identity():
    import bench
    assert bench.reduce_over_ranks([3.0, 4.0], 7.0, "cpu") == ([3.0, 4.0], 7.0)


def test_reference_arm_prints_the_contract_line():
    """One step of the reference arm (the fp64 oracle on a bounded row sample) prints one
    JSON line with every key the benchmark contract names."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "1", "--steps", "1",
                        "--warmup", "3", "--cpu-seconds", "0.5"], capture_output=True, text=True, timeout=600,
                       cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["value"] > 0 and j["steps"] == 1
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["value"] == j["value"]
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1


def test_traffic_figures_are_keyed_to_the_current_kernel_sources():
    """bench.py reports the ncu DRAM traffic of a workload only while the forward kernels'
    sources hash to the value the figure was recorded under. An entry left behind by a
    kernel edit is stale: recapture it, or remove it (the bench line then reports null)."""
    import json
    import bench
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "profiles", "fwd_traffic.json")) as f:
        table = json.load(f)
    for name, entry in table.items():
        assert entry["kernel_source_hash"] == bench.kernel_source_hash(), f"stale traffic entry {name}"
        assert bench.traffic_for(name) == entry["dram_bytes_per_launch"]
        # a figure is measured on the source it is keyed to: a capture taken on other source
        # and relabelled afterwards is not a measurement of this kernel
        assert entry.get("captured_at_hash", entry["kernel_source_hash"]) == entry["kernel_source_hash"], name
        assert "re-key" not in entry.get("note", "") and "rekey" not in entry.get("note", ""), name
