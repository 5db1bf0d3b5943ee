"""Host-side logic of bench.py that needs no GPU: the max-over-ranks timing reduction and the per-rank
chunk streams (world size 2 over gloo, on the CPU), the active-bytes formula, and the clock-sample
summary."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        got_world, got_rank, _ = bench.dist_env()
        # every rank contributes its own event time; all must see the largest
        t = bench.reduce_max(10.0 + 5.0 * rank)
        bench.barrier()
        out.put((got_rank, got_world, t, bench.shard_seed(0, got_rank)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_max_and_distinct_streams():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in range(2))
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[2] == 15.0 for r in res)          # max over ranks, seen by every rank
    assert res[0][3] != res[1][3]                    # each rank draws its own chunks (weak scaling)


def test_single_process_helpers_without_a_process_group():
    assert bench.reduce_max(3.5) == 3.5
    bench.barrier()  # no process group: a no-op


def test_active_bytes_formula():
    # decode layer, 17 active experts: router weights + gain/bias + x + y + W1_i and W2_i in bf16
    d, E, de, L = 2048, 64, 256, 8
    assert bench.active_bytes(d, E, de, L, 17) == 4 * d * E + 8 * E + 2 * L * d + 4 * L * d + 17 * 4 * d * de
    assert bench.active_bytes(d, E, de, L, 0) == 4 * d * E + 8 * E + 6 * L * d


def test_clock_summary_parses_samples(tmp_path):
    cs = bench.ClockSampler(0)
    cs.proc = object()  # pretend nvidia-smi ran
    cs.path = str(tmp_path / "clk.csv")
    with open(cs.path, "w") as f:
        f.write("1965, 1965, 500.1, 0x0, Not Active, Not Active, Not Active, Not Active\n")
        f.write("1860, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("1950, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    s = cs.summary()
    assert s["sm_mhz"] == 1950 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3


@pytest.mark.parametrize("workload,prefix", [("cls_losses", "cls_losses_"), ("fp8", "decode_"),
                                             ("backward", "backward_")])
def test_reference_arm_of_the_other_workloads(workload, prefix):
    # the workloads with runners of their own time the oracle too, under the GPU runner's metric and config
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload",
                          workload, "--steps", "1", "--warmup", "3"], capture_output=True, text=True, cwd=root,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["value"] > 0 and j["cpu_baseline"]["kind"] == "oracle"
    assert j["config"]["workload"].startswith(prefix)
    assert j["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_prints_the_contract_line():
    # bench.py --impl reference times the fp64 oracle on the host cores (no GPU) and prints one JSON
    # line with the benchmark's keys, its own CPU-baseline record and a host-only end-to-end figure
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "3"], capture_output=True, text=True, cwd=root, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["steps"] == 2 and j["warmup"] == 3 and j["value"] > 0
    assert j["config"]["workload"].startswith("tiny")
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == j["value"]
    e2e = j["e2e"]
    assert e2e["value"] == j["value"] and e2e["unit"] == j["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_gpus_flag_launches_that_many_ranks():
    # bench.py --gpus 2 started without a launcher runs itself as two ranks; with the reference arm
    # (the host-only fp64 oracle) rank 0 alone times and prints one JSON line that reports both ranks
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--workload", "tiny", "--steps", "2", "--warmup", "3"], capture_output=True, text=True,
                         cwd=root, timeout=600, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2
