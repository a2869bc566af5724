"""Host-side pieces of bench.py, on the CPU: the algorithmic byte counts, the
max-over-ranks reduction with two gloo ranks, and the reference arm's
rank-0-only output under a two-rank launch."""
import argparse
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402
from harness import inputs  # noqa: E402


def test_algorithmic_bytes_dsv3():
    cfg = inputs.CONFIGS["dsv3"]
    nb = bench.algorithmic_bytes(cfg, rows=cfg.T * cfg.k, kept=cfg.T * cfg.k)
    T, H, k = 4096, 7168, 8
    assert nb["dispatch"] == T * H * 2 + T * k * 4 + T * k * H + T * k * 56 * 4     # 301.07 MB
    assert nb["combine"] == T * k * H * 2 + T * k * 8 + T * H * 2                   # 528.74 MB
    assert nb["route"] == T * 256 * 4 + T * k * 8
    assert abs(nb["dispatch"] / 1e6 - 301.07) < 0.01
    assert abs(nb["combine"] / 1e6 - 528.74) < 0.01


def test_algorithmic_bytes_prefill_and_fp8_payload():
    """Prefill counts only the rows that are filled (padding rows are neither
    read nor written); the FP8 payload moves H code bytes and H/128 scales per
    row instead of 2H bytes."""
    cfg = inputs.CONFIGS["prefill"]
    T, H, k, S = 32768, 7168, 8, 56
    kept = T * k
    rows = 256 * 1105                               # padded: E x capacity
    nb = bench.algorithmic_bytes(cfg, rows=rows, kept=kept)
    assert nb["dispatch"] == T * H * 2 + T * k * 4 + kept * H + kept * S * 4    # 2408.6 MB
    assert nb["combine"] == kept * H * 2 + T * k * 8 + T * H * 2                # 4230.0 MB
    assert abs(nb["dispatch"] / 1e6 - 2408.58) < 0.01 and abs(nb["combine"] / 1e6 - 4229.96) < 0.01
    nb8 = bench.algorithmic_bytes(inputs.CONFIGS["dsv3"], rows=32768, kept=32768, combine_fp8=True)
    assert nb8["combine"] == 32768 * 7168 + 32768 * 56 * 4 + 32768 * 8 + 4096 * 7168 * 2  # 301.1 MB
    dropped = bench.algorithmic_bytes(cfg, rows=rows, kept=kept - 1000)
    assert nb["combine"] - dropped["combine"] == 1000 * H * 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    bench.init_dist(world, "gloo")
    got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank], world, torch.device("cpu"))
    bench.barrier(world)
    q.put((rank, got))
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 10.0, 0.5]


@pytest.mark.parametrize("world", [1, 2])
def test_reference_arm_prints_one_line_from_rank0(world, tmp_path):
    outs = []
    for rank in range(world):
        env = dict(os.environ, WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1")
        p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                            "--config", "tiny", "--steps", "3", "--warmup", "3",
                            "--gpus", str(world)],
                           env=env, capture_output=True, text=True, timeout=300)
        assert p.returncode == 0, p.stderr
        outs.append(p.stdout.strip())
    assert outs[0] and all(o == "" for o in outs[1:])
    line = json.loads(outs[0])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_default_workloads_and_headline():
    """The default run measures the decode and prefill targets; the largest
    workload (prefill) carries the headline; unknown names are refused."""
    names = bench.config_names(bench.DEFAULT_CONFIGS)
    assert names == ["dsv3", "kimi", "prefill"]
    assert bench.headline_name(names) == "prefill"
    assert bench.headline_name(["tiny", "mixtral"]) == "mixtral"
    assert bench.config_names("dsv3, dsv3,kimi") == ["dsv3", "kimi"]
    with pytest.raises(SystemExit):
        bench.config_names("dsv3,nope")


def test_both_arms_print_the_same_config():
    """The reference arm and ours build `config` from the same function, so
    the driver can match the two lines."""
    args = argparse.Namespace(fused=False, two_phase=False, combine_fp8=False)
    a = bench.line_config(args, ["dsv3", "kimi", "prefill"], 1)
    b = bench.line_config(args, bench.config_names(bench.DEFAULT_CONFIGS), 1)
    assert a == b
    assert a["workload"].startswith("prefill:") and set(a["workloads"]) == {"dsv3", "kimi", "prefill"}


def test_repeated_region_count():
    """About target seconds of K-step regions, never fewer than the minimum
    nor more than the maximum."""
    assert bench.repetitions(0.003, 1.0) == 334
    assert bench.repetitions(0.5, 1.0) == bench.MIN_REPS
    assert bench.repetitions(1e-7, 1.0) == bench.MAX_REPS
    assert bench.repetitions(0.0, 1.0) == bench.MIN_REPS


def test_gpus_must_match_the_launched_ranks():
    """--gpus N without N launched ranks is refused before any work."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--impl", "reference", "--config", "tiny"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode != 0 and "WORLD_SIZE=1" in p.stderr


def test_clock_summary_uses_the_samples_inside_the_timed_regions():
    """Samples inside the [start, end] windows decide the clock and the
    throttle reasons; samples outside count only when none fell inside."""
    import datetime as dt
    t0 = dt.datetime(2026, 1, 1, 12, 0, 0)

    def line(sec, mhz, power_cap="Not Active", thermal="Not Active"):
        ts = (t0 + dt.timedelta(seconds=sec)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, {mhz}, 1965, 900.0, 0x0, Not Active, Not Active, {thermal}, {power_cap}"

    out = "\n".join([line(0.0, 1965), line(1.0, 1700, power_cap="Active"),
                     line(1.2, 1720, power_cap="Active"), line(1.4, 1710, power_cap="Active"),
                     line(3.0, 1965, thermal="Active"), "garbage line"])
    win = [[t0 + dt.timedelta(seconds=0.9), t0 + dt.timedelta(seconds=1.5)]]
    got = bench.summarise_clock_samples(out, win)
    assert got["samples"] == 5 and got["samples_in_timed_region"] == 3
    assert got["sm_mhz"] == 1710.0 and got["sm_mhz_min"] == 1700.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]          # the thermal sample lies outside
    none_inside = bench.summarise_clock_samples(out, [[t0 + dt.timedelta(seconds=5),
                                                       t0 + dt.timedelta(seconds=6)]])
    assert none_inside["samples_in_timed_region"] == 0 and none_inside["sm_mhz"] == 1720.0
    assert none_inside["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
