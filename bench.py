#!/usr/bin/env python
"""Benchmark of the MoE route -> layout -> dispatch -> combine path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config dsv3,kimi,prefill]
                    [--impl ours|reference]

One step = one pass of the whole path over one batch of seeded synthetic
input: moe_route_topk, moe_dispatch_layout, moe_dispatch_fp8 (or _bf16) and
moe_combine_bf16.  The stand-in expert between dispatch and combine is not
part of the path (it needs trained weights): its outputs are prepared once,
before timing, and stay resident, as a grouped GEMM would leave them.

By default one run measures the decode workloads dsv3 and kimi and the
prefill workload, one after the other, and prints ONE JSON line: the
headline fields (value, roofline, e2e, cpu_baseline) belong to the largest
workload, prefill; every workload's step and dispatch+combine figures are in
its `configs` entry.

Timing: W untimed warm-up steps, then timed regions of exactly K steps, each
between a barrier + device synchronise on both sides.  The K-step region is
repeated until about a second of timed work has run (at least 5 times), and
the median region gives the reported time; the spread is reported beside it.
When a step moves more than twice the L2 size (126 MB) its inputs cannot
stay in L2 from one step to the next ("inputs larger than L2"); smaller
workloads write a 512 MiB buffer before every step to flush L2, outside the
timed events.  Each step and each stage is timed with CUDA events on the
stream the kernels run on; the timed loop calls the C ABI directly with
pre-marshalled arguments.  Clocks and throttle reasons are sampled with
nvidia-smi across the repeated regions.  With N > 1 (torchrun) every rank
runs an independent replica (the path does not shard: no data-path
collective); the reported time is the maximum over ranks and `value` the
bytes of all ranks over that time.

`value` is the effective HBM bandwidth of a step: the algorithmic bytes the
path must move (each token read once, each row written once, see
algorithmic_bytes) divided by the step time.  The reference arm
(--impl reference) times the oracle, a plain single-threaded CPU program,
on samples of the same headline workload, with the same metric and config.
"""
from __future__ import annotations

import argparse
import datetime as _dt
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from harness import experts, inputs  # noqa: E402

METRIC = "dispatch+combine µs/layer and effective HBM GB/s (% of B200 roofline), 1 GPU"
SPEC_HBM_GBS = 8000.0          # B200 HBM3e bandwidth the roofline target is quoted against
FALLBACK_HBM_GBS = 6650.0      # earlier measured copy bandwidth on this machine
L2_FLUSH_BYTES = 512 << 20
STEPS_PER_GRAPH = 10           # consecutive steps captured in one CUDA graph (no-flush workloads)
DEFAULT_CONFIGS = "dsv3,kimi,prefill"
REGION_TARGET_S = 1.0          # timed work per workload for the step (repeated K-step regions)
E2E_SETS = 3                   # e2e leg: streams with a device buffer set each, taken in turn
MIN_REPS, MAX_REPS = 5, 4000
DTYPES = {"route": "f32 logits -> f32 weights, int32 ids",
          "layout": "int32",
          "dispatch": "bf16 rows -> e4m3 codes + f32 1x128 scales (bf16 copy for bf16 workloads)",
          "combine": "bf16 rows, f32 multiply and add, bf16 out"}


# --------------------------------------------------------------------------
# algorithmic bytes
# --------------------------------------------------------------------------

def algorithmic_bytes(cfg: inputs.Config, rows: int, kept: int, combine_fp8: bool = False) -> dict:
    """Minimal bytes each stage must move.  kept = slots that have a row
    (T*k when nothing is dropped); rows = receive rows laid out.  With
    combine_fp8 the expert rows come back as E4M3 codes + 1x128 scales."""
    T, H, E, k, R = cfg.T, cfg.H, cfg.E, cfg.k_total, cfg.R
    E_lay = cfg.E_phys if cfg.n_shared else E
    S = H // 128
    route = T * E * 4 + T * k * 8
    layout = T * k * 4 + E_lay * 4 * (2 + R) + 4 + R * 4 + T * k * 4 + rows * 4
    if cfg.dispatch == "fp8":
        dispatch = T * H * 2 + T * k * 4 + kept * H + kept * S * 4
    else:
        dispatch = T * H * 2 + T * k * 4 + kept * H * 2
    if combine_fp8:
        combine = kept * H + kept * S * 4 + T * k * 8 + T * H * 2
    else:
        combine = kept * H * 2 + T * k * 8 + T * H * 2
    return dict(route=route, layout=layout, dispatch=dispatch, combine=combine,
                step=route + layout + dispatch + combine)


def load_peak() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def combine_traffic(cfg_name: str, fp8: bool = False):
    """DRAM bytes per launch of the combine kernel from the committed ncu
    summary, or None when that summary is missing or the kernel source has
    changed since it was taken."""
    kind = "combine_fp8" if fp8 else "combine"
    path = os.path.join(ROOT, "profiles", f"{kind}_{cfg_name}_traffic.json")
    src = os.path.join(ROOT, "combine_moe_route_08_b200", "csrc", "combine.cu")
    try:
        with open(path) as f:
            rec = json.load(f)
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256") != sha:
        return None
    return rec.get("dram_bytes_per_launch")


def config_names(arg: str) -> list[str]:
    names = [n.strip() for n in arg.split(",") if n.strip()]
    bad = [n for n in names if n not in inputs.CONFIGS]
    if not names or bad:
        raise SystemExit(f"unknown workload(s) {bad}; choose from {sorted(inputs.CONFIGS)}")
    return list(dict.fromkeys(names))


def headline_name(names: list[str]) -> str:
    """The largest workload of the run (tokens x hidden size): its figures
    are the line's headline."""
    return max(names, key=lambda n: (inputs.CONFIGS[n].T * inputs.CONFIGS[n].H, names.index(n)))


def pipeline_text(args) -> str:
    if args.fused:
        return "fused: route + layout + dispatch in one cooperative launch (moe_route_dispatch), then combine"
    if args.two_phase:
        return ("two-phase: private-region layout, send into E*R private regions of T_r rows, "
                "receiver compaction")
    return "direct scatter into the packed (or padded) rows"


def line_config(args, names: list[str], n_gpus: int) -> dict:
    """The workload description shared by both arms (no measured value in it)."""
    head = inputs.CONFIGS[headline_name(names)]
    return {
        "workload": head.describe(),
        "workloads": {n: inputs.CONFIGS[n].describe() for n in names},
        "parallelism": f"replicas x{n_gpus}",
        "pipeline": pipeline_text(args),
        "combine_payload": ("fp8 e4m3 + 1x128 fp32 scales (the dispatched rows)"
                            if args.combine_fp8 else "bf16 (stand-in expert output)"),
        "l2": ("inputs larger than L2 (no flush) for workloads that move more than 2 x L2 per "
               f"step; a {L2_FLUSH_BYTES >> 20} MiB write before every step outside the timed "
               "events otherwise"),
    }


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.windows: list[list] = []
        uuid = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
        except Exception:
            uuid = None
        self.sel = uuid or str(device_index)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def mark_start(self):
        self.windows.append([_dt.datetime.now(), None])

    def mark_end(self):
        if self.windows:
            self.windows[-1][1] = _dt.datetime.now()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0, "samples_in_timed_region": 0}
        time.sleep(0.1)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        return summarise_clock_samples(out, self.windows)


def summarise_clock_samples(out: str, windows: list) -> dict:
    """nvidia-smi CSV lines (ClockSampler.FIELDS, no header, no units) ->
    median SM clock, maximum clock, active throttle reasons and sample
    counts, from the samples inside the [start, end] windows when there are
    any, else from all of them."""
    rows = []
    for line in out.strip().splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            ts = _dt.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
        except ValueError:
            continue
        rows.append((ts, parts))
    inside = [p for ts, p in rows
              if any(a is not None and b is not None and a <= ts <= b for a, b in windows)]
    use = inside or [p for _, p in rows]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({n for p in use for n, v in zip(names, p[5:9]) if v.lower() == "active"})
    sm = [float(p[1]) for p in use if p[1].replace(".", "").isdigit()]
    smax = [float(p[2]) for p in use if p[2].replace(".", "").isdigit()]
    return {"sm_mhz": float(np.median(sm)) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "sm_mhz_min": min(sm) if sm else None,
            "reasons": reasons, "samples": len(rows), "samples_in_timed_region": len(inside),
            "from": "samples inside the timed regions" if inside else
                    "no sample fell inside the timed regions: samples around them"}


# --------------------------------------------------------------------------
# multi-rank plumbing (replicas: only a barrier and a max of the timings)
# --------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=_dt.timedelta(seconds=120))
    return dist


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index] if device is not None else None)
        else:
            dist.barrier()


def max_over_ranks(values: list[float], world: int, device) -> list[float]:
    """Element-wise maximum of per-rank timings (all ranks call this)."""
    if world == 1:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def repetitions(region_s: float, target_s: float) -> int:
    """How many K-step regions make about target_s seconds of timed work."""
    if not region_s > 0:
        return MIN_REPS
    return int(min(MAX_REPS, max(MIN_REPS, math.ceil(target_s / region_s))))


# --------------------------------------------------------------------------
# the oracle as CPU baseline / reference arm
# --------------------------------------------------------------------------

def oracle_step_on_sample(cfg: inputs.Config, wl: dict, tokens: int) -> tuple[float, int]:
    """Run the oracle's route -> layout -> dispatch -> combine on the first
    `tokens` tokens (whole logical ranks) of the workload; returns (seconds,
    algorithmic bytes of that sample)."""
    import oracle
    sub = inputs.Config(cfg.name, cfg.index, tokens // cfg.R if tokens % cfg.R == 0 else tokens,
                        cfg.R if tokens % cfg.R == 0 else 1, cfg.H, cfg.E, cfg.k, cfg.dispatch,
                        cfg.layout, cfg.expert, cfg.zipf, cfg.n_shared)
    T = sub.T
    logits = wl["logits_np"][:T]
    xb = wl["x_bits"][:T]
    E_lay = cfg.E_phys if cfg.n_shared else cfg.E
    t0 = time.perf_counter()
    if cfg.n_shared:
        idx, w, _ = oracle.route_ex(logits, cfg.k, cfg.n_shared, 1.0, *wl["placement"],
                                    cfg.E_phys, max(1, T // sub.R))
    else:
        idx, w = oracle.route(logits, cfg.k)
    lay = oracle.layout(idx, E_lay, sub.R)
    cap = 0
    if cfg.layout == "padded":
        cap = int(lay["expert_counts"].max())
        lay = oracle.layout(idx, E_lay, sub.R, cap)
    rows = lay["recv_src"].shape[0]
    pos = lay["dispatch_pos"]
    if cfg.dispatch == "fp8":
        oracle.dispatch_fp8(xb, pos, rows)
    else:
        oracle.dispatch_bf16(xb, pos, rows)
    y = wl["y_bank_bits"]
    pos_bank = np.where(pos >= 0, pos % y.shape[0], -1).astype(np.int32)
    oracle.combine(y, pos_bank, w)
    dt = time.perf_counter() - t0
    kept = int(np.sum(pos >= 0))
    return dt, algorithmic_bytes(sub, rows, kept)["step"]


def cpu_inputs(cfg: inputs.Config) -> dict:
    logits = inputs.make_logits(cfg)
    x = inputs.make_x(cfg)
    bank = inputs.make_row_bank(cfg.H, seed=cfg.seed * 10 + 2, n=min(cfg.T * cfg.k_total, 32768))
    return dict(logits_np=logits.numpy(), x_bits=inputs.bf16_bits(x),
                y_bank_bits=inputs.bf16_bits(bank),
                placement=inputs.expert_placement(cfg) if cfg.n_shared else None)


def cpu_baseline(cfg: inputs.Config, budget_s: float = 10.0) -> dict:
    """The oracle as it stands, single-threaded, on whole-workload steps
    repeated until about `budget_s` seconds of CPU work."""
    wl = cpu_inputs(cfg)
    total_t, total_b, n = 0.0, 0, 0
    while n == 0 or total_t < budget_s:
        dt, b = oracle_step_on_sample(cfg, wl, cfg.T)
        total_t += dt
        total_b += b
        n += 1
    return {"value": total_b / total_t / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "host_cores": os.cpu_count(), "workload": cfg.name,
            "sample": f"{n} full {cfg.name} step(s) (T={cfg.T}), {total_t:.1f} s of CPU work, "
                      f"1 thread of {os.cpu_count()} host cores",
            "s_per_step": total_t / n}


def run_reference(args) -> None:
    world, rank, _ = dist_env()
    if rank != 0:
        return  # the oracle runs on rank 0 only; other ranks exit without work
    names = config_names(args.config)
    cfg = inputs.CONFIGS[headline_name(names)]
    wl = cpu_inputs(cfg)
    # size each step so that warm-up + timed steps fit in about two minutes
    dt1, _ = oracle_step_on_sample(cfg, wl, cfg.R)           # one token per rank
    per_token = dt1 / cfg.R
    budget = 120.0 / max(1, args.steps + args.warmup)
    ranks = max(1, min(cfg.T_r, int(budget / per_token / cfg.R)))
    tokens = ranks * cfg.R
    for _ in range(args.warmup):
        oracle_step_on_sample(cfg, wl, tokens)
    tt, tb = 0.0, 0
    for _ in range(args.steps):
        dt, b = oracle_step_on_sample(cfg, wl, tokens)
        tt += dt
        tb += b
    value = tb / tt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16+e4m3", "dtypes": DTYPES, "data": "synthetic",
        "config": line_config(args, names, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "workload": cfg.name,
                         "sample": f"{tokens} of {cfg.T} {cfg.name} tokens per step "
                                   f"({ranks} per logical rank), 1 thread of {os.cpu_count()}"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def measure(cfg: inputs.Config, args, dev, world: int, local: int) -> dict:
    """Set up one workload on the device and time it (all ranks call this)."""
    import combine_moe_route_08_b200 as moe

    T, H, E, R = cfg.T, cfg.H, cfg.E, cfg.R
    k = cfg.k_total                         # slots per token (routed + shared)
    E_lay = cfg.E_phys if cfg.n_shared else E   # experts the layout sees
    logits_h = inputs.make_logits(cfg)
    x_h = inputs.make_x(cfg)
    logits = logits_h.to(dev)
    x = x_h.to(dev)
    s = torch.cuda.Stream(dev)
    ws = moe.Workspace(dev)

    if cfg.n_shared:
        offs_h, ids_h = inputs.expert_placement(cfg)
        replica_offsets = torch.from_numpy(offs_h).to(dev)
        replica_ids = torch.from_numpy(ids_h).to(dev)
    with torch.cuda.stream(s):
        if cfg.n_shared:
            idx, w = moe.moe_route_topk_ex(logits, cfg.k, cfg.n_shared, 1.0, replica_offsets,
                                           replica_ids, cfg.E_phys, cfg.T_r)
        else:
            idx, w = moe.moe_route_topk(logits, k)
        cap = 0
        if cfg.layout == "padded":  # capacity = max observed count, read once, untimed
            probe = moe.moe_dispatch_layout(idx, E_lay, R, workspace=ws)
            cap = int(probe["expert_counts"].max().item())
            del probe
        rows = T * k if cap == 0 else E_lay * cap
        lay = moe.moe_dispatch_layout(idx, E_lay, R, capacity=cap, rows=rows, workspace=ws)
        if args.combine_fp8 and cfg.dispatch != "fp8":
            raise SystemExit("--combine-fp8 needs FP8-dispatch workloads")
        if args.fused and args.two_phase:
            raise SystemExit("--fused runs the direct layout")
        if args.two_phase:
            if cap:
                raise SystemExit("--two-phase needs packed-layout workloads")
            max_m = cfg.T_r                      # a rank sends at most T_r tokens to an expert
            lay["private_pos"] = torch.empty(T, k, dtype=torch.int32, device=dev)
            moe.moe_dispatch_layout_private(idx, E_lay, R, max_m, out=lay, workspace=ws)
            prows = E_lay * R * max_m
        if args.two_phase and cfg.dispatch == "fp8":
            priv_q, priv_scale = moe.moe_dispatch_fp8(x, lay["private_pos"], prows)
        elif args.two_phase:
            priv_x = moe.moe_dispatch_bf16(x, lay["private_pos"], prows)
        if cfg.dispatch == "fp8":
            recv_q, recv_scale = moe.moe_dispatch_fp8(x, lay["dispatch_pos"], rows)
            y = experts.dequantise(recv_q, recv_scale)
        else:
            recv_x = moe.moe_dispatch_bf16(x, lay["dispatch_pos"], rows)
            y = recv_x.clone() if cfg.expert == "identity" else experts.affine(
                recv_x, inputs.make_expert_noise(cfg, rows))
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        kept = int((lay["dispatch_pos"] >= 0).sum().item())
        flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    s.synchronize()

    # the C ABI calls of a step with their arguments marshalled once
    lib, sp = moe.lib, s.cuda_stream
    ws_buf = ws.get(moe.moe_layout_workspace_bytes(T, k, E_lay, R))
    pos = lay["dispatch_pos"]
    route_call = (
        (lib.moe_route_topk_ex, (logits.data_ptr(), T, E, cfg.k, 0, cfg.n_shared, 1.0,
                                 replica_offsets.data_ptr(), replica_ids.data_ptr(),
                                 replica_ids.numel(), cfg.E_phys, cfg.T_r, idx.data_ptr(),
                                 w.data_ptr(), None, sp))
        if cfg.n_shared else
        (lib.moe_route_topk, (logits.data_ptr(), T, E, k, 0, idx.data_ptr(), w.data_ptr(), sp)))
    lay_args = (idx.data_ptr(), T, k, E_lay, R, cap, rows, lay["expert_counts"].data_ptr(),
                lay["expert_src_counts"].data_ptr(), lay["rank_counts"].data_ptr(),
                lay["expert_offsets"].data_ptr(), pos.data_ptr(), lay["recv_src"].data_ptr())
    if not args.two_phase:
        layout_call = (lib.moe_dispatch_layout, lay_args + (ws_buf.data_ptr(), ws_buf.numel(), None, sp))
        dispatch_calls = [
            (lib.moe_dispatch_fp8, (x.data_ptr(), T, H, k, pos.data_ptr(), recv_q.data_ptr(),
                                    recv_scale.data_ptr(), rows, None, sp)) if cfg.dispatch == "fp8" else
            (lib.moe_dispatch_bf16, (x.data_ptr(), T, H, k, pos.data_ptr(), recv_x.data_ptr(), rows,
                                     None, sp))]
    else:
        # the pages' two-phase form: private-region layout, send into the private
        # regions, receiver compaction into the packed rows
        ppos = lay["private_pos"]
        layout_call = (lib.moe_dispatch_layout_private,
                       lay_args[:5] + (max_m,) + lay_args[6:] +
                       (ppos.data_ptr(), ws_buf.data_ptr(), ws_buf.numel(), None, sp))
        if cfg.dispatch == "fp8":
            dispatch_calls = [
                (lib.moe_dispatch_fp8, (x.data_ptr(), T, H, k, ppos.data_ptr(), priv_q.data_ptr(),
                                        priv_scale.data_ptr(), prows, None, sp)),
                (lib.moe_compact_fp8, (priv_q.data_ptr(), priv_scale.data_ptr(), prows,
                                       ppos.data_ptr(), pos.data_ptr(), T, H, k, recv_q.data_ptr(),
                                       recv_scale.data_ptr(), rows, None, sp))]
        else:
            dispatch_calls = [
                (lib.moe_dispatch_bf16, (x.data_ptr(), T, H, k, ppos.data_ptr(), priv_x.data_ptr(),
                                         prows, None, sp)),
                (lib.moe_compact_bf16, (priv_x.data_ptr(), prows, ppos.data_ptr(), pos.data_ptr(),
                                        T, H, k, recv_x.data_ptr(), rows, None, sp))]
    if args.combine_fp8:
        # the expert rows come back in the dispatch's FP8 format: the stand-in
        # expert returns its input, the dispatched codes and scales
        combine_call = (lib.moe_combine_fp8, (recv_q.data_ptr(), recv_scale.data_ptr(),
                                              pos.data_ptr(), w.data_ptr(), T, H, k, rows,
                                              out.data_ptr(), None, sp))
    else:
        combine_call = (lib.moe_combine_bf16, (y.data_ptr(), pos.data_ptr(), w.data_ptr(), T, H,
                                               k, rows, out.data_ptr(), None, sp))
    if args.fused:
        # route + layout + dispatch in one cooperative launch, then combine
        # (with shared experts: the extended route, the layout over E_phys)
        fws_buf = moe.Workspace(dev).get(moe.moe_route_dispatch_workspace_bytes(T, k, E_lay, R))
        if cfg.n_shared:
            head = (logits.data_ptr(), T, E, cfg.k, 0, cfg.n_shared, 1.0,
                    replica_offsets.data_ptr(), replica_ids.data_ptr(), replica_ids.numel(),
                    cfg.E_phys, R, cap, x.data_ptr(), H, idx.data_ptr(), w.data_ptr(),
                    *lay_args[7:])
            f8, f16 = lib.moe_route_dispatch_ex_fp8, lib.moe_route_dispatch_ex_bf16
        else:
            head = (logits.data_ptr(), T, E, k, 0, R, cap, x.data_ptr(), H, idx.data_ptr(),
                    w.data_ptr(), *lay_args[7:])
            f8, f16 = lib.moe_route_dispatch_fp8, lib.moe_route_dispatch_bf16
        tail = (rows, fws_buf.data_ptr(), fws_buf.numel(), None, sp)
        fused_call = ((f8, head + (recv_q.data_ptr(), recv_scale.data_ptr()) + tail)
                      if cfg.dispatch == "fp8" else (f16, head + (recv_x.data_ptr(),) + tail))
        calls = [fused_call, combine_call]
        stage_end = [0, 0, 0]      # route, layout and dispatch all end with the fused call
    else:
        calls = [route_call, layout_call, *dispatch_calls, combine_call]
        # stage j ends after these call indices: route, layout, dispatch (1 or 2 calls)
        stage_end = [0, 1, 1 + len(dispatch_calls)]

    def step(ev=None):
        """One pass of the path; with `ev`, events ev[1..3] mark the stage ends."""
        for j, (fn, a) in enumerate(calls):
            rc = fn(*a)
            if rc != 0:
                raise moe.MoeError(rc, fn.__name__)
            if ev is not None:
                for q, end in enumerate(stage_end):
                    if end == j:
                        ev[q + 1].record(s)

    nb = algorithmic_bytes(cfg, rows, kept, args.combine_fp8)
    K, W = args.steps, args.warmup
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20)
    flush_needed = nb["step"] < 2 * l2
    if flush_needed:
        l2_mode = (f"flushed before every step ({L2_FLUSH_BYTES >> 20} MiB write outside the timed "
                   f"events; a step moves {nb['step'] / 1e6:.1f} MB < 2 x L2)")
    else:
        l2_mode = (f"inputs larger than L2: a step moves {nb['step'] / 1e6:.1f} MB > 2 x L2 "
                   f"({l2 / 1e6:.0f} MB), so no input stays in L2 between steps; no flush")

    def flush(i):
        if flush_needed:
            flush.buf.fill_(i)
    flush.buf = flush_buf

    # Steps run as replays of CUDA graphs of the C ABI calls (the library
    # launches its kernels with programmatic dependent launch).  Workloads
    # timed without an L2 flush put STEPS_PER_GRAPH consecutive steps in one
    # graph, as a model forward puts many layers in one graph, so the graph
    # launch latency is not paid per step; a 1-step graph runs the remainder.
    # Flushed workloads replay one step per graph with the flush in between.
    G = STEPS_PER_GRAPH if not flush_needed else 1
    with torch.cuda.stream(s):
        for i in range(2):
            step()
    s.synchronize()

    def capture(fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(n):
                fn()
        return g

    def timed_replays(g_many, g_one, n_steps):
        """n_steps steps as replays; returns per-step events (or region events)."""
        if G == 1:
            evs = []
            for i in range(n_steps):
                flush(i)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(s)
                g_one.replay()
                b.record(s)
                evs.append((a, b))
            return evs
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(n_steps // G):
            g_many.replay()
        for _ in range(n_steps % G):
            g_one.replay()
        b.record(s)
        return [(a, b)]

    def ms_per(evs, n_steps):
        return float(sum(a.elapsed_time(b) for a, b in evs)) / n_steps

    def region(g_many, g_one, sampler=None):
        """One timed region of exactly K steps between a barrier and a device
        synchronise on both sides; ms per step."""
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        if sampler is not None:
            sampler.mark_start()
        evs = timed_replays(g_many, g_one, K)
        s.synchronize()
        torch.cuda.synchronize(dev)
        if sampler is not None:
            sampler.mark_end()
        barrier(world, dev)
        return ms_per(evs, K)

    def repeated_regions(g_many, g_one, target_s, sampler):
        """Calibrate with one untimed-for-the-record region, then run the same
        number of K-step regions on every rank; per-rank median ms per step."""
        with torch.cuda.stream(s):
            t0 = time.perf_counter()
            region(g_many, g_one)
            region_s = time.perf_counter() - t0
            reps = int(max_over_ranks([float(repetitions(region_s, target_s))], world, dev)[0])
            got = [region(g_many, g_one, sampler) for _ in range(reps)]
        return float(np.median(got)), float(min(got)), float(max(got)), reps

    g_step1 = capture(step, 1)
    g_stepG = capture(step, G) if G > 1 else g_step1
    # dispatch+combine as the pages count it (layout + dispatch + combine,
    # route excluded): its own graphs, timed the same way
    dc_calls = calls if args.fused else calls[1:]   # fused: the route cannot be left out

    def dc_step():
        for fn, a in dc_calls:
            rc = fn(*a)
            if rc != 0:
                raise moe.MoeError(rc, fn.__name__)
    g_dc1 = capture(dc_step, 1)
    g_dcG = capture(dc_step, G) if G > 1 else g_dc1

    with torch.cuda.stream(s):
        timed_replays(g_stepG, g_step1, W)          # warm-up
        timed_replays(g_dcG, g_dc1, W)
        s.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    local_step, step_min, step_max, reps = repeated_regions(g_stepG, g_step1, args.region_seconds,
                                                            sampler)
    local_dc, dc_min, dc_max, dc_reps = repeated_regions(g_dcG, g_dc1, args.region_seconds / 2,
                                                         sampler)
    clocks = sampler.stop()

    # per-stage breakdown: G consecutive steps captured with timing events
    # between the stages (event record nodes inside the graph); each replay is
    # read back before the next
    K2 = min(K, 200)
    stage_ms = None
    try:
        xev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)]
               for _ in range(G)]
        g_st = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_st, stream=s):
            for q in range(G):
                xev[q][0].record(s)
                step(xev[q])
                xev[q][4].record(s)
        rows_ms = []
        with torch.cuda.stream(s):
            for i in range(max(1, K2 // G) + 2):
                flush(i)
                g_st.replay()
                s.synchronize()
                if i >= 2:
                    rows_ms += [[xev[q][j].elapsed_time(xev[q][j + 1]) for j in range(4)]
                                for q in range(G)]
        stage_ms = np.array(rows_ms).mean(0)
        stage_how = (f"event record nodes between the stages of {G} consecutive step(s) "
                     "inside one graph")
        del g_st
    except (RuntimeError, TypeError):
        stage_ms = None
    if stage_ms is None:  # one graph per stage, events between replays
        gs = []
        bounds = [0, *[j + 1 for j in stage_end], len(calls)]
        for j in range(4):
            if bounds[j] == bounds[j + 1]:
                gs.append(None)   # a stage merged into the previous call
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for fn, a in calls[bounds[j]:bounds[j + 1]]:
                    fn(*a)
            gs.append(g)
        rows_ms = []
        with torch.cuda.stream(s):
            for i in range(K2):
                flush(i)
                e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
                e[0].record(s)
                for j, g in enumerate(gs):
                    if g is not None:
                        g.replay()
                    e[j + 1].record(s)
                rows_ms.append(e)
            s.synchronize()
        stage_ms = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in rows_ms]).mean(0)
        stage_how = "one graph per stage, events between the replays"
        del gs

    # the combine kernel alone: G launches back to back in one graph, each
    # chained to the previous one by programmatic dependent launch, no event
    # node between them (workloads that move more than 2 x L2 per step only:
    # every launch then reads its rows from HBM)
    comb_alone_ms = None
    if not flush_needed:
        cfn, cargs = calls[-1]

        def comb_only():
            rc = cfn(*cargs)
            if rc != 0:
                raise moe.MoeError(rc, cfn.__name__)
        g_c = capture(comb_only, G)
        n_c = max(3, int(0.1 / max(float(stage_ms[3]) * 1e-3 * G, 1e-6)))
        with torch.cuda.stream(s):
            for _ in range(2):
                g_c.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            for _ in range(n_c):
                g_c.replay()
            b.record(s)
            s.synchronize()
        comb_alone_ms = max_over_ranks([a.elapsed_time(b) / (n_c * G)], world, dev)[0]
        del g_c

    # eager: the same calls launched one by one from Python, no graph -- the
    # cost a caller that does not capture graphs pays (launch latency included)
    K3 = min(K, 200)
    with torch.cuda.stream(s):
        for i in range(3):
            flush(i)
            step()
        s.synchronize()
        eev = []
        if flush_needed:
            for i in range(K3):
                flush(i)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(s)
                step()
                b.record(s)
                eev.append((a, b))
        else:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            for i in range(K3):
                step()
            b.record(s)
            eev.append((a, b))
        s.synchronize()
    local_eager = ms_per(eev, K3)
    ms = max_over_ranks([local_step, local_dc, local_eager, *[float(v) for v in stage_ms]], world,
                        dev)
    ms_step, ms_dc, ms_eager, ms_route, ms_layout, ms_dispatch, ms_combine = ms
    del g_step1, g_stepG, g_dc1, g_dcG

    # ---- end to end through the public API, host buffers in and out ----
    # Every step copies its inputs (logits, x) in from page-locked host memory
    # and its result out to page-locked host memory, inside the timed region.
    # Direct and fused pipelines go through the library's host-buffer entry
    # points (moe_route_dispatch_*_host, moe_combine_*_host), which enqueue
    # the copies and the kernels on one stream; consecutive steps take turns
    # on E2E_SETS streams with a device buffer set each, so one step's copies
    # overlap its neighbours' kernels and copies in the other direction.
    # The two-phase and shared-expert pipelines have no host-buffer entry
    # point: their steps are the device-pointer calls between torch copies on
    # two copy streams, double-buffered the same way.
    logits_pin = logits_h.pin_memory()
    x_pin = x_h.pin_memory()
    nsets = max(2, args.e2e_sets)
    out_pins = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(nsets)]
    n_e2e = min(K, 100)
    first, last = max(W, 3), max(W, 3) + n_e2e
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    host_api = not args.two_phase and not cfg.n_shared
    if host_api:
        e2e_how = ("host-buffer C ABI entry points per step (moe_route_dispatch_"
                   f"{'fp8' if cfg.dispatch == 'fp8' else 'bf16'}_host"
                   f"{' with MOE_HOST_FUSED' if args.fused else ''}, moe_combine_"
                   f"{'fp8' if args.combine_fp8 else 'bf16'}_host): every step's inputs copied "
                   "in from page-locked host memory and its result copied out, inside the "
                   f"timed region; steps take turns on {nsets} streams with a device buffer "
                   "set each; no L2 flush")
        streams = [torch.cuda.Stream(dev) for _ in range(nsets)]
        step_calls = []
        for q in range(nsets):
            with torch.cuda.stream(streams[q]):
                b = dict(logits=torch.empty_like(logits), x=torch.empty_like(x),
                         topk_idx=torch.empty_like(idx), topk_w=torch.empty_like(w),
                         out=torch.empty_like(out))
                for key in ("expert_counts", "expert_src_counts", "rank_counts",
                            "expert_offsets", "dispatch_pos", "recv_src"):
                    b[key] = torch.empty_like(lay[key])
                if cfg.dispatch == "fp8":
                    b["recv_q"], b["recv_scale"] = torch.empty_like(recv_q), torch.empty_like(recv_scale)
                else:
                    b["recv_x"] = torch.empty_like(recv_x)
                nbytes = (moe.moe_route_dispatch_workspace_bytes(T, k, E_lay, R) if args.fused
                          else moe.moe_layout_workspace_bytes(T, k, E_lay, R))
                b["ws"] = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
                b["status"] = torch.zeros(1, dtype=torch.int32, device=dev)
            sq = streams[q].cuda_stream
            stp = b["status"].data_ptr()
            head = (logits_pin.data_ptr(), x_pin.data_ptr(), T, E, k, 0, R, cap, H,
                    moe.MOE_HOST_FUSED if args.fused else 0,
                    *[b[key].data_ptr() for key in ("logits", "x", "topk_idx", "topk_w",
                                                    "expert_counts", "expert_src_counts",
                                                    "rank_counts", "expert_offsets",
                                                    "dispatch_pos", "recv_src")])
            tail = (rows, b["ws"].data_ptr(), b["ws"].numel(), stp, sq)
            if cfg.dispatch == "fp8":
                rd = (lib.moe_route_dispatch_fp8_host,
                      head + (b["recv_q"].data_ptr(), b["recv_scale"].data_ptr()) + tail)
            else:
                rd = (lib.moe_route_dispatch_bf16_host, head + (b["recv_x"].data_ptr(),) + tail)
            pw = (b["dispatch_pos"].data_ptr(), b["topk_w"].data_ptr(), T, H, k, rows,
                  b["out"].data_ptr(), out_pins[q].data_ptr(), stp, sq)
            cb = ((lib.moe_combine_fp8_host, (b["recv_q"].data_ptr(), b["recv_scale"].data_ptr())
                   + pw) if args.combine_fp8 else (lib.moe_combine_bf16_host, (y.data_ptr(),) + pw))
            step_calls.append(([rd, cb], b))
        ev_start = torch.cuda.Event()
        ev_end = [torch.cuda.Event() for _ in range(nsets)]
        torch.cuda.synchronize(dev)
        for i in range(last):
            q = i % nsets
            if i == first:
                torch.cuda.synchronize(dev)      # warm-up steps done on every stream
                t0.record(streams[0])
                ev_start.record(streams[0])
                for sq in streams[1:]:
                    sq.wait_event(ev_start)
            for fn, a in step_calls[q][0]:
                rc = fn(*a)
                if rc != 0:
                    raise moe.MoeError(rc, fn.__name__)
        for q in range(nsets):
            ev_end[q].record(streams[q])
            streams[0].wait_event(ev_end[q])
        t1.record(streams[0])
        torch.cuda.synchronize(dev)
        # no kernel reported an error (a capacity drop, a wait that gave up), and
        # the last step's result reached the host: the bits of the device buffer
        for _, b in step_calls:
            if int(b["status"].item()) not in (moe.MOE_OK, moe.MOE_ERR_CAPACITY):
                raise moe.MoeError(int(b["status"].item()), "host-buffer step")
        last_set = step_calls[(last - 1) % nsets][1]
        if not torch.equal(out_pins[(last - 1) % nsets].view(torch.int16),
                           last_set["out"].cpu().view(torch.int16)):
            raise RuntimeError("host result differs from the device buffer it was copied from")
        del step_calls, last_set, b
    else:
        e2e_how = ("device-pointer C ABI calls per step between torch copies: every step's "
                   "inputs copied in from page-locked host memory and its output copied out, on "
                   "two copy streams overlapping the neighbouring steps' compute; inputs and "
                   "output double-buffered; no L2 flush (this pipeline has no host-buffer "
                   "entry point)")
        logits2, x2, out2 = torch.empty_like(logits), torch.empty_like(x), torch.empty_like(out)
        swap = {logits.data_ptr(): logits2.data_ptr(), x.data_ptr(): x2.data_ptr(),
                out.data_ptr(): out2.data_ptr()}
        calls2 = [(fn, tuple(swap.get(v, v) if isinstance(v, int) else v for v in a))
                  for fn, a in calls]
        sets = [(logits, x, out, calls), (logits2, x2, out2, calls2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        torch.cuda.synchronize(dev)
        for i in range(last):
            lg, xx, oo, cl = sets[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[i % 2])   # step i-2 has finished reading this set
                if i == first:
                    t0.record(s_in)
                lg.copy_(logits_pin, non_blocking=True)
                xx.copy_(x_pin, non_blocking=True)
                ev_in[i % 2].record(s_in)
            s.wait_event(ev_in[i % 2])
            if i >= 2:
                s.wait_event(ev_out[i % 2])           # step i-2's output has left this buffer
            for fn, a in cl:
                rc = fn(*a)
                if rc != 0:
                    raise moe.MoeError(rc, fn.__name__)
            ev_done[i % 2].record(s)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i % 2])
                out_pins[i % 2].copy_(oo, non_blocking=True)
                ev_out[i % 2].record(s_out)
                if i == last - 1:
                    t1.record(s_out)
        torch.cuda.synchronize(dev)
        del calls2, sets
    e2e_ms = max_over_ranks([t0.elapsed_time(t1) / n_e2e], world, dev)[0]
    h2d = logits_h.numel() * 4 + x_h.numel() * 2
    d2h = out.numel() * 2

    peak, peak_kind = load_peak()
    n_gpus = world
    comb_gbs = nb["combine"] / (ms_combine * 1e-3) / 1e9
    dc_bytes = nb["layout"] + nb["dispatch"] + nb["combine"]
    dc_gbs = dc_bytes / (ms_dc * 1e-3) / 1e9
    if args.fused:
        stages = {"route+layout+dispatch": (ms_route + ms_layout + ms_dispatch) * 1e3,
                  "combine": ms_combine * 1e3}
        dc_how = ("CUDA graphs of the fused route+layout+dispatch launch + combine (the route "
                  "is inside the fused launch, so it is included), K-step regions timed like the step")
        kernels_per_step = 2
    else:
        stages = {"route": ms_route * 1e3, "layout": ms_layout * 1e3,
                  "dispatch": ms_dispatch * 1e3, "combine": ms_combine * 1e3}
        dc_how = "CUDA graphs of layout + dispatch + combine, K-step regions timed like the step"
        kernels_per_step = moe.kernels_per_step(T, k, E_lay, R, two_phase=args.two_phase)
    res = {
        "workload": cfg.describe(), "capacity": cap, "rows": rows, "l2": l2_mode,
        "value": n_gpus * nb["step"] / (ms_step * 1e-3) / 1e9,
        "ms_per_step": ms_step,
        "us_per_layer": ms_step * 1e3,
        "regions": {"steps_per_region": K, "repeats": reps, "median_us": ms_step * 1e3,
                    "min_us": step_min * 1e3, "max_us": step_max * 1e3,
                    "how": (f"{reps} regions of exactly K = {K} steps (replays of CUDA graphs of "
                            f"{G} consecutive step(s)), each between a barrier and a device "
                            "synchronise; the median region per rank, the maximum over ranks")},
        "stages_us": stages,
        "stage_timing": stage_how,
        "eager": {"us_per_step": ms_eager * 1e3, "steps": K3,
                  "how": "the same C ABI calls launched one by one, no CUDA graph, "
                         "events around the steps (L2 as for the headline)"},
        "dispatch_combine": {"us": ms_dc * 1e3, "bytes": dc_bytes, "how": dc_how,
                             "repeats": dc_reps, "min_us": dc_min * 1e3, "max_us": dc_max * 1e3,
                             "gbs": dc_gbs, "frac_of_8tbs": dc_gbs / SPEC_HBM_GBS,
                             "frac_of_measured": dc_gbs / peak},
        "bytes_per_step": nb,
        "roofline": {"bound": "hbm",
                     "kernel": "k_combine_fp8" if args.combine_fp8 else (
                         "k_combine_bf16_w32" if moe.moe_combine_bf16_long_form(T, H, k)
                         else "k_combine_bf16"),
                     "achieved": comb_gbs,
                     "peak": peak, "unit": "GB/s", "frac": comb_gbs / peak,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_kind == "measured" else "fallback 6650 GB/s",
                     "traffic": combine_traffic(cfg.name, args.combine_fp8),
                     "algorithmic_bytes_per_launch": nb["combine"],
                     "how": "algorithmic bytes of one launch over the combine stage's mean "
                            "CUDA-event time inside the step graph",
                     "alone": None if comb_alone_ms is None else {
                         "us": comb_alone_ms * 1e3,
                         "achieved": nb["combine"] / (comb_alone_ms * 1e-3) / 1e9,
                         "frac": nb["combine"] / (comb_alone_ms * 1e-3) / 1e9 / peak,
                         "how": f"the combine launched {G} times back to back in one CUDA graph "
                                "(programmatic dependent launch between them), events around "
                                "the replays; the stage time above also holds the launch and "
                                "ramp that the event nodes between stages expose"}},
        "e2e": {"value": n_gpus * nb["step"] / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "us_per_step": e2e_ms * 1e3, "h2d_bytes_per_step": h2d,
                "how": e2e_how,
                "d2h_bytes_per_step": d2h},
        "kernels_per_step": kernels_per_step,
        "clocks": clocks,
    }
    sm = clocks.get("sm_mhz")
    if sm:
        res["clocks"]["us_x_mhz"] = ms_step * 1e3 * sm
        res["clocks"]["dispatch_combine_us_x_mhz"] = ms_dc * 1e3 * sm
    del calls
    return res


def summary(res: dict) -> dict:
    """A workload's entry in the line's `configs`."""
    dc = res["dispatch_combine"]
    return {"workload": res["workload"], "us_per_layer": res["us_per_layer"], "value": res["value"],
            "unit": "GB/s", "regions": res["regions"], "stages_us": res["stages_us"],
            "eager_us": res["eager"]["us_per_step"],
            "dispatch_combine": {k: dc[k] for k in ["us", "gbs", "frac_of_8tbs", "frac_of_measured",
                                                    "bytes", "repeats", "min_us", "max_us"]},
            "roofline": {k: res["roofline"][k] for k in ["kernel", "achieved", "peak", "frac",
                                                         "traffic", "alone"]},
            "e2e_us": res["e2e"]["us_per_step"], "clocks": res["clocks"],
            "capacity": res["capacity"], "rows": res["rows"], "l2": res["l2"]}


def run_ours(args) -> None:
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    names = config_names(args.config)
    head = headline_name(names)
    results = {}
    for name in names:
        results[name] = measure(inputs.CONFIGS[name], args, dev, world, local)
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
    hr = results[head]
    K, W = args.steps, args.warmup
    if rank == 0:
        line = {
            "metric": METRIC, "value": hr["value"], "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": hr["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16+e4m3", "dtypes": DTYPES,
            "data": "synthetic",
            "config": line_config(args, names, world),
            "headline": head,
            "us_per_layer": hr["us_per_layer"],
            "timing": hr["regions"]["how"],
            "stages_us": hr["stages_us"],
            "stage_timing": hr["stage_timing"],
            "eager": hr["eager"],
            "dispatch_combine": hr["dispatch_combine"],
            "bytes_per_step": hr["bytes_per_step"],
            "roofline": hr["roofline"],
            "e2e": hr["e2e"],
            "gpu_launches": hr["kernels_per_step"] * K,
            "gpu_launches_how": (f"{hr['kernels_per_step']} library kernels per step x K = {K} "
                                 "steps per timed region (each region repeated, see timing)"),
            "clocks": hr["clocks"],
            "configs": {n: summary(r) for n, r in results.items()},
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(inputs.CONFIGS[head])
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world, dev)
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1,
                    help="ranks (one per GPU, launched by torch.distributed.run): independent replicas")
    ap.add_argument("--steps", type=int, default=20, help="steps per timed region")
    ap.add_argument("--warmup", type=int, default=5, help="untimed warm-up steps")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours",
                    help="reference: time the CPU oracle on samples of the headline workload")
    ap.add_argument("--config", default=DEFAULT_CONFIGS,
                    help="comma-separated seeded synthetic workloads, measured in turn; the "
                         f"largest is the headline (choices: {', '.join(sorted(inputs.CONFIGS))})")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip timing the oracle on the host (cpu_baseline)")
    ap.add_argument("--two-phase", action="store_true",
                    help="dispatch as the pages' two-phase form (private regions + compaction)")
    ap.add_argument("--fused", action="store_true",
                    help="route + layout + dispatch as one cooperative launch, then combine")
    ap.add_argument("--combine-fp8", action="store_true",
                    help="expert rows come back as E4M3 + 1x128 scales (moe_combine_fp8)")
    ap.add_argument("--e2e-sets", type=int, default=E2E_SETS,
                    help="e2e leg: streams (each with its own device buffers) the steps take "
                         "turns on, so copies of neighbouring steps overlap")
    ap.add_argument("--region-seconds", type=float, default=REGION_TARGET_S,
                    help="timed work per workload: the K-step region repeats (at least 5 times) "
                         "until about this many seconds (dispatch+combine: half of it)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.steps < 1:
        ap.error("--steps must be at least 1")
    if args.region_seconds < 0:
        ap.error("--region-seconds must be >= 0")
    config_names(args.config)
    world = dist_env()[0]
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} with WORLD_SIZE={world}: launch one rank per GPU with "
                 "torch.distributed.run --nproc-per-node N")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
