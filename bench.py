#!/usr/bin/env python
"""SS2D forward throughput on B200: state-updates/s and HBM GB/s against the roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl ss2d|reference]
                    [--backward] [--gate]

A step is one fused SS2D forward (CrossScan -> S6 -> CrossMerge) over one batch of
the workload, with every input already resident in HBM.  The default workload is
VMamba-T stage 1 (B=128, D=192, H=W=56, N=16, fp32), whose inputs (about 2 GB) are
larger than the 126 MB L2, so no L2 flush is needed between timed steps.

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch shard of
the same size (weak scaling); the path has no exchange step, so there is no
collective on the data path -- only a barrier and a max over ranks of the timing.

Rank 0 prints one JSON line.  `--impl reference` times the fp64 CPU oracle on a
bounded sample of the same workload instead (rank 0 only).

`--workload 5` is the bidirectional scan of bimamba_inner_ref (Vim-T tokens, gated by
silu(z)): a step is one bidirectional forward (plus its backward under `--backward`).

`--paths diagonal` runs the fused forward (and backward) over the diagonal path set of
"Visual Mamba实战从零开始搭建图像分类模型附PyTorch代码" (section 3) instead of the cross scan.

`--proj` times the fused forward with its producer: per-path x_proj, then the scan computing
dt = softplus(dt_proj . x_dbl[:R] + bias) per step (MambaInnerFn.forward's projections);
with `--backward` each step adds the backward through the scan and both projections.
`--proj --conv 4` puts the per-path causal depthwise conv with SiLU (MambaInnerFn's
causal_conv1d, width 4) in front of the producer; the scan then runs in sequence form.

`--backward` adds the fused backward to every step; `--gate` times the scan in its
sequence form instead, u (B, 4D, L) with the output gate out * silu(z) and the last
state (selective_scan_fn's z and return_last_state), plus its backward with dz
under `--backward`.  Neither is the headline line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import ss2d_inputs  # noqa: E402

METRIC = "SS2D fwd state-updates/s (B·4·D·L·N) and achieved HBM GB/s vs B200 roofline"
UNIT = "state-updates/s"
SM_COUNT = 148
MUFU_EX2_PER_CLK_PER_SM = 16  # measured on this B200 pool: 16.00 MUFU.EX2 per clock per SM
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "source": "fallback"}
REFERENCE_ITEMS_PER_STEP = 16


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


def fwd_algorithmic_bytes(w) -> int:
    """Bytes the forward must move at least once: read x, delta, B, C, the fp32 parameters; write y."""
    s = 4 if w.dtype == "f32" else 2
    Bn, Dn, L, N = w.batch, w.dim, w.L, w.d_state
    return s * (Bn * Dn * L + 4 * Bn * Dn * L + 8 * Bn * N * L) + s * Bn * Dn * L + 4 * 4 * Dn * (N + 2)


def seq_fwd_algorithmic_bytes(w, gate: bool) -> int:
    """The sequence-form forward: read u, delta (B, 4D, L), B, C, z if gated; write out and
    the last state (B, 4D, N) fp32."""
    s = 4 if w.dtype == "f32" else 2
    Bn, Dn, L, N = w.batch, w.dim, w.L, w.d_state
    seq = 4 * Bn * Dn * L
    return s * (seq * (3 if gate else 2) + 8 * Bn * N * L) + s * seq + 4 * 4 * Bn * Dn * N + 4 * 4 * Dn * (N + 2)


def bidir_algorithmic_bytes(w, backward: bool) -> int:
    """The bidirectional scan.  Forward: read x, delta, z (B, D, L), B, C (B, N, L); write y.
    Backward: read x, delta, z, dy, B, C; write dx, ddelta, dz, dB, dC.  Plus A, A_b, D, bias
    (and their gradients)."""
    s = 4 if w.dtype == "f32" else 2
    Bn, Dn, L, N = w.batch, w.dim, w.L, w.d_state
    seq, bc = Bn * Dn * L, 2 * Bn * N * L
    params = 4 * (2 * Dn * N + 2 * Dn)
    if backward:
        return s * (4 * seq + bc) + s * (3 * seq + bc) + 2 * params
    return s * (3 * seq + bc) + s * seq + params


def proj_algorithmic_bytes(w, R: int) -> int:
    """The fused forward with its producer: read x and the small weights once, write y and the
    saved projections x_dbl (B, 4, R+2N, L); delta, B and C never go through HBM as inputs."""
    s = 4 if w.dtype == "f32" else 2
    Bn, Dn, L, N = w.batch, w.dim, w.L, w.d_state
    weights = 4 * (4 * (R + 2 * N) * Dn + 4 * Dn * R + 4 * Dn * (N + 2))
    return s * Bn * Dn * L + s * Bn * Dn * L + s * Bn * 4 * (R + 2 * N) * L + weights


def bwd_algorithmic_bytes(w, gate: bool = False) -> int:
    """Bytes the backward must move at least once.  Fused form: read x, delta, B, C, dy, write
    dx, ddelta, dB, dC.  Sequence form: u, delta, B, C, dout (+ z) in, du, ddelta, dB, dC (+ dz)
    out.  Plus the fp32 parameters and their gradients."""
    s = 4 if w.dtype == "f32" else 2
    Bn, Dn, L, N = w.batch, w.dim, w.L, w.d_state
    img = Bn * Dn * L
    bc = 8 * Bn * N * L
    params = 2 * 4 * 4 * Dn * (N + 2)
    if gate:
        seq = 4 * img
        return s * (seq * 2 + bc) + s * seq + s * (seq * 2 + bc) + 2 * s * seq + params
    return s * (2 * img + 4 * img + bc) + s * (img + 4 * img + bc) + params


# the files the recorded forward scan kernel is compiled from
FWD_KERNEL_SOURCES = ("selective_scan_crossscan_b200/csrc/scan_fwd.cu", "selective_scan_crossscan_b200/csrc/common.cuh",
                      "selective_scan_crossscan_b200/csrc/kernels.h", "include/ss2d.h")


def source_hash(files=FWD_KERNEL_SOURCES) -> str:
    """Hash of a kernel's source files: ncu traffic figures are only reused for the exact same kernel."""
    h = hashlib.sha256()
    for rel in files:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(rel.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name: str):
    """dram read+write bytes per launch of the dominant kernel from a committed ncu capture, if the
    kernel's sources have not changed since it was taken; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(workload_name)
    if not entry:
        return None
    files = tuple(entry.get("sources") or FWD_KERNEL_SOURCES)
    try:
        if entry.get("source_hash") != source_hash(files):
            return None
    except OSError:
        return None
    return entry.get("traffic_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="ss2d_clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()
        return False

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [v for v in sm if v > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shard_seed(workload_index: int, rank: int) -> int:
    """every rank draws its own batch shard of the workload"""
    return workload_index + 1000 * rank


# ------------------------------------------------------------------ CPU oracle

def oracle_sample(w, seed: int, item: int):
    """one batch item of the workload, on the host, as float64 arrays for the oracle"""
    one = w.with_batch(1)
    return ss2d_inputs.make_inputs(one, seed=seed + 7919 * item, device="cpu", with_dy=False)


def _oracle_item(oracle, w, item: int) -> float:
    """Seconds the fp64 oracle's SS2D forward takes on batch item `item` (inputs drawn untimed)."""
    inp = oracle_sample(w, 0, item)
    args = [oracle._f64(inp[k]) for k in ("x", "delta", "A", "B", "C", "D", "delta_bias")]
    t0 = time.perf_counter()
    oracle.ss2d_forward(*args, True)
    return time.perf_counter() - t0


def time_oracle(w, seconds_budget: float = 15.0, steps: int | None = None, warmup: int = 1,
                items_per_step: int = 1):
    """Time the fp64 oracle's SS2D forward on whole batch items of the workload (bounded sample).

    steps=None: after `warmup` untimed items, time items one by one until `seconds_budget` seconds
    of oracle time are spent or every batch item has run.  Otherwise: exactly `steps` steps of
    `items_per_step` items each after the warm-up."""
    import oracle
    oracle.build()
    for i in range(warmup):
        _oracle_item(oracle, w, i)
    items_done, t_total, step_s = 0, 0.0, []
    item = warmup
    if steps is None:
        while items_done < w.batch and (items_done == 0 or t_total < seconds_budget):
            t_total += _oracle_item(oracle, w, item % w.batch)
            items_done += 1
            item += 1
    else:
        for _ in range(steps):
            t = 0.0
            for _ in range(items_per_step):
                t += _oracle_item(oracle, w, item % w.batch)
                item += 1
            step_s.append(t)
            t_total += t
            items_done += items_per_step
    per_item_updates = w.with_batch(1).updates
    value = items_done * per_item_updates / t_total
    what = (f"{items_done} batch item(s) of {w.name} ({per_item_updates} updates each"
            + (f", {items_per_step} per step" if steps is not None else "") + ")")
    return dict(value=value, unit=UNIT, cores=oracle.num_threads(), kind="oracle",
                ms_per_item=1e3 * t_total / max(items_done, 1),
                ms_per_step=1e3 * t_total / len(step_s) if step_s else None,
                sample=f"{what}, fp64 C oracle with OpenMP over (batch, channel)",
                seconds=t_total)


# ----------------------------------------------------------------- GPU bench

def run_gpu(args, world, rank, local):
    import selective_scan_crossscan_b200 as ss
    from selective_scan_crossscan_b200 import _build

    if rank == 0 or not os.path.exists(ss.library_path()):
        _build.build()
    barrier(world)
    w = ss2d_inputs.workload(args.workload)
    if args.batch:
        w = w.with_batch(args.batch)
    dev = torch.device("cuda", local)
    bidir = w.kind == "bidir"
    if args.proj:
        inp = ss2d_inputs.make_proj_inputs(w, seed=shard_seed(args.workload, rank), device=dev, d_conv=args.conv)
    elif bidir:
        inp = ss2d_inputs.make_bimamba_inputs(w, seed=shard_seed(args.workload, rank), device=dev,
                                              with_dy=args.backward, with_z=True)
    elif args.gate:
        inp = ss2d_inputs.make_scan_inputs(w, seed=shard_seed(args.workload, rank), device=dev,
                                           with_dout=args.backward, with_z=True)
    else:
        inp = ss2d_inputs.make_inputs(w, seed=shard_seed(args.workload, rank), device=dev, with_dy=args.backward)
    y = torch.empty((w.batch, w.dim, w.height, w.width), dtype=w.torch_dtype, device=dev)
    nbytes = ss.workspace_bytes(w.batch, w.dim, w.height, w.width, w.d_state, ss.OP_FORWARD, w.torch_dtype)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    if args.proj:
        pargs = (inp["x"], inp["x_proj_weight"], inp["dt_proj_weight"], inp["dt_proj_bias"], inp["A"], inp["D"])

        npj = ss.workspace_bytes(w.batch, w.dim, w.height, w.width, w.d_state, ss.OP_FORWARD_PROJ, w.torch_dtype)
        wsp = torch.empty(max(npj, 1), dtype=torch.uint8, device=dev)

        if args.conv:
            cargs = (inp["x"], inp["conv_weight"], inp["conv_bias"]) + pargs[1:]
            npc = ss.workspace_bytes(w.batch, w.dim, w.height, w.width, w.d_state, ss.OP_FORWARD_PROJ_CONV,
                                     w.torch_dtype)
            wspc = torch.empty(max(npc, 1), dtype=torch.uint8, device=dev)
        if args.backward:
            gdy = torch.Generator(device=dev)
            gdy.manual_seed(shard_seed(args.workload, rank) + 7000)
            dy = torch.randn((w.batch, w.dim, w.height, w.width), generator=gdy, device=dev).to(w.torch_dtype)
            nbp = ss.workspace_bytes(w.batch, w.dim, w.height, w.width, w.d_state, ss.OP_BACKWARD_PROJ,
                                     w.torch_dtype)
            wsbp = torch.empty(max(nbp, 1), dtype=torch.uint8, device=dev)

            if args.conv:
                nbc = ss.workspace_bytes(w.batch, w.dim, w.height, w.width, w.d_state, ss.OP_BACKWARD_PROJ_CONV,
                                         w.torch_dtype)
                wsbc = torch.empty(max(nbc, 1), dtype=torch.uint8, device=dev)

                def step():
                    # the same with the per-path causal conv in front of the producer
                    _, xd, cs = ss.ss2d_forward_proj_conv(*cargs, True, out=y, return_x_dbl=True,
                                                          return_chunk_states=True, workspace=wspc)
                    ss.ss2d_backward_proj_conv(*cargs, xd, dy, True, chunk_states=cs, workspace=wsbc)
            else:
                def step():
                    # forward keeping x_dbl and the chunk states, then the backward through scan and producer
                    _, xd, cs = ss.ss2d_forward_proj(*pargs, True, out=y, return_x_dbl=True,
                                                     return_chunk_states=True, workspace=wsp)
                    ss.ss2d_backward_proj(*pargs, xd, dy, True, chunk_states=cs, workspace=wsbp)
        elif args.conv:
            def step():
                ss.ss2d_forward_proj_conv(*cargs, True, out=y, workspace=wspc)
        else:
            def step():
                ss.ss2d_forward_proj(*pargs, True, out=y, workspace=wsp)
    elif bidir:
        y_seq = torch.empty((w.batch, w.dim, w.L), dtype=w.torch_dtype, device=dev)
        nbf = ss.workspace_bytes(w.batch, w.dim, 1, w.L, w.d_state, ss.OP_BIMAMBA_FORWARD, w.torch_dtype)
        wsf = torch.empty(max(nbf, 1), dtype=torch.uint8, device=dev)
        nbb = ss.workspace_bytes(w.batch, w.dim, 1, w.L, w.d_state, ss.OP_BIMAMBA_BACKWARD, w.torch_dtype)
        wsb2 = torch.empty(max(nbb, 1), dtype=torch.uint8, device=dev)
        bargs = (inp["x"], inp["delta"], inp["A"], inp["A_b"], inp["B"], inp["C"], inp["D"], inp["z"],
                 inp["delta_bias"], True)

        def step():
            # bidirectional forward (keeping the chunk states under --backward), then its backward
            res = ss.bimamba_forward(*bargs, out=y_seq, return_chunk_states=args.backward, workspace=wsf)
            if args.backward:
                ss.bimamba_backward(*bargs, inp["dy"], chunk_states=res[1], workspace=wsb2)
    elif args.gate:
        seq_out = torch.empty((w.batch, 4 * w.dim, w.L), dtype=w.torch_dtype, device=dev)

        def step():
            # gated sequence-form forward (keeping the chunk states under --backward), then the
            # gated backward from them
            res = ss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                        inp["delta_bias"], True, out=seq_out, z=inp["z"], return_last_state=True,
                                        return_chunk_states=args.backward)
            if args.backward:
                ss.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                      inp["delta_bias"], True, inp["dout"], chunk_states=res[2], z=inp["z"])
    elif args.paths == "diagonal":
        tables = ss.path_tables(w.height, w.width, ss.PATHS_DIAGONAL, device=dev)
        nf = ss.workspace_bytes(w.batch, w.dim, w.height, w.width, w.d_state, ss.OP_FORWARD_TABLE, w.torch_dtype)
        wst = torch.empty(max(nf, 1), dtype=torch.uint8, device=dev)
        cs = None
        if args.backward:
            nb = ss.workspace_bytes(w.batch, w.dim, w.height, w.width, w.d_state, ss.OP_BACKWARD_TABLE,
                                    w.torch_dtype)
            wsb = torch.empty(max(nb, 1), dtype=torch.uint8, device=dev)
            cs = torch.empty((w.batch, 4 * w.dim, -(-w.L // ss.CHUNK_LEN), w.d_state), dtype=torch.float32,
                             device=dev)
        targs = (inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"], True)

        def step():
            if args.backward:
                _, c = ss.ss2d_forward_table(*targs, tables, out=y, return_chunk_states=True, workspace=wst)
                ss.ss2d_backward_table(*targs, inp["dy"], tables, chunk_states=c, workspace=wsb)
            else:
                ss.ss2d_forward_table(*targs, tables, out=y, workspace=wst)
    elif args.backward:
        nb = ss.workspace_bytes(w.batch, w.dim, w.height, w.width, w.d_state, ss.OP_BACKWARD, w.torch_dtype)
        wsb = torch.empty(max(nb, 1), dtype=torch.uint8, device=dev)
        cs = torch.empty((w.batch, 4 * w.dim, -(-w.L // ss.CHUNK_LEN), w.d_state), dtype=torch.float32, device=dev)

        def step():
            # forward keeping the chunk states, then the fused backward from them
            ss.ss2d_forward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                            True, out=y, workspace=ws, chunk_states_out=cs)
            ss.ss2d_backward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                             True, inp["dy"], chunk_states=cs, workspace=wsb)
    else:
        def step():
            ss.ss2d_forward(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["delta_bias"],
                            True, out=y, workspace=ws)

    # kernels per step (to size the trace-event list)
    before = ss.launch_count()
    step()
    torch.cuda.synchronize(dev)
    launches_per_step = ss.launch_count() - before

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    # timed region: events around every step, plus the library's per-kernel trace events
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    traces = [[torch.cuda.Event(enable_timing=True) for _ in range(launches_per_step)] for _ in range(args.steps)]
    begin = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.__enter__()
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = ss.launch_count()
    begin.record(stream)
    for i in range(args.steps):
        starts[i].record(stream)
        with ss.trace_events(traces[i]):
            step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    gpu_launches = ss.launch_count() - launches0
    if sampler:
        sampler.__exit__(None, None, None)
    total_ms = begin.elapsed_time(end)
    ms_local = total_ms / args.steps
    ms = max_over_ranks(ms_local, world)

    # per-kernel durations inside the timed region
    per_kernel = [0.0] * launches_per_step
    for i in range(args.steps):
        prev = starts[i]
        for j, ev in enumerate(traces[i]):
            per_kernel[j] += prev.elapsed_time(ev)
            prev = ev
    per_kernel = [t / args.steps for t in per_kernel]
    dom = max(range(launches_per_step), key=lambda j: per_kernel[j])
    dom_ms = per_kernel[dom]

    units_total = sum_over_ranks(float(w.updates), world)
    value = units_total / (ms / 1e3)

    peaks = load_peaks()
    clocks = sampler.summary() if sampler else None
    # algorithmic bytes of the dominant kernel: the backward's when a backward runs in the step
    if args.proj and args.conv and not args.backward:
        alg_bytes = seq_fwd_algorithmic_bytes(w, gate=False)  # the scan runs in sequence form on u
    elif args.proj and not args.backward:
        alg_bytes = proj_algorithmic_bytes(w, inp["R"])
    elif bidir:
        alg_bytes = bidir_algorithmic_bytes(w, args.backward)
    elif args.backward:
        alg_bytes = bwd_algorithmic_bytes(w, gate=args.gate)
    elif args.gate:
        alg_bytes = seq_fwd_algorithmic_bytes(w, gate=True)
    else:
        alg_bytes = fwd_algorithmic_bytes(w)
    bytes_per_update = alg_bytes / w.updates
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved_gbs = bytes_per_update * w.updates / (dom_ms / 1e3) / 1e9
    sm_max = float(peaks.get("sm_max_mhz", FALLBACK_PEAKS["sm_max_mhz"]))
    sfu_peak = MUFU_EX2_PER_CLK_PER_SM * SM_COUNT * sm_max * 1e6 / 1e9  # G ex2/s at max clock
    sfu_achieved = w.updates / (dom_ms / 1e3) / 1e9  # one exp(dt*A) per state update
    # the traffic record is of the fused forward's scan kernel: other lines have no capture
    traffic = (recorded_traffic(w.name)
               if not (args.backward or args.gate or bidir or args.paths != "cross" or args.proj) else None)

    e2e = None
    if not (args.no_e2e or args.backward or args.gate or bidir or args.paths != "cross" or args.proj):
        e2e = run_e2e(args, w, inp, dev, stream, world, rank)

    result = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32" if w.dtype == "f32" else "bf16",
        "data": "synthetic (seeded; VMamba init recipe for A, D, delta_bias)",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "global_batch": w.batch * world, "dim": w.dim,
                   "height": w.height, "width": w.width, "d_state": w.d_state, "paths": w.paths,
                   "parallelism": f"batch shards x{world}, no collective",
                   "pass": ("forward + backward" if args.backward else "forward")
                   + (" (sequence form, gate z + last state)" if args.gate else "")
                   + (" (bidirectional, gate z)" if bidir else "")
                   + (f" ({args.paths} paths)" if args.paths != "cross" else "")
                   + (" (with the per-path x_proj/dt_proj producer)" if args.proj else "")
                   + (f" (and its per-path causal conv, width {args.conv})" if args.proj and args.conv else ""),
                   "l2": f"inputs {alg_bytes / 1e9:.2f} GB > 126 MB L2, no flush needed"},
        # the dominant (scan) kernel is bound by its exponentials on the SFU: that is the roofline;
        # the HBM view the metric names is reported beside it
        "roofline": {"bound": "alu", "achieved": sfu_achieved, "peak": sfu_peak, "unit": "G ex2/s",
                     "frac": sfu_achieved / sfu_peak, "traffic": traffic,
                     "kernel": f"launch {dom} of {launches_per_step} per step", "kernel_ms": dom_ms,
                     "algorithmic_ex2_per_update": 1,
                     "peak_source": "derived: 16 MUFU.EX2 per clock per SM (measured on this pool) x 148 SMs x "
                                    f"{sm_max:.0f} MHz maximum SM clock"},
        "hbm_roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved_gbs / hbm_peak, "traffic": traffic,
                         "algorithmic_bytes_per_update": bytes_per_update,
                         "peak_source": f"{peaks.get('source')} hbm_gbs (b.copy_ burst)"},
        "kernel_ms": per_kernel,
        "gpu_launches": gpu_launches,
        "clocks": clocks,
        "e2e": e2e,
    }
    # the oracle sample times the fused forward, so it is reported beside the forward line only
    if rank == 0 and world == 1 and not (args.no_cpu_baseline or args.backward or args.gate or bidir
                                         or args.paths != "cross" or args.proj):
        result["cpu_baseline"] = time_oracle(w, seconds_budget=args.cpu_seconds)
    return result


def run_e2e(args, w, inp, dev, stream, world, rank):
    """The same metric end to end through the public API: pinned host inputs -> device, fused
    forward, device -> host read of y, every step."""
    import selective_scan_crossscan_b200 as ss
    keys = ("x", "delta", "A", "B", "C", "D", "delta_bias")
    host = {k: inp[k].to("cpu").pin_memory() for k in keys}
    devbuf = {k: torch.empty_like(inp[k]) for k in keys}
    y_host = torch.empty((w.batch, w.dim, w.height, w.width), dtype=w.torch_dtype).pin_memory()
    h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
    d2h = y_host.numel() * y_host.element_size()
    nbytes = ss.workspace_bytes(w.batch, w.dim, w.height, w.width, w.d_state, ss.OP_FORWARD, w.torch_dtype)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    y = torch.empty((w.batch, w.dim, w.height, w.width), dtype=w.torch_dtype, device=dev)

    def step():
        for k in keys:
            devbuf[k].copy_(host[k], non_blocking=True)
        ss.ss2d_forward(devbuf["x"], devbuf["delta"], devbuf["A"], devbuf["B"], devbuf["C"], devbuf["D"],
                        devbuf["delta_bias"], True, out=y, workspace=ws)
        y_host.copy_(y, non_blocking=True)

    steps = max(1, min(args.steps, 5))
    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    b = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    b.record(stream)
    for _ in range(steps):
        step()
    e.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(b.elapsed_time(e) / steps, world)
    units = sum_over_ranks(float(w.updates), world)
    return {"value": units / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms, "steps": steps}


def run_reference(args, world, rank):
    w = ss2d_inputs.workload(args.workload)
    # a step is a slice of REFERENCE_ITEMS_PER_STEP whole batch items (about half a second of oracle time
    # for VMamba-T stage 1), so the default --steps/--warmup run takes well under a minute
    base = time_oracle(w, steps=args.steps, warmup=args.warmup, items_per_step=REFERENCE_ITEMS_PER_STEP)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": base["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": base["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded; VMamba init recipe for A, D, delta_bias)",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "dim": w.dim, "height": w.height,
                   "width": w.width, "d_state": w.d_state, "paths": 4},
        "cpu_baseline": {"value": base["value"], "unit": UNIT, "cores": base["cores"], "kind": "oracle",
                         "sample": base["sample"]},
        "e2e": {"value": base["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=1, help="index into ss2d_inputs.WORKLOADS (default 1)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (small cases for profiling; not a bench line)")
    ap.add_argument("--impl", choices=["ss2d", "reference"], default="ss2d")
    ap.add_argument("--backward", action="store_true",
                    help="time forward (keeping chunk states) + fused backward per step")
    ap.add_argument("--gate", action="store_true",
                    help="time the sequence-form scan with the output gate z and the last state instead")
    ap.add_argument("--paths", choices=["cross", "diagonal"], default="cross",
                    help="path set of the fused SS2D (default: the cross scan)")
    ap.add_argument("--conv", type=int, default=0, metavar="D_CONV",
                    help="with --proj: put the per-path causal depthwise conv (width D_CONV, SiLU) in front")
    ap.add_argument("--proj", action="store_true",
                    help="time the fused forward with its per-path x_proj/dt_proj producer instead")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="time budget of the CPU oracle sample")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps(run_reference(args, world, rank)), flush=True)
            return 0
        result = run_gpu(args, world, rank, local)
        if rank == 0:
            print(json.dumps(result), flush=True)
        return 0
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
