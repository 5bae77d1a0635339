#!/usr/bin/env python
"""Throughput of the Gated DeltaNet-2 forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one chunked GDN-2 forward (every chunk-path row: TMA loads,
cumulative log-decay, operand build, the A/B/QX/QP GEMM, (I+A)^-1, the W/U
GEMMs, the state scan and the output epilogue) over the full GDN-2 workload:
8 sequences x 4096 tokens x 16 heads x 128, bf16 inputs, fp32 state, chunk 64,
channel-wise decay and decoupled channel-wise gates, S0 ~ N(0, 0.02).  Inputs
(0.96 GB) are resident in HBM and larger than L2.  `value` is prefill
tokens/s over all ranks (weak scaling: every rank runs its own batch; the
units shard with no data-path collective).

With --gpus N > 1 the script runs one rank per GPU: launched by torchrun it
checks that WORLD_SIZE equals N; launched plainly it starts the N ranks itself
through torch.distributed.run (rendezvous on 127.0.0.1).  Times are CUDA-event
times on each rank, reported as the maximum over ranks; rank 0 prints.

`configs` times the other prefill workloads on the same line: the tied
scalar-gate Gated DeltaNet batch (4 x 4096 x 16) and the packed varlen batch
(16 sequences of 4k-64k tokens, 524,288 in total), each with its roofline.

The same JSON line carries `decode`: 1024 recurrent decode steps over 256
sequences x 16 heads with a 268 MB fp32 state built by a 2048-token chunked
prefill (tokens/s and fraction of HBM bandwidth), the roofline of the chunk
kernel, the end-to-end number through host buffers, the float64 CPU oracle as
`cpu_baseline`, and the SM clocks sampled while timing.

`bwd` times gdn2_chunk_bwd (all gradients of the forward: a checkpointing
chunked forward, then the chunked reverse pass on the tensor cores) on the
prefill workload with random bf16 dO and dS_T; `bwd.token_serial` times the
fp32 token-serial gdn2_bwd on the same inputs once, for comparison.

`--impl reference` times the float64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import atexit
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s (GDN-2 fwd, 16h×128d, T=4k); decode tok/s, % HBM BW"
WORKLOAD = "gdn2_b8_t4k"
# tcgen05 GEMMs the chunk kernel issues per token-head (C=64, d=128):
# G1 8*C*dk + R 2*C*dv + 2*dk*dv + M 2*C*dv + O 2*dk*dv + 4*C*dv + dS 4*dk*dv
FLOP_PER_TOKHEAD = 8 * 64 * 128 + 8 * 64 * 128 + 8 * 128 * 128
# with x_r == p_r (tied gates) the first GEMM runs at N = 64: 4 C dk instead of 8 C dk
FLOP_PER_TOKHEAD_TIED = FLOP_PER_TOKHEAD - 4 * 64 * 128
BYTES_PER_TOKHEAD = 6 * 128 * 2 + 128 * 2                      # six bf16 inputs + bf16 o
BYTES_PER_TOKHEAD_SCALAR = 3 * 128 * 2 + 2 * 2 + 128 * 2       # q, k, v + scalar alpha, beta + o
STATE_BYTES = 128 * 128 * 4                                    # one fp32 state
# fp32 operations of the token-serial backward per token-head (d_k = d_v = 128): per
# state element, the forward sweep and the block recompute take 7 each (decay, erase
# read, erase and write updates) and the reverse step 26.
BWD_FLOP_PER_TOKHEAD = (7 + 7 + 26) * 128 * 128
# tcgen05 products of the chunked backward per chunk-head (C = 64, d = 128): G1 128x128x128,
# dM 128x64x(128 + 64), R 128x64x192, M and dR 128x64x64 each, [dA dB; dQX dQP], the adjoint
# update and the S_r terms of dk_r, dq_r 128x128x128 each, dV 128x64x256, [dx_r | dp_r]
# 128x128x256, the rest of dk_r, dq_r 128x128x128; per token-head, plus the checkpointing
# forward's products.
CBWD_FLOP_PER_TOKHEAD = 2 * (128 * 128 * 128 * 5 + 128 * 64 * (192 + 192 + 64 + 64 + 256)
                             + 128 * 128 * 256) // 64 + FLOP_PER_TOKHEAD
# DRAM bytes of one gdn2_chunk_bwd per token-head: the forward reads the six bf16 inputs and
# writes the checkpoint (bf16 S_r and T tiles, 40 KB per 64 tokens); the reverse pass reads the
# six inputs, dO and the checkpoint and writes six bf16 gradients (final states and dS_T, dS0
# per sequence are not counted)
CBWD_BYTES_PER_TOKHEAD = 6 * 256 + 640 + (7 * 256 + 640) + 6 * 256
# the tied scalar-gate batch: q, k, v (and dO, dq, dk, dv) per channel, log_a and b per token
CBWD_BYTES_PER_TOKHEAD_SCALAR = (3 * 256 + 4) + 640 + (4 * 256 + 4 + 640) + (3 * 256 + 4)


def fp32_peak_tflops(sm_max_mhz: float) -> float:
    """CUDA-core fp32 peak: 148 SMs x 128 FMA lanes x 2 flops x the max SM clock."""
    return 148 * 128 * 2 * sm_max_mhz * 1e6 / 1e12


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def kernel_sha() -> str:
    h = hashlib.sha256()
    for f in ("chunk_tc.cu", "sm100_ptx.cuh", "common.cuh", "tc_util.cuh"):
        with open(os.path.join(ROOT, "gated_delta_rule_159_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def bwd_kernel_sha() -> str:
    h = hashlib.sha256()
    for f in ("chunk_tc.cu", "bwd_tc.cu", "sm100_ptx.cuh", "common.cuh", "tc_util.cuh"):
        with open(os.path.join(ROOT, "gated_delta_rule_159_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def bwd_traffic_per_call():
    """DRAM bytes of one gdn2_chunk_bwd call on the bench workload (both kernels) from the
    committed ncu summary, if it was taken on the current kernel sources (else None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "chunk_bwd_traffic.json")) as f:
            t = json.load(f)
        if t.get("kernel_sha") == bwd_kernel_sha():
            return t["bytes_per_call_full_workload"]
    except Exception:
        pass
    return None


def traffic_per_launch():
    """DRAM bytes per chunk-kernel launch from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "chunk_tc_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        if t.get("kernel_sha") == kernel_sha():
            return t["bytes_per_launch_full_workload"]
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons every 200 ms for the whole run.  It starts
    before the first timed region, so its own start-up (process launch, NVML
    initialisation) runs beside untimed work; each timed region then takes the samples
    around it (``stats``)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.file = None
        self.samples = []  # (host time, SM MHz, max SM MHz, active reasons)

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu_index), "-lms", "200"], stdout=self.file,
                                         stderr=subprocess.DEVNULL)
            atexit.register(self.kill)  # an exception between start and stop must not leave it running
        except Exception:
            self.proc = None

    def kill(self):
        if self.proc is not None and self.proc.poll() is None:
            self.proc.kill()

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        self.proc = None
        for r in rows:
            try:
                mhz, mx = float(r[2]), float(r[3])
                reasons = {nm for nm, val in zip(self.REASONS, r[6:10]) if val.strip().lower() == "active"}
            except (ValueError, IndexError):
                continue
            try:
                t = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                t = None  # an unreadable timestamp: the sample counts for every region
            self.samples.append((t, mhz, mx, reasons))

    def stats(self, t0: float, t1: float, margin: float = 0.25):
        """Median SM clock, max clock and the active reasons of the samples taken from
        ``margin`` seconds before host time ``t0`` to ``margin`` after ``t1`` (the two
        samples nearest the region if none falls inside)."""
        if not self.samples:
            return None
        sel = [x for x in self.samples if x[0] is None or t0 - margin <= x[0] <= t1 + margin]
        if not sel:
            mid = 0.5 * (t0 + t1)
            sel = sorted(self.samples, key=lambda x: abs(x[0] - mid))[:2]
        return {"sm_mhz": statistics.median(x[1] for x in sel), "sm_max_mhz": max(x[2] for x in sel),
                "reasons": sorted(set().union(*(x[3] for x in sel))), "samples": len(sel)}


# ----------------------------------------------------------------------------- ranks
def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def ensure_ranks(gpus: int, argv, script: str):
    """One process per GPU.  Under torchrun (WORLD_SIZE set) the world size must equal
    ``gpus``.  Without it and with ``gpus`` > 1, start ``gpus`` ranks of this same command
    through torch.distributed.run (rendezvous on 127.0.0.1) and return their exit status;
    otherwise return None and let the caller run as the only rank."""
    ws = os.environ.get("WORLD_SIZE")
    if ws is not None:
        if int(ws) != gpus:
            raise SystemExit(f"WORLD_SIZE={ws} but --gpus {gpus}: run one rank per GPU")
        return None
    if gpus <= 1:
        return None
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}", script, *argv]
    return subprocess.call(cmd)


def rank_env():
    """(world, rank, local rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device) -> float:
    """The maximum of ``x`` over all ranks (a device-side time is reported as its max)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def emit(line: dict, rank: int):
    """Rank 0 prints the one JSON line."""
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(inp, max_seconds: float, n_units: int = 0):
    """Time the float64 oracle on whole (sequence, head) units of the workload,
    as many as fit ~max_seconds of wall time on this host (all cores), or
    exactly ``n_units`` units when given."""
    import oracle
    import torch
    T = inp["T_tot"] // inp["n_seqs"]
    H = inp["q"].shape[1]
    threads = oracle.max_threads()
    units_all = [(n, h) for n in range(inp["n_seqs"]) for h in range(H)]

    def run(units):
        sl = lambda t, n, h: t[n * T:(n + 1) * T, h:h + 1].float().cpu().numpy().astype(np.float64)  # noqa: E731
        cat = {name: np.concatenate([sl(inp[name], n, h) for (n, h) in units])
               for name in ("q", "k", "v", "log_a", "b", "w")}
        S0 = np.stack([inp["S0"][n, h:h + 1].cpu().numpy().astype(np.float64) for (n, h) in units])
        cu = np.arange(len(units) + 1, dtype=np.int64) * T
        t0 = time.perf_counter()
        oracle.gdn2_fwd(cat["q"], cat["k"], cat["v"], cat["log_a"], cat["b"], cat["w"], S0=S0, cu_seqlens=cu,
                        n_threads=threads)
        return time.perf_counter() - t0

    n0 = min(len(units_all), threads)
    if n_units:
        units = units_all[:n_units]
        dt = run(units)
    else:
        # calibrate on one unit per thread, then size the sample
        dt0 = run(units_all[:n0])
        per_batch = max(dt0, 1e-3)
        batches = max(1, min(int(max_seconds / per_batch), math.ceil(len(units_all) / n0)))
        units = units_all[:min(len(units_all), batches * n0)]
        dt = run(units) if len(units) > n0 else dt0
    tokens = len(units) * T / H  # tokens of the metric (a token carries all H heads)
    return {"value": tokens / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(units)} of {len(units_all)} (sequence, head) units x {T} tokens of {WORKLOAD}, "
                      f"float64 C recurrence, {threads} OpenMP threads, {dt:.1f} s",
            "seconds": dt, "n_units": len(units)}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    import torch
    _, rank, _ = rank_env()
    if rank != 0:
        return 0
    from gated_delta_rule_159_b200 import inputs
    inp = inputs.make_inputs(WORKLOAD, "cuda" if torch.cuda.is_available() else "cpu", seed=0)
    per_step = []
    cb = oracle_sample(inp, max_seconds=args.reference_step_seconds)  # sizes the per-step sample
    for i in range(args.warmup + args.steps):
        r = oracle_sample(inp, 0.0, n_units=cb["n_units"])
        if i >= args.warmup:
            per_step.append(r)
        cb = r
    vals = [r["value"] for r in per_step]
    secs = [r["seconds"] for r in per_step]
    value = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(inp, None),
            "cpu_baseline": {k: cb[k] for k in ("unit", "cores", "kind", "sample")} | {"value": value},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_block(inp, world):
    w = inp["workload"]
    return {"workload": w.name, "batch": inp["n_seqs"], "seq_len": inp["T_tot"] // inp["n_seqs"],
            "heads": w.n_heads, "d_k": w.d_k, "d_v": w.d_v, "chunk": w.chunk,
            "gates": "channel-wise decay, decoupled channel-wise erase/write",
            "tokens_per_step_per_gpu": inp["T_tot"], "l2": "inputs_exceed_l2",
            "parallelism": f"dp{world}" if world else "cpu"}


# ----------------------------------------------------------------------------- our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-step-seconds", type=float, default=6.0)
    ap.add_argument("--batch", type=int, default=0, help="override the batch size (small profiling cases)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--bwd-steps", type=int, default=10)
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-token-serial-bwd", action="store_true",
                    help="skip the one timed step of the token-serial gdn2_bwd")
    ap.add_argument("--no-long", action="store_true")
    ap.add_argument("--split", type=int, default=0,
                    help="segments per sequence of the long-context split forward (0: as many as keep "
                         "the 16 heads' segments within the SM count)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--config-steps", type=int, default=5)
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    rc = ensure_ranks(args.gpus, sys.argv[1:], os.path.abspath(__file__))
    if rc is not None:
        return rc

    import torch
    import torch.distributed as dist

    world, rank, local = rank_env()
    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    from gated_delta_rule_159_b200 import gdn2, inputs

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def rmax(x: float) -> float:
        return max_over_ranks(x, world, dev)

    hbm_peak, tc_peak, peak_src = peaks()
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()

    # ---------------- prefill (the step)
    inp = inputs.make_inputs(WORKLOAD, dev, seed=rank, n_seqs=args.batch or None)
    N, T_tot = inp["n_seqs"], inp["T_tot"]
    T = T_tot // N
    names = ("q", "k", "v", "log_a", "b", "w")
    args4 = [inp[n].view(N, T, *inp[n].shape[1:]) for n in names]
    o = torch.empty(N, T, 16, 128, dtype=torch.bfloat16, device=dev)
    ST = torch.empty(N, 16, 128, 128, dtype=torch.float32, device=dev)
    dims = gdn2.make_dims(N, T, 16, 128, 128, 64, gdn2.BF16, gdn2.BF16, 0)
    ws = torch.empty(gdn2.workspace_size(dims), dtype=torch.uint8, device=dev)

    def step():
        gdn2.chunk_fwd(*args4, inp["S0"], None, o=o, S_T=ST, workspace=ws)

    for _ in range(args.warmup):
        step()
    barrier()
    stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    w_prefill = time.time()
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    barrier()
    w_prefill = (w_prefill, time.time())
    total_ms = ev[0][0].elapsed_time(ev[-1][1])
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = rmax(total_ms)
    status = gdn2.check_status(ws)
    if status != gdn2.OK:
        raise RuntimeError(f"chunk kernel reported device status {status}")
    tokens_all = T_tot * world * args.steps
    value = tokens_all / (total_ms / 1e3)
    ms_per_step = total_ms / args.steps

    avg_launch_s = statistics.mean(launch_ms) / 1e3
    units = N * 16
    alg_bytes = BYTES_PER_TOKHEAD * T_tot * 16 + 2 * units * STATE_BYTES
    alg_flops = FLOP_PER_TOKHEAD * T_tot * 16
    achieved = alg_bytes / avg_launch_s / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                "traffic": traffic_per_launch(), "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
                "kernel": "chunk_tc_kernel", "alg_bytes_per_launch": alg_bytes,
                "avg_launch_ms": avg_launch_s * 1e3,
                "tensor_tflops": alg_flops / avg_launch_s / 1e12,
                "tensor_frac": alg_flops / avg_launch_s / 1e12 / tc_peak,
                "tensor_peak": tc_peak, "alg_flops_per_launch": alg_flops}

    # ---------------- end to end through host buffers (pinned), same workload
    e2e = None
    if not args.no_e2e:
        # Pipelined over two buffer sets: step i+1's inputs go host -> device on one stream
        # while step i computes and its o and S_T go device -> host on another (the host
        # link is full duplex); every step still moves its own inputs and results.
        host = {n: args4[i].cpu().pin_memory() for i, n in enumerate(names)}
        S0_h = inp["S0"].cpu().pin_memory()
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        ST_h = torch.empty(ST.shape, dtype=ST.dtype).pin_memory()
        dev_in = [{n: torch.empty_like(args4[i]) for i, n in enumerate(names)} for _ in range(2)]
        S0_d = [torch.empty_like(inp["S0"]) for _ in range(2)]
        o_d = [torch.empty_like(o) for _ in range(2)]
        ST_d = [torch.empty_like(ST) for _ in range(2)]
        ws_d = [torch.empty_like(ws) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}

        def e2e_run(steps, start_event=None):
            if start_event is not None:
                s_in.wait_event(start_event)
            for i in range(steps):
                b = i % 2
                with torch.cuda.stream(s_in):
                    s_in.wait_event(ev["comp"][b])  # the forward that read buffer b is done
                    for n in names:
                        dev_in[b][n].copy_(host[n], non_blocking=True)
                    S0_d[b].copy_(S0_h, non_blocking=True)
                    ev["in"][b].record(s_in)
                stream.wait_event(ev["in"][b])
                stream.wait_event(ev["out"][b])  # o_d[b] has been read back
                gdn2.chunk_fwd(*(dev_in[b][n] for n in names), S0_d[b], None, o=o_d[b], S_T=ST_d[b],
                               workspace=ws_d[b])
                ev["comp"][b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev["comp"][b])
                    o_h.copy_(o_d[b], non_blocking=True)
                    ST_h.copy_(ST_d[b], non_blocking=True)
                    ev["out"][b].record(s_out)
            stream.wait_stream(s_out)

        e2e_run(2)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(args.e2e_steps, start_event=e0)
        e1.record(stream)
        barrier()
        e2e_ms = rmax(e0.elapsed_time(e1))
        h2d = sum(t.numel() * t.element_size() for t in host.values()) + S0_h.numel() * 4
        d2h = o_h.numel() * o_h.element_size() + ST_h.numel() * 4
        e2e = {"value": T_tot * world * args.e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "ms_per_step": e2e_ms / args.e2e_steps,
               "path": "pinned host -> device copies, gdn2_chunk_fwd via the Python binding, o and S_T back; "
                       "two buffer sets, copies of the next step overlap this step's compute and read-back"}
        del host, dev_in, o_h, ST_h, o_d, ST_d, ws_d, S0_d

    # ---------------- CPU baseline (rank 0, one GPU only)
    cpu = None
    if not args.no_cpu and world == 1 and rank == 0:
        cpu = oracle_sample(inp, args.cpu_seconds)
        cpu.pop("seconds")
        cpu.pop("n_units")

    cfg = config_block(inp, world)
    del inp, args4
    torch.cuda.empty_cache()

    # ---------------- the other prefill workloads: tied scalar-gate Gated DeltaNet (4 x 4096 x 16)
    # and the packed varlen long-context batch (16 sequences of 4k-64k tokens, 524,288 in total)
    configs = None
    if not args.no_configs:
        configs = {}
        for wname in ("gdn_scalar_b4_t4k", "gdn2_varlen_16x4k-64k"):
            ci = inputs.make_inputs(wname, dev, seed=600 + rank)
            wl = ci["workload"]
            Nc, Tc = ci["n_seqs"], ci["T_tot"]
            kw = dict(scalar_decay=ci["scalar_decay"], scalar_gates=ci["scalar_gates"], tied_gates=ci["tied_gates"])
            if ci["equal_lengths"]:
                cargs = [None if ci[n] is None else ci[n].view(Nc, Tc // Nc, *ci[n].shape[1:]) for n in names]
                cu, cu_h = None, None
            else:
                cargs = [ci[n] for n in names]
                cu, cu_h = ci["cu_seqlens"], ci["cu_host"]
            co = torch.empty(*cargs[2].shape, dtype=torch.bfloat16, device=dev)
            cS = torch.empty(Nc, 16, 128, 128, dtype=torch.float32, device=dev)
            cdims = gdn2.make_dims(Nc, Tc if cu is not None else Tc // Nc, 16, 128, 128, 64, gdn2.BF16, gdn2.BF16,
                                   gdn2.flags_of(**kw))
            cws = torch.empty(gdn2.workspace_size(cdims), dtype=torch.uint8, device=dev)

            def cstep():
                gdn2.chunk_fwd(*cargs, ci["S0"], cu, cu_seqlens_host=cu_h, o=co, S_T=cS, workspace=cws, **kw)

            for _ in range(args.warmup):
                cstep()
            barrier()
            reps = args.config_steps
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(reps):
                cstep()
            a1.record(stream)
            barrier()
            cms = rmax(a0.elapsed_time(a1)) / reps
            if gdn2.check_status(cws) != gdn2.OK:
                raise RuntimeError(f"chunk kernel reported a timed-out wait ({wname})")
            tokheads = Tc * 16
            units_c = Nc * 16
            per_tok = BYTES_PER_TOKHEAD_SCALAR if wl.scalar_gates else BYTES_PER_TOKHEAD
            states = (2 if ci["S0"] is not None else 1) * units_c * STATE_BYTES
            cbytes = per_tok * tokheads + states
            cflops = (FLOP_PER_TOKHEAD_TIED if ci["tied_gates"] else FLOP_PER_TOKHEAD) * tokheads
            gbs = cbytes / (cms / 1e3) / 1e9
            tfs = cflops / (cms / 1e3) / 1e12
            bound = "hbm" if cbytes / (hbm_peak * 1e9) >= cflops / (tc_peak * 1e12) else "tensor"
            configs[wname] = {
                "ms": cms, "value": Tc * world / (cms / 1e3), "unit": "tokens/s", "steps": reps,
                "sequences": Nc, "tokens": Tc, "units": units_c,
                "gates": "tied scalar alpha, beta (b = w = beta 1)" if wl.scalar_gates else
                         "channel-wise decay, decoupled channel-wise erase/write",
                "roofline": {"bound": bound, "achieved": gbs if bound == "hbm" else tfs,
                             "peak": hbm_peak if bound == "hbm" else tc_peak,
                             "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
                             "frac": gbs / hbm_peak if bound == "hbm" else tfs / tc_peak,
                             "hbm_frac": gbs / hbm_peak, "tensor_frac": tfs / tc_peak,
                             "alg_bytes_per_launch": cbytes, "alg_flops_per_launch": cflops,
                             "traffic": None, "peak_source": peak_src}}
            del ci, cargs, co, cS, cws
            torch.cuda.empty_cache()

    # ---------------- decode
    decode = None
    launches = args.steps  # one chunk_tc_kernel launch per timed prefill step
    if not args.no_decode:
        dc = inputs.DECODE
        Nd, Hd, d, steps = dc["n_seqs"], dc["n_heads"], dc["d"], args.decode_steps
        wpre = inputs.Workload("decode_prefill", Nd, dc["prefill_len"], Hd, d, d, 64, torch.bfloat16, 0.05, False, 0.0)
        pre = inputs.make_inputs(wpre, dev, seed=100 + rank)
        _, S = gdn2.chunk_fwd(*(pre[n].view(Nd, dc["prefill_len"], *pre[n].shape[1:]) for n in names), None, None)
        del pre
        torch.cuda.empty_cache()
        di = inputs.make_decode_inputs(Nd, Hd, d, steps, dev, seed=200 + rank)
        od = torch.empty(Nd, Hd, d, dtype=torch.float32, device=dev)
        for t in range(3):
            gdn2.decode_step(*(di[n][t] for n in names), S, o=od)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        w_decode = time.time()
        e0.record(stream)
        for t in range(steps):
            gdn2.decode_step(*(di[n][t] for n in names), S, o=od)
        e1.record(stream)
        barrier()
        plain_ms = rmax(e0.elapsed_time(e1))
        # The same steps captured once as a CUDA graph and replayed: one graph launch
        # per decode loop, so the per-step host launch gap leaves the timed region.
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for t in range(steps):
                gdn2.decode_step(*(di[n][t] for n in names), S, o=od)
        graph.replay()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        barrier()
        w_decode = (w_decode, time.time())
        dms = rmax(e0.elapsed_time(e1))
        del graph
        if gdn2.decode_status() != gdn2.OK:
            raise RuntimeError("decode kernel reported a timed-out wait")
        step_bytes = 2 * Nd * Hd * d * d * 4 + 6 * Nd * Hd * d * 2 + Nd * Hd * d * 4
        gbs = step_bytes * steps / (dms / 1e3) / 1e9

        def decode_variant(fn, reps, vec_bytes):
            """Plain launch loop of `reps` steps of fn(t); returns (us per step, HBM fraction)."""
            for t in range(3):
                fn(t)
            barrier()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for t in range(reps):
                fn(t)
            a1.record(stream)
            barrier()
            ms = rmax(a0.elapsed_time(a1))
            vb = 2 * Nd * Hd * d * d * 4 + vec_bytes + Nd * Hd * d * 4
            return 1e3 * ms / reps, vb * reps / (ms / 1e3) / 1e9 / hbm_peak

        # continuous batching: the same 256 x 16 rows read and update slots of a pool of 512
        # sequences' states through a shuffled slot index
        reps_v = min(steps, 256)
        pool = torch.zeros(2 * Nd, Hd, d, d, dtype=torch.float32, device=dev)
        gperm = torch.Generator(device="cpu")
        gperm.manual_seed(700 + rank)
        slots = torch.randperm(2 * Nd, generator=gperm)[:Nd].to(torch.int32).to(dev)
        pool[slots.long()] = S
        idx_us, idx_frac = decode_variant(
            lambda t: gdn2.decode_step_indexed(*(di[n][t] for n in names), pool, slots, o=od), reps_v,
            6 * Nd * Hd * d * 2)
        del pool
        # the scalar-gate Gated DeltaNet decode (one alpha and one beta per row, b = w = beta)
        sc_la = di["log_a"][:, :, :, 0].contiguous()
        sc_b = di["b"][:, :, :, 0].contiguous()
        sc_us, sc_frac = decode_variant(
            lambda t: gdn2.decode_step(di["q"][t], di["k"][t], di["v"][t], sc_la[t], sc_b[t], None, S, o=od,
                                       scalar_decay=True, scalar_gates=True, tied_gates=True), reps_v,
            3 * Nd * Hd * d * 2 + 2 * Nd * Hd * 2)
        del sc_la, sc_b
        decode = {"value": Nd * world * steps / (dms / 1e3), "unit": "tokens/s", "steps": steps,
                  "us_per_step": 1e3 * dms / steps, "bytes_per_step": step_bytes, "hbm_gbs": gbs,
                  "hbm_frac": gbs / hbm_peak, "peak_source": peak_src, "sequences": Nd, "heads": Hd,
                  "state_bytes": Nd * Hd * d * d * 4, "clocks": w_decode, "kernel": "decode_stream_kernel",
                  "launch": "CUDA graph of all steps, replayed once",
                  "plain_loop_us_per_step": 1e3 * plain_ms / steps,
                  "gpu_launches": steps,
                  "indexed": {"us_per_step": idx_us, "hbm_frac": idx_frac, "steps": reps_v,
                              "rows": f"{Nd} x {Hd} rows into a pool of {2 * Nd} x {Hd} states, shuffled slots",
                              "kernel": "decode_stream_kernel", "launch": "plain loop"},
                  "scalar_gates": {"us_per_step": sc_us, "hbm_frac": sc_frac, "steps": reps_v,
                                   "gates": "scalar alpha and tied scalar beta per row",
                                   "kernel": "decode_stream_kernel", "launch": "plain loop"}}
        del di, S

    # ---------------- backward (gradients of the prefill step)
    bwd = None
    if not args.no_bwd:
        bi = inputs.make_inputs(WORKLOAD, dev, seed=300 + rank, n_seqs=args.batch or None)
        Nb, Tb = bi["n_seqs"], bi["T_tot"] // bi["n_seqs"]
        gen = torch.Generator(device=dev)
        gen.manual_seed(400 + rank)
        dO = torch.randn(Nb, Tb, 16, 128, generator=gen, device=dev).to(torch.bfloat16)
        dS_T = torch.randn(Nb, 16, 128, 128, generator=gen, device=dev) * 0.1
        bargs = [bi[n].view(Nb, Tb, *bi[n].shape[1:]) for n in names]
        bdims = gdn2.make_dims(Nb, Tb, 16, 128, 128, 64, gdn2.BF16, gdn2.BF16, 0)
        cws = torch.empty(gdn2.chunk_bwd_workspace_size(bdims), dtype=torch.uint8, device=dev)

        def cstep():
            return gdn2.chunk_bwd(*bargs, dO, S0=bi["S0"], dS_T=dS_T, workspace=cws)

        for _ in range(3):
            cstep()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w_bwd = time.time()
        e0.record(stream)
        for _ in range(args.bwd_steps):
            cstep()
        e1.record(stream)
        barrier()
        w_bwd = (w_bwd, time.time())
        cms = rmax(e0.elapsed_time(e1)) / args.bwd_steps
        st = gdn2.lib.gdn2_check_status(gdn2._ptr(cws), gdn2._stream(dev))
        tokheads = Nb * Tb * 16
        gbs = CBWD_BYTES_PER_TOKHEAD * tokheads / (cms / 1e3) / 1e9
        ctf = CBWD_FLOP_PER_TOKHEAD * tokheads / (cms / 1e3) / 1e12
        bwd = {"value": Nb * Tb * world / (cms / 1e3), "unit": "tokens/s", "ms_per_step": cms,
               "steps": args.bwd_steps, "status": st,
               "dtype": "bf16 operands, fp32 accumulation (tcgen05), bf16 gradients",
               "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                            "traffic": bwd_traffic_per_call() if Nb == 8 else None, "peak_source": peak_src,
                            "alg_bytes_per_tokhead": CBWD_BYTES_PER_TOKHEAD,
                            "scope": "whole gdn2_chunk_bwd call (checkpointing forward + reverse pass)"},
               "tensor": {"achieved": ctf, "peak": tc_peak, "unit": "TFLOP/s", "frac": ctf / tc_peak,
                          "alg_flops_per_tokhead": CBWD_FLOP_PER_TOKHEAD},
               "kernels": ["chunk_tc_kernel (checkpointing forward)", "bwd_tc_kernel"],
               "gpu_launches": 2 * args.bwd_steps, "workspace_bytes": cws.numel(), "clocks": w_bwd}
        del cws
        # the tied scalar-gate Gated DeltaNet batch (4 x 4096 x 16) through the same backward
        si = inputs.make_inputs("gdn_scalar_b4_t4k", dev, seed=310 + rank)
        Ns, Ts = si["n_seqs"], si["T_tot"] // si["n_seqs"]
        sdO = torch.randn(Ns, Ts, 16, 128, generator=gen, device=dev).to(torch.bfloat16)
        sdS = torch.randn(Ns, 16, 128, 128, generator=gen, device=dev) * 0.1
        sargs = [None if si[n] is None else si[n].view(Ns, Ts, *si[n].shape[1:]) for n in names]
        sdims = gdn2.make_dims(Ns, Ts, 16, 128, 128, 64, gdn2.BF16, gdn2.BF16,
                               gdn2.SCALAR_DECAY | gdn2.SCALAR_GATES | gdn2.TIED_GATES)
        sws = torch.empty(gdn2.chunk_bwd_workspace_size(sdims), dtype=torch.uint8, device=dev)

        def sstep():
            return gdn2.chunk_bwd(*sargs, sdO, S0=si["S0"], dS_T=sdS, scalar_decay=True, scalar_gates=True,
                                  tied_gates=True, workspace=sws)

        for _ in range(3):
            sstep()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(args.bwd_steps):
            sstep()
        e1.record(stream)
        barrier()
        sms = rmax(e0.elapsed_time(e1)) / args.bwd_steps
        sst = gdn2.lib.gdn2_check_status(gdn2._ptr(sws), gdn2._stream(dev))
        sgbs = CBWD_BYTES_PER_TOKHEAD_SCALAR * Ns * Ts * 16 / (sms / 1e3) / 1e9
        bwd["gdn_scalar_b4_t4k"] = {
            "value": Ns * Ts * world / (sms / 1e3), "unit": "tokens/s", "ms_per_step": sms, "status": sst,
            "gates": "scalar alpha, tied scalar beta (Gated DeltaNet)",
            "roofline": {"bound": "hbm", "achieved": sgbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": sgbs / hbm_peak, "traffic": None, "peak_source": peak_src,
                         "alg_bytes_per_tokhead": CBWD_BYTES_PER_TOKHEAD_SCALAR},
            "units": Ns * 16, "workspace_bytes": sws.numel()}
        del si, sdO, sdS, sargs, sws
        if not args.no_token_serial_bwd:
            bws = torch.empty(gdn2.bwd_workspace_size(bdims), dtype=torch.uint8, device=dev)

            def bstep():
                return gdn2.bwd(*bargs, dO, S0=bi["S0"], dS_T=dS_T, workspace=bws)

            bstep()
            torch.cuda.synchronize()
            barrier()
            e0.record(stream)
            bstep()
            e1.record(stream)
            barrier()
            bms = rmax(e0.elapsed_time(e1))
            tflops = BWD_FLOP_PER_TOKHEAD * tokheads / (bms / 1e3) / 1e12
            bwd["token_serial"] = {
                "value": Nb * Tb * world / (bms / 1e3), "unit": "tokens/s", "ms_per_step": bms, "steps": 1,
                "dtype": "f32 arithmetic, bf16 inputs and gradients",
                "roofline": {"bound": "alu", "achieved": tflops, "peak": None, "unit": "TFLOP/s",
                             "frac": None, "traffic": None,
                             "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x sm_max_mhz",
                             "alg_flops_per_tokhead": BWD_FLOP_PER_TOKHEAD},
                "kernels": ["bwd_kernel", "finish_kernel"], "workspace_bytes": bws.numel()}
            del bws
        del bi, dO, dS_T, bargs

    # ---------------- long context: one sequence of 65,536 tokens, 16 heads (16 units on 148
    # SMs), plain chunked forward against the sequence-parallel split forward
    long_ctx = None
    if not args.no_long:
        wl = inputs.Workload("long_b1_t64k", 1, 65536, 16, 128, 128, 64, torch.bfloat16, 0.05, False, 0.02)
        li = inputs.make_inputs(wl, dev, seed=500 + rank)
        largs = [li[n].view(1, 65536, *li[n].shape[1:]) for n in names]
        ldims = gdn2.make_dims(1, 65536, 16, 128, 128, 64, gdn2.BF16, gdn2.BF16, 0)
        if args.split <= 0:  # one segment unit per SM at most: 148 SMs / 16 heads -> 9 segments
            args.split = max(1, torch.cuda.get_device_properties(dev).multi_processor_count // 16)
        lws = torch.empty(gdn2.split_workspace_size(ldims, args.split), dtype=torch.uint8, device=dev)
        pws = torch.empty(gdn2.workspace_size(ldims), dtype=torch.uint8, device=dev)

        def timed(fn, reps=3):
            fn()
            torch.cuda.synchronize()
            barrier()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(reps):
                fn()
            a1.record(stream)
            barrier()
            return rmax(a0.elapsed_time(a1)) / reps

        t_plain = timed(lambda: gdn2.chunk_fwd(*largs, li["S0"], None, workspace=pws))
        t_split = timed(lambda: gdn2.chunk_fwd_split(*largs, li["S0"], n_split=args.split, workspace=lws))
        if gdn2.check_status(lws) != gdn2.OK or gdn2.check_status(pws) != gdn2.OK:
            raise RuntimeError("chunk kernel reported a timed-out wait")
        long_ctx = {"workload": "1 sequence x 65536 tokens x 16 heads x 128, gates as gdn2_b8_t4k",
                    "plain_ms": t_plain, "split_ms": t_split, "n_split": args.split,
                    "plain_tokens_per_s": 65536 * world / (t_plain / 1e3),
                    "split_tokens_per_s": 65536 * world / (t_split / 1e3)}
        if world > 1 and 65536 % world == 0:
            # one 65,536-token sequence spread over the ranks: rank r holds tokens
            # [r L, (r + 1) L), L = 65536 / N; each rank's segment maps are all-gathered
            Lr = 65536 // world
            rargs = [a[:, rank * Lr:(rank + 1) * Lr].contiguous() for a in largs]
            t_ranks = timed(lambda: gdn2.chunk_fwd_seq_ranks(*rargs, li["S0"]))
            long_ctx.update({"ranks_ms": t_ranks, "ranks": world,
                             "ranks_tokens_per_s": 65536 / (t_ranks / 1e3),
                             "ranks_path": "gdn2_segment_maps, all-gather of (F, G) over NCCL, "
                                           "gdn2_affine_prefix, gdn2_segment_correct"})
        del li, largs, lws, pws

    # clocks of each timed region, from the samples taken around it
    sampler.stop()
    clocks = sampler.stats(*w_prefill)
    if decode is not None:
        decode["clocks"] = sampler.stats(*decode["clocks"])
    if bwd is not None:
        bwd["clocks"] = sampler.stats(*bwd["clocks"])
        ts = bwd.get("token_serial")
        if ts is not None:
            peak32 = fp32_peak_tflops((bwd["clocks"] or {}).get("sm_max_mhz") or 1965.0)
            ts["roofline"]["peak"] = peak32
            ts["roofline"]["frac"] = ts["roofline"]["achieved"] / peak32
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; shapes and distributions of the "
                                                          "full GDN-2 workload)",
            "config": cfg, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clocks, "configs": configs, "decode": decode, "bwd": bwd,
            "long_context": long_ctx}
    emit(line, rank)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
