"""Throughput benchmark of the SANA ReLU-linear-attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload sweep|fused|1024px|2048px|4096px] [--no-fused] [--no-cpu]

One step (default workload "sweep") is one pass of the linear-attention op over
each of the SANA latent sizes the metric names (C = 2240, H = 70, D = 32, bf16):
1024px B=1 N=1024, 2048px B=8 N=4096 (per-token LogNormal scales), 4096px B=2
N=16384 (keys x100, norm off).  Each pass runs the op's two halves through the
C ABI (sana_linattn_kv_state: pass 1 + combine, then sana_linattn_apply: pass 2,
exactly the kernels sana_linattn_forward launches) so each half is timed with
CUDA events on its stream.  The fused-QKV variant (2048px B=4, x @ Wqkv first) is
timed in the same run and reported under "fused".

value: tokens of all ranks / device time of the K timed steps (max over ranks).
e2e: the same metric through sana_linattn_forward with host (pinned) buffers,
host->device copies of q, k, v and the device->host copy of the output inside the
timed region; the fused and Mix-FFN legs carry their own e2e (x uploaded, the
output downloaded each step).  cpu_baseline: the fp64 CPU oracle, as it stands, on a bounded
sample of the same workload (rank 0, N=1 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "linear-attn Mtokens/s at C=2240, N=1K–16K; % of B200 HBM roofline"
HBM_FALLBACK_GBS = 6650.0
HBM_NOMINAL_GBS = 8000.0          # B200 HBM3e nominal (DGX figure), for context
BF16_FALLBACK_TFLOPS = 1590.0
# algorithmic bytes per token of each pass (bf16, C = 2240): pass 1 reads k and v,
# pass 2 reads q and writes out; 17,920 B/token for the whole op
PASS_BYTES_PER_TOKEN = 2 * 2240 * 2


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return (float(j["hbm_gbs"]), float(j["bf16_tflops"]),
                float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured")
    except Exception:
        return HBM_FALLBACK_GBS, BF16_FALLBACK_TFLOPS, 1400.0, "fallback"


# ----------------------------------------------------------------------------- workloads
def sweep_workloads():
    from relu_linear_attention_attn_b200.synthetic import WORKLOADS
    return {"1024px": WORKLOADS["1024px-b1"], "2048px": WORKLOADS["2048px-b8-lognormal"], "4096px": WORKLOADS["4096px-b2-overflow"]}


def select(workload: str):
    sw = sweep_workloads()
    if workload == "sweep":
        return list(sw.values())
    if workload in sw:
        return [sw[workload]]
    raise SystemExit(f"unknown workload {workload}")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"sana_bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return None
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except Exception:
            return None
        if not rows:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1])]
        mx = [num(r[2]) for r in rows if num(r[2])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        top = max(sm) if sm else 0
        loaded = [s for s in sm if s >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- distributed
def spawn_ranks_if_needed(args):
    """`--gpus N` with N > 1 runs one process per GPU.  Started without a launcher
    (no WORLD_SIZE in the environment), the script re-executes itself under
    torch.distributed.run with N ranks on this node; started by a launcher, the
    launcher's world size must equal N."""
    world = os.environ.get("WORLD_SIZE")
    if world is None:
        if args.gpus > 1:
            import socket
            with socket.socket() as s:
                s.bind(("127.0.0.1", 0))
                port = s.getsockname()[1]
            cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                   f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
                   "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
            os.execv(sys.executable, cmd)
        return
    if int(world) != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but the launcher started {world} ranks")


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        # NCCL reports its communicator (rank count, transport) at init
        os.environ.setdefault("NCCL_DEBUG", "INFO")
        os.environ.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    from relu_linear_attention_attn_b200.sharding import max_over_ranks as mor
    return x if world == 1 else mor(x, device="cuda")


# the sources the two pass kernels compile from: a recorded ncu traffic figure is
# reported only while these hash to the value stored beside it
KERNEL_SOURCES = ("relu_linear_attention_attn_b200/csrc/tc_kernels.cuh",
                  "relu_linear_attention_attn_b200/csrc/sana_common.cuh",
                  "relu_linear_attention_attn_b200/csrc/sm100_primitives.cuh")


# the sources the Mix-FFN kernels compile from
MIXFFN_SOURCES = ("relu_linear_attention_attn_b200/csrc/mixffn_kernels.cuh",
                  "relu_linear_attention_attn_b200/csrc/sm100_pair.cuh",
                  "relu_linear_attention_attn_b200/csrc/f32x2.cuh",
                  "relu_linear_attention_attn_b200/csrc/tc_kernels.cuh",
                  "relu_linear_attention_attn_b200/csrc/sana_common.cuh",
                  "relu_linear_attention_attn_b200/csrc/sm100_primitives.cuh")


def kernel_source_hash(sources=KERNEL_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str, sources=KERNEL_SOURCES):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu record,
    or None when there is none or the kernel sources changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            rec = json.load(f).get(f"{kernel}@{workload}")
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != kernel_source_hash(sources):
        return None
    return rec["dram_read_bytes"] + rec["dram_write_bytes"]


# ----------------------------------------------------------------------------- CPU oracle
def cpu_oracle_sample(pairs, budget_s: float = 12.0):
    """Time the fp64 oracle as it stands on a bounded sample of the workload: whole
    batch items taken in order until about budget_s of CPU work is done.
    pairs: [(workload, CPU input tensors)]."""
    from oracle import oracle as O
    tokens, t_total, parts = 0, 0.0, []
    for w, x in pairs:
        for b in range(w.B):
            q, k, v = (x[n][b:b + 1] for n in ("q", "k", "v"))
            t0 = time.perf_counter()
            O.forward(q, k, v, x["gq"], x["gk"], w.H, w.eps)
            t_total += time.perf_counter() - t0
            tokens += w.N
            parts.append(f"{w.name}[b={b}]")
            if t_total >= budget_s:
                break
        if t_total >= budget_s:
            break
    # the O(N^2) brute force of Eq. (1), on the tiny workload only
    from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs
    wt = WORKLOADS["tiny-512px-f32"]
    xt = make_inputs(wt)
    reps, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < 0.5:
        O.quadratic_forward(xt["q"], xt["k"], xt["v"], xt["gq"], xt["gk"], wt.H, wt.eps)
        reps += 1
    t_brute = (time.perf_counter() - t0) / reps
    return {"value": tokens / t_total / 1e6, "unit": "Mtokens/s", "cores": O.host_threads(),
            "kind": "oracle", "sample": f"{tokens} tokens ({', '.join(parts)}), fp64 C oracle, "
                                        f"{t_total:.1f} s",
            "brute_force_tiny": {"value": wt.tokens / t_brute / 1e6, "unit": "Mtokens/s",
                                 "workload": wt.name, "kind": "oracle O(N^2) form",
                                 "ms_per_call": t_brute * 1e3}}


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on the host cores, same metric and config."""
    if rank != 0:
        return
    from oracle import oracle as O
    from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs
    if args.workload == "mixffn":
        return run_reference_mixffn(args, O)
    fused = args.workload in ("fused", "w8a8")
    wl = [WORKLOADS["fused-2048px-b4"] if args.workload == "fused" else WORKLOADS["w8a8-2048px-b4"]] if fused else \
        select(args.workload)
    # each step: one whole batch item of every workload in the sweep, bounded so
    # the --steps/--warmup run stays within a few minutes
    data = []
    for w in wl:
        x = make_inputs(w)
        if args.workload == "fused":
            data.append((w, x["x"][:1], x["W"], x["gq"], x["gk"]))
        elif args.workload == "w8a8":
            Wq, sw = O.quantize_i8(x["W"].float().numpy(), axis=0)
            data.append((w, x["x"][:1], (Wq, sw), x["gq"], x["gk"]))
        else:
            data.append((w, x["q"][:1], x["k"][:1], x["v"][:1], x["gq"], x["gk"]))
    per_step_tokens = sum(d[0].N for d in data)

    def step():
        for d in data:
            if args.workload == "fused":
                w, xx, W, gq, gk = d
                O.fused_forward(xx, W, gq, gk, w.H, w.eps)
            elif args.workload == "w8a8":
                w, xx, (Wq, sw), gq, gk = d
                xq, sx = O.quantize_i8(xx.float().numpy())
                O.w8a8_fused_forward(xq, sx, Wq, sw, gq, gk, w.H, w.eps)
            else:
                w, q, k, v, gq, gk = d
                O.forward(q, k, v, gq, gk, w.H, w.eps)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = per_step_tokens * args.steps / dt / 1e6
    sample = (f"one batch item of each workload per step ({per_step_tokens} tokens): "
              + ", ".join(f"{d[0].name} N={d[0].N}" for d in data))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "Mtokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(args, wl, world),
            "cpu_baseline": {"value": value, "unit": "Mtokens/s", "cores": O.host_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "Mtokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def mixffn_cpu_sample():
    """The oracle's Mix-FFN as it stands on a bounded sample (128 tokens of the
    2048px batch of 4, about 10 s of host work)."""
    from oracle import oracle as O
    from relu_linear_attention_attn_b200.synthetic import MIXFFN_WORKLOADS, make_mixffn_inputs
    w = MIXFFN_WORKLOADS["mixffn-2048px-b4"]
    x = make_mixffn_inputs(w)
    f = lambda t: None if t is None else t.float().numpy()
    tok = [(i * 1031) % w.tokens for i in range(128)]
    t0 = time.perf_counter()
    O.mixffn_forward(f(x["x"]), f(x["W1"]), f(x["b1"]), f(x["wdw"]), f(x["bdw"]), f(x["W2"]),
                     f(x["b2"]), w.Hs, w.Ws, w.gate, tokens=tok)
    dt = time.perf_counter() - t0
    return {"value": len(tok) / dt / 1e6, "unit": "Mtokens/s", "cores": O.host_threads(),
            "kind": "oracle", "sample": f"{len(tok)} tokens of {w.name} (3x3 neighbourhoods), "
                                        f"fp64 numpy oracle, {dt:.1f} s"}


def run_reference_mixffn(args, O):
    """The oracle's Mix-FFN on a bounded sample of the 2048px batch of 4: each step
    forms Y for 64 tokens spread over the grids (their 3x3 neighbourhoods' expand,
    the depthwise conv + GLU, the project), in fp64 on the host cores."""
    from relu_linear_attention_attn_b200.synthetic import MIXFFN_WORKLOADS, make_mixffn_inputs
    w = MIXFFN_WORKLOADS["mixffn-2048px-b4"]
    x = make_mixffn_inputs(w)
    f = lambda t: None if t is None else t.float().numpy()
    args_np = (f(x["x"]), f(x["W1"]), f(x["b1"]), f(x["wdw"]), f(x["bdw"]), f(x["W2"]), f(x["b2"]))
    tok = [(i * 1031) % w.tokens for i in range(64)]

    def step():
        O.mixffn_forward(*args_np, w.Hs, w.Ws, w.gate, tokens=tok)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = len(tok) * args.steps / dt / 1e6
    sample = f"64 tokens of {w.name} per step (3x3 neighbourhoods, fp64 oracle)"
    line = {"impl": "reference", "metric": "Mix-FFN tokens per second", "value": value,
            "unit": "Mtokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hs": w.Hs, "Ws": w.Ws, "C": w.C, "F": w.F},
            "cpu_baseline": {"value": value, "unit": "Mtokens/s", "cores": O.host_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "Mtokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def config_block(args, wl, world=1):
    return {"workload": "sana-latent-sweep-N1K-16K" if args.workload == "sweep" else
            args.workload,
            "parts": [{"name": w.name, "B": w.B, "N": w.N, "C": w.C, "H": w.H, "D": w.D,
                       "recipe": w.recipe, "gains": w.gains, "eps": w.eps} for w in wl],
            "global_batch_tokens": sum(w.tokens for w in wl),
            "l2": "inputs larger than L2: one step streams >1.1 GB, so each workload's "
                  "inputs are evicted before they are used again",
            "parallelism": f"dp{world} (batch-sharded, no collective)"}


# ----------------------------------------------------------------------------- our arm
def run_seq_shard(args, sla, rank, world, dev, stream, hbm_gbs):
    """--shard seq: every workload's sequence split over the ranks; each step runs
    sharding.sequence_parallel_forward (per-rank state of its token range through
    sana_linattn_kv_state, one fp32 sum all-reduce of the state over NCCL, then
    sana_linattn_apply on the rank's own queries).  The whole job processes each
    workload once per step, so value = all tokens / step time (strong scaling)."""
    import torch

    from relu_linear_attention_attn_b200 import sharding
    from relu_linear_attention_attn_b200.synthetic import make_inputs
    wl = select(args.workload)
    sets = []
    for w in wl:
        x = make_inputs(w)
        n0, cnt = sharding.token_shard(w.N, rank, world)
        d = {n: x[n][:, n0:n0 + cnt].contiguous().to(dev) for n in ("q", "k", "v")}
        d["gq"] = None if x["gq"] is None else x["gq"].to(dev)
        d["gk"] = None if x["gk"] is None else x["gk"].to(dev)
        sets.append((w, d))

    def step():
        for w, d in sets:
            sharding.sequence_parallel_forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H,
                                               w.eps)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        barrier(world)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world) / args.steps
    tokens = sum(w.tokens for w in wl)
    value = tokens / (ms * 1e-3) / 1e6
    state_bytes = sum(w.B * w.H * w.D * (w.D + 1) * 4 for w in wl)
    line = {"metric": METRIC, "value": value, "unit": "Mtokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_block(args, wl, world) |
            {"parallelism": f"sp{world} (sequence-sharded: per-rank state, one fp32 sum "
                            f"all-reduce of {state_bytes} B per step, per-rank apply)"},
            "launch": "eager sequence_parallel_forward calls (NCCL all-reduce between the passes)",
            "roofline": {"bound": "hbm", "achieved": tokens * 2 * PASS_BYTES_PER_TOKEN / world /
                         (ms * 1e-3) / 1e9, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": tokens * 2 * PASS_BYTES_PER_TOKEN / world / (ms * 1e-3) / 1e9 /
                         hbm_gbs, "traffic": None,
                         "kernel": "the whole op per rank (its token share of q, k, v, out)"},
            "gpu_launches": args.steps * len(wl) * 3, "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local):
    import torch

    import relu_linear_attention_attn_b200 as sla
    from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs

    sla.load()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_kind = measured_peaks()
    if args.shard == "seq":
        if args.workload not in ("sweep", "1024px", "2048px", "4096px"):
            raise SystemExit("--shard seq applies to the attention workloads")
        return run_seq_shard(args, sla, rank, world, dev, stream, hbm_gbs)
    wl = select(args.workload) if args.workload not in ("fused", "w8a8", "mixffn") else []

    # inputs resident in HBM; each rank works on its own batch (weak scaling)
    sets = []
    for w in wl:
        w_r = w.scaled(seed=w.seed + 1000 * rank) if rank else w
        x = make_inputs(w_r)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        D = w.D
        d["kv"] = torch.empty((w.B, w.H, D, D + 1), dtype=torch.float32, device=dev)
        d["out"] = torch.empty_like(d["q"])
        nb = sla.workspace_bytes(w.B, w.N, w.C, w.H)
        d["ws"] = torch.empty(nb, dtype=torch.uint8, device=dev)
        sets.append((w, d, x))
    tokens_per_step = sum(w.tokens for w in wl)

    # a read of 512 MB evicts every input from L2 and leaves it clean (no dirty
    # output of the previous launch left to write back during the timed one)
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush_sink = torch.empty(1, dtype=torch.int64, device=dev)

    def flush():
        torch.sum(flush_buf.view(torch.int64), dim=0, keepdim=True, out=flush_sink)

    def step(events=None):
        """The forward's two kernels as separate calls (sana_linattn_forward_pass1,
        _pass2: exactly the forward), each after an L2 flush and bracketed by
        events."""
        cur = torch.cuda.current_stream(dev)
        for i, (w, d, _) in enumerate(sets):
            flush()
            if events is not None:
                events[i][0].record(cur)
            sla.forward_pass1(d["k"], d["v"], d["gk"], w.H, w.eps, d["ws"])
            if events is not None:
                events[i][1].record(cur)
            flush()
            if events is not None:
                events[i][2].record(cur)
            sla.forward_pass2(d["q"], d["gq"], w.H, w.eps, d["ws"], out=d["out"])
            if events is not None:
                events[i][3].record(cur)

    line = {"metric": METRIC, "unit": "Mtokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_block(args, wl, world)}

    def fwd_step():
        for w, d, _ in sets:
            sla.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps, out=d["out"],
                        workspace=d["ws"])

    if sets:
        for _ in range(args.warmup):
            fwd_step()
            step()
        torch.cuda.synchronize()
        ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in sets]
              for _ in range(args.steps)]
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)

        # (1) value: K steps of sana_linattn_forward (pass 2 chained to pass 1 by
        # programmatic dependent launch), eager and as one CUDA graph of the K steps.
        barrier(world)
        torch.cuda.synchronize()
        t_start.record(stream)
        for _ in range(args.steps):
            fwd_step()
        t_end.record(stream)
        torch.cuda.synchronize()
        eager_ms = max_over_ranks(t_start.elapsed_time(t_end), world) / args.steps
        graph = None
        graph_ms = None          # the workloads on concurrent streams
        if not args.eager:
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.stream(side):
                with torch.cuda.graph(graph, stream=side):
                    for _ in range(args.steps):
                        fwd_step()
            torch.cuda.synchronize()
            graph.replay()
            torch.cuda.synchronize()
            if len(sets) > 1 and args.concurrency == "streams":
                # The workloads are independent problems: each gets a stream that
                # runs its K forward calls back to back; the graph forks from and
                # joins to the capture stream, so the persistent kernels of one
                # workload fill the SMs another's leave idle in its tail.
                wstreams = [torch.cuda.Stream() for _ in sets]
                graph_ms = torch.cuda.CUDAGraph()
                with torch.cuda.stream(side):
                    with torch.cuda.graph(graph_ms, stream=side):
                        for ws_ in wstreams:
                            ws_.wait_stream(side)
                        for ws_, (w, d, _) in zip(wstreams, sets):
                            with torch.cuda.stream(ws_):
                                for _ in range(args.steps):
                                    sla.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H,
                                                w.eps, out=d["out"], workspace=d["ws"])
                        for ws_ in wstreams:
                            side.wait_stream(ws_)
                torch.cuda.synchronize()
                graph_ms.replay()
                torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            # keep the GPU busy for ~0.3 s inside the sampling window (untimed), so the
            # clock samples see the clocks the timed steps run at
            t0 = time.perf_counter()
            while time.perf_counter() - t0 < 0.3:
                if graph is not None:
                    graph.replay()
                else:
                    fwd_step()
                torch.cuda.synchronize()
            barrier(world)
            torch.cuda.synchronize()
            t_start.record(stream)
            if graph is not None:
                graph.replay()
            else:
                for _ in range(args.steps):
                    fwd_step()
            t_end.record(stream)
            torch.cuda.synchronize()
            barrier(world)
            if graph_ms is not None:
                t_s2 = torch.cuda.Event(enable_timing=True)
                t_e2 = torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                barrier(world)
                t_s2.record(stream)
                graph_ms.replay()
                t_e2.record(stream)
                torch.cuda.synchronize()
                barrier(world)
        # (2) per-pass durations for the roofline: the same K steps as kv_state +
        # apply (the two halves of sana_linattn_forward), events between the passes.
        barrier(world)
        torch.cuda.synchronize()
        for s_ in range(args.steps):
            step(ev[s_])
        torch.cuda.synchronize()
        one_stream_ms = max_over_ranks(t_start.elapsed_time(t_end), world) / args.steps
        ms_per_step = one_stream_ms
        if graph_ms is not None:
            ms_per_step = max_over_ranks(t_s2.elapsed_time(t_e2), world) / args.steps
        value = tokens_per_step * world / (ms_per_step * 1e-3) / 1e6
        # per-pass durations (average per launch) and algorithmic bytes
        parts = []
        p1_ms = p2_ms = 0.0
        p1_b = p2_b = 0
        for i, (w, d, _) in enumerate(sets):
            a = statistics.fmean(ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(args.steps))
            b = statistics.fmean(ev[s][i][2].elapsed_time(ev[s][i][3]) for s in range(args.steps))
            by = w.tokens * PASS_BYTES_PER_TOKEN
            p1_ms += a
            p2_ms += b
            p1_b += by
            p2_b += by
            parts.append({"workload": w.name, "tokens": w.tokens, "ms": a + b,
                          "Mtokens_per_s": w.tokens / ((a + b) * 1e-3) / 1e6,
                          "pass1_ms": a, "pass2_ms": b,
                          "hbm_frac_of_measured": 2 * by / ((a + b) * 1e-3) / 1e9 / hbm_gbs})
        # roofline of the dominant pass, on the largest launch shape of the sweep
        dom_name, dom_kernel = ("pass 1 (state)", "kv_partials_persistent") if p1_ms >= p2_ms else \
            ("pass 2 (apply)", "apply_persistent")
        big = max(range(len(sets)), key=lambda i: sets[i][0].tokens * 1e9 + sets[i][0].N)
        wb = sets[big][0]
        ms_big = parts[big]["pass1_ms" if p1_ms >= p2_ms else "pass2_ms"]
        bytes_big = wb.tokens * PASS_BYTES_PER_TOKEN
        achieved = bytes_big / (ms_big * 1e-3) / 1e9
        line.update({"value": value, "ms_per_step": ms_per_step,
                     "launch": ("eager sana_linattn_forward calls" if graph is None else
                                "one CUDA graph of the K steps of sana_linattn_forward calls" +
                                (", each workload on its own stream (independent problems "
                                 "run concurrently; the graph forks and joins once)"
                                 if graph_ms is not None else ", one stream")),
                     "value_one_stream": tokens_per_step * world / (one_stream_ms * 1e-3) / 1e6,
                     "eager_value": tokens_per_step * world / (eager_ms * 1e-3) / 1e6,
                     "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs,
                                  "unit": "GB/s", "frac": achieved / hbm_gbs,
                                  "traffic": ncu_traffic(dom_kernel, wb.name),
                                  "kernel": dom_kernel, "pass": dom_name,
                                  "workload": wb.name,
                                  "algorithmic_bytes_per_launch": bytes_big,
                                  "launch_ms": ms_big,
                                  "peak_kind": f"{peak_kind} copy bandwidth (hbm_gbs)",
                                  "sweep_pass_frac": (p1_b if p1_ms >= p2_ms else p2_b) /
                                  ((p1_ms if p1_ms >= p2_ms else p2_ms) * 1e-3) / 1e9 / hbm_gbs,
                                  "sweep_op_frac": 2 * p1_b / ((p1_ms + p2_ms) * 1e-3) / 1e9
                                  / hbm_gbs,
                                  # the whole op's roof in tokens/s (17,920 B/token per GPU)
                                  "op_roof_mtok_s": {
                                      "measured": hbm_gbs * 1e9 / (2 * PASS_BYTES_PER_TOKEN) / 1e6
                                      * world,
                                      "nominal_8tbs": HBM_NOMINAL_GBS * 1e9
                                      / (2 * PASS_BYTES_PER_TOKEN) / 1e6 * world},
                                  "value_frac_of_op_roof": {
                                      "measured": value / (hbm_gbs * 1e9 /
                                                           (2 * PASS_BYTES_PER_TOKEN) / 1e6 * world),
                                      "nominal_8tbs": value / (HBM_NOMINAL_GBS * 1e9 /
                                                               (2 * PASS_BYTES_PER_TOKEN) / 1e6 *
                                                               world)}},
                     "parts": parts,
                     "gpu_launches": args.steps * sum(sla.forward_kernels(w.B, w.N, w.C, w.H)
                                                      for w, _, _ in sets),
                     "per_pass_timing": "a second K-step loop of the forward's two kernels as "
                                        "separate calls (sana_linattn_forward_pass1, _pass2), "
                                        "each after a 512 MB L2-evicting read, CUDA events "
                                        "around each launch",
                     "clocks": clk.summary()})

        if world == 1 and rank == 0 and not args.no_cpu and args.workload == "sweep":
            line["configs"] = configs_measure(args, sla, sets, dev, hbm_gbs, bf16_tf, peak_kind)
        if not args.no_fused:
            line["causal"] = causal_measure(args, sla, sets, stream, world, hbm_gbs)
            line["backward"] = backward_measure(args, sla, sets, stream, world, hbm_gbs)

        # e2e: the public call with host buffers, copies inside the timed region
        if not args.no_e2e:
            line["e2e"] = e2e_measure(args, sla, sets, stream, world)

    if args.workload == "w8a8" or (args.workload == "sweep" and not args.no_fused):
        line["w8a8"] = w8a8_measure(args, sla, WORKLOADS["w8a8-2048px-b4"], rank, dev, stream, world, bf16_tf,
                                    peak_kind)
        if args.workload == "w8a8":
            f = line["w8a8"]
            line.update({"value": f["value"], "ms_per_step": f["ms_per_step"],
                         "roofline": f["roofline"], "gpu_launches": f["gpu_launches"],
                         "clocks": f.get("clocks")})
            line["config"] = {"workload": WORKLOADS["w8a8-2048px-b4"].name, "B": 4, "N": 4096, "C": 2240,
                              "H": 70, "parallelism": f"dp{world}"}
    if args.workload == "mixffn" or (args.workload == "sweep" and not args.no_fused):
        line["mixffn"] = mixffn_measure(args, sla, rank, dev, stream, world, bf16_tf, hbm_gbs,
                                        peak_kind)
        if args.workload == "mixffn":
            f = line["mixffn"]
            line.update({"metric": "Mix-FFN tokens per second", "value": f["value"],
                         "ms_per_step": f["ms_per_step"], "roofline": f["roofline"],
                         "gpu_launches": f["gpu_launches"], "clocks": f.get("clocks"),
                         "e2e": f["e2e"]})
            line["config"] = {"workload": f["workload"], "B": 4, "Hs": 64, "Ws": 64, "C": 2240,
                              "F": 5600, "parallelism": f"dp{world}"}
    if args.workload == "fused" or (args.workload == "sweep" and not args.no_fused):
        line["fused"] = fused_measure(args, sla, WORKLOADS["fused-2048px-b4"], rank, dev, stream, world, bf16_tf,
                                      peak_kind)
        if not sets:
            f = line["fused"]
            line.update({"value": f["value"], "ms_per_step": f["ms_per_step"],
                         "roofline": f["roofline"], "gpu_launches": f["gpu_launches"],
                         "clocks": f.get("clocks"), "e2e": f.get("e2e")})
            line["config"] = {"workload": WORKLOADS["fused-2048px-b4"].name, "B": 4, "N": 4096, "C": 2240, "H": 70,
                              "parallelism": f"dp{world}"}

    if rank == 0 and world == 1 and not args.no_cpu and args.workload == "mixffn":
        line["cpu_baseline"] = mixffn_cpu_sample()
    elif rank == 0 and world == 1 and not args.no_cpu:
        pairs = [(w, x) for w, _, x in sets]
        if not pairs:
            w = WORKLOADS["1024px-b1"]
            pairs = [(w, make_inputs(w))]
        line["cpu_baseline"] = cpu_oracle_sample(pairs)
    if rank == 0:
        print(json.dumps(line), flush=True)


def graph_call_ms(body, steps: int) -> float:
    """Device time per call of `body`, recorded `steps` times into one CUDA graph
    (median of 5 replays after 2 warm-up replays)."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        body()
        side.synchronize()
        with torch.cuda.graph(g, stream=side):
            for _ in range(steps):
                body()
    torch.cuda.synchronize()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / steps)
    del g
    return statistics.median(ts)


def configs_measure(args, sla, sets, dev, hbm_gbs, bf16_tf, peak_kind):
    """One record per named workload of the metric's configurations: the tiny fp32
    check, the three SANA latent sizes and the fused-QKV 2048px batch of 4.

    time: the op alone, `steps` calls in one CUDA graph, each call preceded by a
    read of a 512 MB buffer that evicts the op's inputs from L2 (a cold L2 for every
    call); the flush's own time, measured the same way, is subtracted.
    cpu_baseline + parity: the fp64 oracle, as it stands, on a bounded sample of
    the workload (batch item 0 of the attention workloads; 256 sampled tokens of
    batch item 0 for the fused one, whose state still needs all of that item's
    tokens), timed on the host cores; the GPU output of the same tokens is
    compared with the oracle's (max-abs, mean-abs, normwise relative L2)."""
    import numpy as np
    import torch
    from oracle import oracle as O
    from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs

    steps = max(3, min(args.steps, 20))
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    sink = torch.empty(1, dtype=torch.int64, device=dev)

    def do_flush():
        torch.sum(flush.view(torch.int64), dim=0, keepdim=True, out=sink)
    t_flush = graph_call_ms(do_flush, steps)

    def errs(got, ref):
        g = np.asarray(got, dtype=np.float64)
        d = np.abs(g - ref)
        return {"max_abs": float(d.max()), "mean_abs": float(d.mean()),
                "rel_l2": float(np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-300)),
                "finite": bool(np.isfinite(g).all())}

    recs = {}
    # the tiny fp32 check and the three latent sizes
    tiny = WORKLOADS["tiny-512px-f32"]
    xt = make_inputs(tiny)
    dt = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in xt.items()}
    dt["out"] = torch.empty_like(dt["q"])
    dt["ws"] = torch.empty(sla.workspace_bytes(tiny.B, tiny.N, tiny.C, tiny.H), dtype=torch.uint8,
                           device=dev)
    for w, d, x in [(tiny, dt, xt)] + [(w, d, x) for w, d, x in sets]:
        def call(w=w, d=d):
            sla.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps, out=d["out"],
                        workspace=d["ws"])
        ms = graph_call_ms(lambda: (do_flush(), call()), steps) - t_flush
        call()
        torch.cuda.synchronize()
        got = d["out"][:1].float().cpu().numpy()
        t0 = time.perf_counter()
        ref = O.forward(x["q"][:1], x["k"][:1], x["v"][:1], x["gq"], x["gk"], w.H, w.eps)
        t_cpu = time.perf_counter() - t0
        by = w.tokens * (2 * w.C * (4 if w.dtype == "f32" else 2) * 2)
        rec = {"B": w.B, "N": w.N, "C": w.C, "H": w.H, "dtype": w.dtype, "us": ms * 1e3,
               "Mtokens_per_s": w.tokens / (ms * 1e-3) / 1e6,
               "parity_vs_oracle": errs(got, ref) | {"sample": "batch item 0, every token"},
               "cpu_oracle": {"Mtokens_per_s": w.N / t_cpu / 1e6, "cores": O.host_threads(),
                              "sample": "batch item 0"}}
        if w.dtype == "bf16":
            rec["hbm_frac"] = {"measured": by / (ms * 1e-3) / 1e9 / hbm_gbs,
                               "nominal_8tbs": by / (ms * 1e-3) / 1e9 / HBM_NOMINAL_GBS}
        recs[w.name] = rec
    del dt
    # the fused QKV variant
    wf = WORKLOADS["fused-2048px-b4"]
    xf = make_inputs(wf)
    df = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in xf.items()}
    of = torch.empty_like(df["x"])
    wsf = torch.empty(sla.workspace_bytes(wf.B, wf.N, wf.C, wf.H, fused=True), dtype=torch.uint8,
                      device=dev)

    def fcall():
        sla.qkv_fused(df["x"], df["W"], df["gq"], df["gk"], wf.H, wf.eps, out=of, workspace=wsf)
    ms = graph_call_ms(lambda: (do_flush(), fcall()), steps) - t_flush
    fcall()
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    tok = np.sort(rng.choice(wf.N, size=256, replace=False))
    got = of[0].float().cpu().numpy()[tok]
    t0 = time.perf_counter()
    ref = O.fused_forward(xf["x"][:1], xf["W"], xf["gq"], xf["gk"], wf.H, wf.eps, tokens=tok)
    t_cpu = time.perf_counter() - t0
    fl = 2.0 * wf.tokens * wf.C * 3 * wf.C
    recs[wf.name] = {"B": wf.B, "N": wf.N, "C": wf.C, "H": wf.H, "dtype": "bf16", "us": ms * 1e3,
                     "Mtokens_per_s": wf.tokens / (ms * 1e-3) / 1e6,
                     "tflops": fl / (ms * 1e-3) / 1e12,
                     "tensor_frac": {"of": f"{peak_kind} bf16 burst", "value":
                                     fl / (ms * 1e-3) / 1e12 / bf16_tf},
                     "parity_vs_oracle": errs(got, ref.reshape(len(tok), wf.C)) |
                     {"sample": "256 sampled tokens of batch item 0"},
                     "cpu_oracle": {"Mtokens_per_s": len(tok) / t_cpu / 1e6,
                                    "cores": O.host_threads(),
                                    "sample": "256 tokens of batch item 0 (with the K, V "
                                              "projection of all its 4096 tokens)"}}
    return {"timing": f"{steps} calls in one CUDA graph, each after a 512 MB read that "
                      "evicts L2; the read's own time subtracted", "workloads": recs}


def e2e_measure(args, sla, sets, stream, world):
    """The metric through the public call with host buffers: every step uploads its
    q, k, v from pinned host memory, runs sana_linattn_forward and downloads the
    output.  Uploads, compute and downloads run on three streams with double-
    buffered device tensors, so step s+1's uploads overlap step s's compute and
    downloads (PCIe is full duplex); the timed region spans the first upload to
    the last download."""
    import torch
    dev = stream.device
    host, bufs = [], []
    for w, d, x in sets:
        h = {n: x[n].pin_memory() for n in ("q", "k", "v")}
        h["out"] = torch.empty_like(x["q"]).pin_memory()
        host.append(h)
    for _ in range(2):
        bufs.append([{n: torch.empty_like(d[n]) for n in ("q", "k", "v", "out")} | {"ws": d["ws"]}
                     for (w, d, _) in sets])
    # each buffer set gets its own workspace so overlapping steps never share one
    for i, (w, d, _) in enumerate(sets):
        bufs[1][i]["ws"] = torch.empty_like(d["ws"])
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = len(sets)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [[ev() for _ in range(n)] for _ in range(2)]
    comp_done = [[ev() for _ in range(n)] for _ in range(2)]
    out_done = [[ev() for _ in range(n)] for _ in range(2)]
    used = [[False] * n for _ in range(2)]
    h2d = sum(3 * w.tokens * w.C * 2 for w, *_ in sets)
    d2h = sum(w.tokens * w.C * 2 for w, *_ in sets)
    tokens = sum(w.tokens for w, *_ in sets)

    def step(si):
        bset = si % 2
        for i, (w, d, _) in enumerate(sets):
            b, h = bufs[bset][i], host[i]
            with torch.cuda.stream(s_in):
                if used[bset][i]:
                    s_in.wait_event(comp_done[bset][i])      # inputs no longer read
                for nm in ("q", "k", "v"):
                    b[nm].copy_(h[nm], non_blocking=True)
                in_done[bset][i].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(in_done[bset][i])
                if used[bset][i]:
                    s_comp.wait_event(out_done[bset][i])      # output no longer read
                sla.forward(b["q"], b["k"], b["v"], d["gq"], d["gk"], w.H, w.eps, out=b["out"],
                            workspace=b["ws"], stream=s_comp)
                comp_done[bset][i].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[bset][i])
                h["out"].copy_(b["out"], non_blocking=True)
                out_done[bset][i].record(s_out)
            used[bset][i] = True

    steps = max(3, min(args.steps, 10))
    for si in range(2):
        step(si)
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    a.record(s_in)
    s_comp.wait_stream(s_in)
    s_out.wait_stream(s_in)
    for si in range(steps):
        step(si)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    z.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(z), world) / steps
    return {"value": tokens * world / (ms * 1e-3) / 1e6, "unit": "Mtokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": steps, "api": "sana_linattn_forward",
            "overlap": "uploads, compute and downloads on three streams, double-buffered"}


def fused_measure(args, sla, w, rank, dev, stream, world, bf16_tf, peak_kind):
    import torch
    from relu_linear_attention_attn_b200.synthetic import make_inputs
    x = make_inputs(w.scaled(seed=w.seed + 1000 * rank) if rank else w)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    out = torch.empty_like(d["x"])
    ws = torch.empty(sla.workspace_bytes(w.B, w.N, w.C, w.H, fused=True), dtype=torch.uint8,
                     device=dev)
    steps = max(3, min(args.steps, 20))

    def call():
        sla.qkv_fused(d["x"], d["W"], d["gq"], d["gk"], w.H, w.eps, out=out, workspace=ws)
    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    with ClockSampler(dev.index) as clk:
        barrier(world)
        torch.cuda.synchronize()
        for a, b in evs:
            a.record(stream)
            call()
            b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms = max_over_ranks(statistics.fmean(a.elapsed_time(b) for a, b in evs), world)
    # e2e: the public call with host buffers (pinned x uploaded, O downloaded each step)
    hx = x["x"].pin_memory()
    ho = torch.empty_like(hx).pin_memory()
    dx = torch.empty_like(d["x"])

    def e2e_step():
        dx.copy_(hx, non_blocking=True)
        sla.qkv_fused(dx, d["W"], d["gq"], d["gk"], w.H, w.eps, out=out, workspace=ws)
        ho.copy_(out, non_blocking=True)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / steps, world)
    flops = 2.0 * w.tokens * w.C * 3 * w.C
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": w.name, "value": w.tokens * world / (ms * 1e-3) / 1e6,
            "unit": "Mtokens/s", "ms_per_step": ms, "steps": steps,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16_tf, "unit": "TFLOP/s",
                         "frac": tf / bf16_tf, "traffic": None,
                         "kernel": "fused_kv + fused_qo (the whole fused op)",
                         "flop_per_launch": flops,
                         "peak_kind": f"{peak_kind} bf16 burst (bf16_tflops)"},
            "e2e": {"value": w.tokens * world / (e2e_ms * 1e-3) / 1e6, "unit": "Mtokens/s",
                    "h2d_bytes_per_step": hx.numel() * hx.element_size(),
                    "d2h_bytes_per_step": ho.numel() * ho.element_size()},
            "gpu_launches": steps * 2, "clocks": clk.summary()}


def causal_measure(args, sla, sets, stream, world, hbm_gbs):
    """The prefix (causal) form over the sweep's workloads (inputs resident, K steps
    of sana_linattn_forward_causal per workload, CUDA events per call)."""
    import torch
    steps = max(3, min(args.steps, 10))
    parts, tot_tok, tot_ms = [], 0, 0.0
    for w, d, _ in sets:
        ws = torch.empty(int(sla.load().sana_linattn_workspace_bytes(w.B, w.N, w.C, w.H, 2)),
                         dtype=torch.uint8, device=d["q"].device)

        def call():
            sla.forward_causal(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps,
                               out=d["out"], workspace=ws)
        for _ in range(max(args.warmup, 3)):
            call()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        for a, b in evs:
            a.record(stream)
            call()
            b.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(statistics.fmean(a.elapsed_time(b) for a, b in evs), world)
        by = w.tokens * 2 * PASS_BYTES_PER_TOKEN
        parts.append({"workload": w.name, "ms": ms, "Mtokens_per_s": w.tokens / (ms * 1e-3) / 1e6,
                      "hbm_frac_of_measured": by / (ms * 1e-3) / 1e9 / hbm_gbs})
        tot_tok += w.tokens
        tot_ms += ms
    big = max(range(len(sets)), key=lambda i: sets[i][0].tokens * 1e9 + sets[i][0].N)
    wb = sets[big][0]
    achieved = wb.tokens * 2 * PASS_BYTES_PER_TOKEN / (parts[big]["ms"] * 1e-3) / 1e9
    return {"value": tot_tok * world / (tot_ms * 1e-3) / 1e6, "unit": "Mtokens/s",
            "ms_per_step": tot_ms, "steps": steps, "parts": parts,
            "chunk_tokens": 128,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": achieved / hbm_gbs, "traffic": None,
                         "kernel": "kv_partials_persistent<chunked> + causal_prefix_states + causal_apply_tc "
                                   "(tensor cores; bf16 with gains 16-byte aligned)",
                         "workload": wb.name,
                         "algorithmic_bytes_per_launch": wb.tokens * 2 * PASS_BYTES_PER_TOKEN,
                         # the two-pass design reads K and V twice (chunk states, then the apply)
                         "design_bytes_per_launch": wb.tokens * 3 * PASS_BYTES_PER_TOKEN,
                         "frac_of_design_bytes": achieved * 1.5 / hbm_gbs},
            "gpu_launches": steps * len(sets) * 3}


def backward_measure(args, sla, sets, stream, world, hbm_gbs):
    """The backward of the op (dq, dk, dv and the gain gradients from dO) over the
    sweep's workloads: inputs and dO resident, K steps of sana_linattn_backward per
    workload, CUDA events per call.  Algorithmic bytes: read q, k, v, dO and write
    dq, dk, dv once each (7 x C x 2 B per token in bf16)."""
    import torch
    from relu_linear_attention_attn_b200.synthetic import make_output_grad
    steps = max(3, min(args.steps, 10))
    parts, tot_tok, tot_ms, tot_ms_st = [], 0, 0.0, 0.0
    launches = 0
    for w, d, _ in sets:
        dev = d["q"].device
        do = make_output_grad(w).to(dev)
        grads = (torch.empty_like(d["q"]), torch.empty_like(d["q"]), torch.empty_like(d["q"]),
                 None if d["gq"] is None else torch.empty(w.C, dtype=torch.float32, device=dev),
                 None if d["gk"] is None else torch.empty(w.C, dtype=torch.float32, device=dev))
        ws = torch.empty(int(sla.load().sana_linattn_backward_workspace_bytes(w.B, w.N, w.C, w.H)),
                         dtype=torch.uint8, device=dev)

        # the forward's state, as a training step holds it from its forward (untimed)
        kv = sla.kv_state(d["k"], d["v"], d["gk"], w.H, w.eps)

        def call():
            sla.backward(d["q"], d["k"], d["v"], d["gq"], d["gk"], do, w.H, w.eps, grads=grads,
                         workspace=ws)

        def call_with_state():
            sla.backward(d["q"], d["k"], d["v"], d["gq"], d["gk"], do, w.H, w.eps, grads=grads,
                         workspace=ws, kv=kv)

        def timed(fn):
            for _ in range(max(args.warmup, 3)):
                fn()
            torch.cuda.synchronize()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
            barrier(world)
            torch.cuda.synchronize()
            for a, b in evs:
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            return max_over_ranks(statistics.fmean(a.elapsed_time(b) for a, b in evs), world)
        ms = timed(call)
        ms_st = timed(call_with_state)
        by = w.tokens * 7 * PASS_BYTES_PER_TOKEN // 2
        parts.append({"workload": w.name, "ms": ms, "Mtokens_per_s": w.tokens / (ms * 1e-3) / 1e6,
                      "hbm_frac_of_measured": by / (ms * 1e-3) / 1e9 / hbm_gbs,
                      "ms_with_forward_state": ms_st,
                      "hbm_frac_with_forward_state": by / (ms_st * 1e-3) / 1e9 / hbm_gbs})
        tot_tok += w.tokens
        tot_ms += ms
        tot_ms_st += ms_st
        launches += steps * (10 if d["gq"] is not None else 6)
        launches += steps * (8 if d["gq"] is not None else 4)
        del do, grads, ws, kv
    big = max(range(len(sets)), key=lambda i: sets[i][0].tokens * 1e9 + sets[i][0].N)
    wb = sets[big][0]
    by_big = wb.tokens * 7 * PASS_BYTES_PER_TOKEN // 2
    achieved = by_big / (parts[big]["ms"] * 1e-3) / 1e9
    return {"value": tot_tok * world / (tot_ms * 1e-3) / 1e6, "unit": "Mtokens/s",
            "ms_per_step": tot_ms, "steps": steps, "parts": parts,
            # sana_linattn_backward_with_state: the forward's state passed in, as a
            # training step holds it (no second pass over k and v for it)
            "value_with_forward_state": tot_tok * world / (tot_ms_st * 1e-3) / 1e6,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": achieved / hbm_gbs, "traffic": None,
                         "kernel": "forward state (pass 1 + combine) + bwd_query_tc + pass 1 "
                                   "(q, dnum; dden-weighted) + combine + bwd_key_tc + gain "
                                   "sums (tensor cores; bf16, N >= 128, gains 16-byte aligned)",
                         "workload": wb.name, "algorithmic_bytes_per_launch": by_big},
            "gpu_launches": launches}


def w8a8_measure(args, sla, w, rank, dev, stream, world, bf16_tf, peak_kind):
    """The fused op with the W8A8 prologue: Wqkv is quantised once (untimed, as a
    deployment would store it); each step quantises x per token and runs the W8A8
    fused kernels.  The projection's roofline is the int8 tensor peak, taken as
    the measured bf16 burst x 2 (the nominal dense int8 : bf16 ratio, 4.5 : 2.25
    PFLOP/s)."""
    import torch
    from relu_linear_attention_attn_b200.synthetic import make_inputs
    x = make_inputs(w.scaled(seed=w.seed + 1000 * rank) if rank else w)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    Wq, sw = sla.quantize_cols_i8(d["W"])
    xq = torch.empty(d["x"].shape, dtype=torch.int8, device=dev)
    sx = torch.empty(d["x"].shape[:-1], dtype=torch.float32, device=dev)
    out = torch.empty_like(d["x"])
    ws = torch.empty(sla.workspace_bytes(w.B, w.N, w.C, w.H, fused=True), dtype=torch.uint8,
                     device=dev)
    steps = max(3, min(args.steps, 20))

    def fused():
        sla.qkv_fused_w8a8(xq, sx, Wq, sw, d["gq"], d["gk"], w.H, w.eps, out=out, workspace=ws)

    def step():
        sla.quantize_rows_i8(d["x"], out=xq, scales=sx)
        fused()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    with ClockSampler(dev.index) as clk:
        barrier(world)
        torch.cuda.synchronize()
        for e in ev:
            e[0].record(stream)
            sla.quantize_rows_i8(d["x"], out=xq, scales=sx)
            e[1].record(stream)
            fused()
            e[2].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    q_ms = max_over_ranks(statistics.fmean(e[0].elapsed_time(e[1]) for e in ev), world)
    f_ms = max_over_ranks(statistics.fmean(e[1].elapsed_time(e[2]) for e in ev), world)
    ops = 2.0 * w.tokens * w.C * 3 * w.C
    i8_peak = 2.0 * bf16_tf
    tops = ops / (f_ms * 1e-3) / 1e12
    return {"workload": w.name, "value": w.tokens * world / ((q_ms + f_ms) * 1e-3) / 1e6,
            "unit": "Mtokens/s", "ms_per_step": q_ms + f_ms, "quantize_x_ms": q_ms,
            "fused_ms": f_ms, "steps": steps,
            "granularity": "int8 symmetric, one scale per token of x and per output channel "
                           "of Wqkv (Wqkv quantised once, untimed)",
            "roofline": {"bound": "tensor", "achieved": tops, "peak": i8_peak, "unit": "TOPS",
                         "frac": tops / i8_peak, "traffic": None,
                         "kernel": "fused_kv<int8> + fused_qo<int8> (the projection is kind::i8)",
                         "op_per_launch": ops,
                         "peak_kind": f"int8 = 2 x {peak_kind} bf16 burst (bf16_tflops), the "
                                      "nominal dense int8:bf16 ratio"},
            "gpu_launches": steps * 3, "clocks": clk.summary()}


def mixffn_measure(args, sla, rank, dev, stream, world, bf16_tf, hbm_gbs, peak_kind):
    """The Mix-FFN tail of the block on the 2048px batch of 4 (64 x 64 latent grid,
    C = 2240, F = 5600): one step = expand GEMM -> depthwise 3x3 + GLU -> project
    GEMM (sana_mixffn_forward's three kernels, inputs resident), CUDA events between
    the launches.  The dominant kernel is the expand GEMM, bound by the tensor peak;
    the depthwise conv + GLU is HBM-bound (reads U, writes Hg: 3F x 2 B per token)."""
    import torch
    from relu_linear_attention_attn_b200.synthetic import MIXFFN_WORKLOADS, make_mixffn_inputs
    w = MIXFFN_WORKLOADS["mixffn-2048px-b4"]
    x = make_mixffn_inputs(w.scaled(seed=w.seed + 1000 * rank) if rank else w)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    M = w.tokens
    u = torch.empty(M, 2 * w.F, dtype=torch.bfloat16, device=dev)
    h = torch.empty(M, w.F, dtype=torch.bfloat16, device=dev)
    y = torch.empty(M, w.C, dtype=torch.bfloat16, device=dev)
    xf = d["x"].reshape(M, w.C)
    steps = max(3, min(args.steps, 20))
    stages = (lambda: sla.gemm_bias(xf, d["W1"], d["b1"], out=u),
              lambda: sla.mixffn_dwconv_glu(u.view(w.B, w.N, 2 * w.F), d["wdw"], d["bdw"], w.Hs,
                                            w.Ws, w.gate, out=h.view(w.B, w.N, w.F)),
              lambda: sla.gemm_bias(h, d["W2"], d["b2"], out=y))
    for _ in range(max(args.warmup, 3)):
        for f in stages:
            f()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    with ClockSampler(dev.index) as clk:
        barrier(world)
        torch.cuda.synchronize()
        for e in ev:
            e[0].record(stream)
            for i, f in enumerate(stages):
                f()
                e[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms = [max_over_ranks(statistics.fmean(e[i].elapsed_time(e[i + 1]) for e in ev), world)
          for i in range(3)]
    # e2e: the public call with host buffers (pinned x uploaded, y downloaded each step)
    hx = x["x"].pin_memory()
    hy = torch.empty_like(hx).pin_memory()
    ws = torch.empty(sla.mixffn_workspace_bytes(w.B, w.Hs, w.Ws, w.C, w.F), dtype=torch.uint8,
                     device=dev)
    dx, dy = torch.empty_like(d["x"]), torch.empty_like(d["x"])

    def e2e_step():
        dx.copy_(hx, non_blocking=True)
        sla.mixffn_forward(dx, d["W1"], d["b1"], d["wdw"], d["bdw"], d["W2"], d["b2"], w.Hs, w.Ws,
                           w.gate, out=dy, workspace=ws)
        hy.copy_(dy, non_blocking=True)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / steps, world)
    fl_expand = 2.0 * M * w.C * 2 * w.F
    fl_project = 2.0 * M * w.F * w.C
    dw_bytes = M * 3 * w.F * 2
    tf = fl_expand / (ms[0] * 1e-3) / 1e12
    return {"workload": w.name, "value": M * world / (sum(ms) * 1e-3) / 1e6,
            "unit": "Mtokens/s", "ms_per_step": sum(ms), "steps": steps,
            "expand_ms": ms[0], "dwconv_glu_ms": ms[1], "project_ms": ms[2],
            "expand_tflops": tf, "project_tflops": fl_project / (ms[2] * 1e-3) / 1e12,
            "dwconv_glu_hbm_frac": dw_bytes / (ms[1] * 1e-3) / 1e9 / hbm_gbs,
            "step_tflops": (fl_expand + fl_project) / (sum(ms) * 1e-3) / 1e12,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16_tf, "unit": "TFLOP/s",
                         "frac": tf / bf16_tf,
                         "traffic": ncu_traffic("gemm_bias_bf16_2sm", w.name, MIXFFN_SOURCES),
                         "kernel": "gemm_bias_bf16_2sm (expand, 16384 x 2240 x 11200; UMMA over SM pairs)",
                         "flop_per_launch": fl_expand,
                         "peak_kind": f"{peak_kind} bf16 burst (bf16_tflops)"},
            "e2e": {"value": M * world / (e2e_ms * 1e-3) / 1e6, "unit": "Mtokens/s",
                    "h2d_bytes_per_step": hx.numel() * 2, "d2h_bytes_per_step": hy.numel() * 2},
            "gpu_launches": steps * 3, "clocks": clk.summary()}


def profile_case(args):
    """--warmup calls of sana_linattn_forward (two kernel launches each; with --causal
    sana_linattn_forward_causal, three; with --backward sana_linattn_backward) on one
    workload, optionally with another batch size; prints a checksum."""
    import torch

    import relu_linear_attention_attn_b200 as sla
    from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs

    fused = args.workload in ("fused", "w8a8")
    w = {"fused": WORKLOADS["fused-2048px-b4"], "w8a8": WORKLOADS["w8a8-2048px-b4"]}.get(args.workload) or select(args.workload)[-1]
    if args.batch:
        w = w.scaled(B=args.batch)
    x = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in make_inputs(w).items()}
    if args.backward:
        from relu_linear_attention_attn_b200.synthetic import make_output_grad
        dout = make_output_grad(w).cuda()
        ws = None
    elif args.causal:
        ws = torch.empty(int(sla.load().sana_linattn_workspace_bytes(w.B, w.N, w.C, w.H, 2)),
                         dtype=torch.uint8, device="cuda")
    else:
        ws = torch.empty(sla.workspace_bytes(w.B, w.N, w.C, w.H, fused=fused),
                         dtype=torch.uint8, device="cuda")
    if args.workload == "w8a8":
        Wq, sw = sla.quantize_cols_i8(x["W"])
    for _ in range(args.warmup):
        if args.workload == "fused":
            out = sla.qkv_fused(x["x"], x["W"], x["gq"], x["gk"], w.H, w.eps, workspace=ws)
        elif args.workload == "w8a8":
            xq, sx = sla.quantize_rows_i8(x["x"])
            out = sla.qkv_fused_w8a8(xq, sx, Wq, sw, x["gq"], x["gk"], w.H, w.eps, workspace=ws)
        elif args.backward:
            out = sla.backward(x["q"], x["k"], x["v"], x["gq"], x["gk"], dout, w.H, w.eps)[0]
        elif args.causal:
            out = sla.forward_causal(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps, workspace=ws)
        else:
            out = sla.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps, workspace=ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": w.name, "B": w.B, "N": w.N, "calls": args.warmup,
                      "checksum": float(out.float().abs().mean())}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="sweep",
                    choices=["sweep", "fused", "w8a8", "mixffn", "1024px", "2048px", "4096px"])
    ap.add_argument("--no-fused", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches, no CUDA graph")
    ap.add_argument("--profile-case", action="store_true",
                    help="no timing: run --warmup forward calls of --workload and exit (a small, "
                         "fixed launch sequence for ncu captures)")
    ap.add_argument("--causal", action="store_true",
                    help="with --profile-case: the prefix (causal) form")
    ap.add_argument("--backward", action="store_true",
                    help="with --profile-case: the backward (dO drawn as in the bench)")
    ap.add_argument("--batch", type=int, default=0,
                    help="with --profile-case: batch size override for the workload")
    ap.add_argument("--concurrency", choices=["streams", "serial"], default="streams",
                    help="sweep: run the workloads on one stream each (independent problems "
                         "overlapping on the SMs) or all on one stream")
    ap.add_argument("--shard", choices=["batch", "seq"], default="batch",
                    help="batch: every rank runs its own batch (weak scaling, no collective); "
                         "seq: the ranks split each sequence and all-reduce the state "
                         "(sharding.sequence_parallel_forward; strong scaling)")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    spawn_ranks_if_needed(args)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, rank, world)
        return
    rank, world, local = dist_setup(args)
    try:
        run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
