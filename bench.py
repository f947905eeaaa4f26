#!/usr/bin/env python
"""Benchmark of the WKV7 hot path on B200.

One step = one wkv7_fwd over the B=8, T=4096, H=64, K=V=64 bf16 workload
(fp32 initial state in, fp32 final state out), inputs resident in HBM.  The
line also carries the decode step (wkv7_step over 1024 x 32 fp32 states, 256
consecutive steps) as HBM GB/s against the measured copy bandwidth.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own replica of the workload (the
(sequence, head) units are independent, no collective on the data path) and
rank 0 prints the whole-job throughput: all ranks' tokens / max-over-ranks time.
``--impl reference`` times the fp64 CPU oracle on a bounded sample instead.
``--family gdn`` measures the Gated DeltaNet entry points (wkv7_gdn_fwd /
wkv7_gdn_step) on workloads of the same shapes instead; ``--family sane`` the
State Anomaly Neutralization ones (wkv7_sane_fwd with the clip after every 16-token
chunk, wkv7_sane_step with do_sane every 16th step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_rnn_wkv7_b200 import replicas, synth  # noqa: E402

METRIC = "WKV7 fwd tokens/s (B=8,T=4096,H=64,D=64 bf16) + decode HBM GB/s vs peak"
FWD = synth.WORKLOADS["fwd_bf16_b8_t4096_h64"]
DEC = synth.WORKLOADS["step_bf16_b1024_h32_256steps"]
TOKEN_HEAD_BYTES = 6 * 64 * 2 + 64 * 2  # r,w,k,v,a,b in + o out, bf16
STATE_BYTES = 64 * 64 * 4
GDN_METRIC = "Gated DeltaNet fwd tokens/s (B=8,T=4096,H=64,D=64 bf16) + decode HBM GB/s vs peak"
GDN_FWD = synth.WORKLOADS["gdn_fwd_bf16_b8_t4096_h64"]
GDN_DEC = synth.WORKLOADS["gdn_step_bf16_b1024_h32_256steps"]
GDN_TOKEN_HEAD_BYTES = 3 * 64 * 2 + 2 * 2 + 64 * 2  # q,k,v + g,beta in, o out, bf16
SANE_METRIC = ("SANE fwd tokens/s (B=8,T=4096,H=64,D=64 bf16, clip every 16 tokens) + decode "
               "HBM GB/s vs peak")
FALLBACK_HBM_GBS = 6650.0


def fwd_algorithmic_bytes(B, T, H, D=64) -> int:
    """bf16 r,w,k,v,a,b in and o out per token-head; fp32 s0 in and sT out per unit."""
    return B * T * H * 7 * D * 2 + 2 * B * H * D * D * 4


def step_algorithmic_bytes(B, H, D=64) -> int:
    return B * H * (2 * D * D * 4 + 7 * D * 2)


def gdn_fwd_algorithmic_bytes(B, T, H, D=64) -> int:
    """bf16 q,k,v in, o out, g and beta in per token-head; fp32 states per unit."""
    return B * T * H * (4 * D * 2 + 2 * 2) + 2 * B * H * D * D * 4


def gdn_step_algorithmic_bytes(B, H, D=64) -> int:
    return B * H * (2 * D * D * 4 + 4 * D * 2 + 2 * 2)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def source_digest(files=None) -> str:
    """Digest of the kernel sources: the named files of csrc/ (the ones a kernel is
    built from), or all of them."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_rnn_wkv7_b200", "csrc")
    for name in sorted(files if files else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current sources of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entries = json.load(f)
    e = entries.get(kernel)
    if not e or e.get("source_digest") != source_digest(e.get("sources")):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device):
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, mx, reasons = [], [], set()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_oracle_sample(target_s: float = 12.0, gdn: bool = False):
    """Time the fp64 oracle (as it stands) on a bounded sample of the B=8,T=4096,H=64
    workload: whole (b, h) units of T=4096 tokens.  Returns the cpu_baseline dict."""
    import oracle  # test infrastructure; used here only for the CPU baseline leg
    if gdn:
        x = synth.gdn_inputs(1, GDN_FWD["T"], GDN_FWD["H"], dtype=torch.bfloat16,
                             seed=GDN_FWD["seed"], s0_std=GDN_FWD["s0_std"])
        names, call = ("q", "k", "v", "g", "beta"), oracle.gdn_fwd
    else:
        x = synth.fwd_inputs(1, FWD["T"], FWD["H"], dtype=torch.bfloat16, seed=FWD["seed"],
                             s0_std=FWD["s0_std"])
        names, call = tuple("rwkvab"), oracle.fwd
    H = FWD["H"]

    def run(units):
        sl = {n: x[n][:, :, :units] for n in names}
        t0 = time.perf_counter()
        _, _, used = call(*(sl[n] for n in names), s0=x["s0"][:, :units])
        return time.perf_counter() - t0, used

    probe_units = min(H, max(2, os.cpu_count() or 1))
    dt, used = run(probe_units)
    units = int(min(H, max(probe_units, probe_units * target_s / max(dt, 1e-3))))
    dt, used = run(units)
    token_heads = units * FWD["T"]
    return {"value": token_heads / H / dt, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"{units} of the 512 (b,h) units of B=8,T=4096,H=64 (b=0, h<{units}), "
                      f"full T=4096 each; tokens/s = token-heads / 64 / wall time"}


def fwd_config(desc: dict, algo: str, world: int, D: int = 64) -> dict:
    return {**desc, "K": D, "V": D, "state": "fp32 s0 in, fp32 sT out", "algo": algo,
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (>= 0.1 GB per step); no flush"}


def reference_arm(args, rank: int):
    """The oracle as the reference arm: each step is one bounded sample."""
    if rank != 0:
        return
    import oracle
    gdn = args.family == "gdn"
    sane = args.family == "sane"
    H, T = FWD["H"], FWD["T"]
    tau = None
    if gdn:
        x = synth.gdn_inputs(1, T, H, dtype=torch.bfloat16, seed=GDN_FWD["seed"],
                             s0_std=GDN_FWD["s0_std"])
        names, call = ("q", "k", "v", "g", "beta"), oracle.gdn_fwd
    else:
        x = synth.fwd_inputs(1, T, H, dtype=torch.bfloat16, seed=FWD["seed"],
                             s0_std=FWD["s0_std"])
        names, call = tuple("rwkvab"), oracle.fwd
    units = min(H, max(4, os.cpu_count() or 1))  # one whole (b, h) unit per host thread
    if sane:  # the SANE oracle runs its units one after another on one host thread
        units = 2
        tau = synth.sane_tau(1, T // 16, H, FWD["seed"])[:, :, :units]
    sl = {n: x[n][:, :, :units] for n in names}

    def one():
        if sane:
            oracle.sane_fwd(*(sl[n] for n in names), tau, s0=x["s0"][:, :units])
            return 1
        return call(*(sl[n] for n in names), s0=x["s0"][:, :units])[2]

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    used = 0
    for _ in range(args.steps):
        used = one()
    dt = time.perf_counter() - t0
    tokens = args.steps * units * T / H
    value = tokens / dt
    fam = "gdn_" if gdn else "sane_" if sane else ""
    line = {"metric": GDN_METRIC if gdn else SANE_METRIC if sane else METRIC, "value": value,
            "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": fwd_config({"workload": fam + "fwd_bf16_b8_t4096_h64",
                                  "B": FWD["B"], "T": T, "H": H}, "oracle", args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                             "sample": f"each step: {units} of the 512 (b,h) units of "
                                       f"B=8,T={T},H={H}, full T each, fp64 sequential "
                                       f"recurrence; tokens/s = token-heads / {H} / time"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--algo", choices=["auto", "recurrent", "chunked"], default="auto")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode leg")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--batch", type=int, default=FWD["B"],
                    help="forward batch (default 8; smaller only for profiling captures)")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward leg")
    ap.add_argument("--only", choices=["all", "fwd", "decode", "bwd"], default="all",
                    help="run only one leg (profiling captures)")
    ap.add_argument("--workload", choices=["b8_t4096_h64", "masked_b16_t4096_h32",
                                           "varlen_64seq_h32"], default="b8_t4096_h64",
                    help="forward workload (the metric is quoted on b8_t4096_h64)")
    ap.add_argument("--head-size", type=int, choices=[64, 128, 256], default=64,
                    help="K = V; 128 / 256 keep C = H x head size at 4096 (forward) and "
                         "2048 (decode), and run on the CUDA-core kernels")
    ap.add_argument("--family", choices=["wkv7", "gdn", "sane"], default="wkv7",
                    help="gdn: the Gated DeltaNet entry points on the B=8,T=4096,H=64 "
                         "forward and 1024x32 decode workloads; sane: the SANE ones")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    from linear_attention_rnn_wkv7_b200 import (library, wkv7_bwd, wkv7_fwd, wkv7_gdn_bwd,
                                                wkv7_gdn_fwd, wkv7_gdn_step, wkv7_sane_fwd,
                                                wkv7_sane_step, wkv7_step)
    library()  # fail loudly if the CUDA library is missing
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    def max_over_ranks(v: float) -> float:
        return replicas.max_over_ranks(v, device=device)

    hbm_peak, peak_kind = load_peaks()
    stream = torch.cuda.current_stream(device)
    fwd = None
    gdn = args.family == "gdn"
    sane = args.family == "sane"
    fwd_fn = wkv7_gdn_fwd if gdn else wkv7_sane_fwd if sane else wkv7_fwd
    step_fn = wkv7_gdn_step if gdn else wkv7_sane_step if sane else wkv7_step
    if args.only in ("all", "fwd"):
        fwd = fwd_leg(args, device, stream, fwd_fn, hbm_peak, peak_kind, max_over_ranks,
                      barrier, rank, world)
    decode = None
    if args.only in ("all", "decode") and not args.no_decode:
        decode = decode_leg(device, stream, step_fn, hbm_peak, peak_kind, max_over_ranks,
                            barrier, rank, gdn, args.head_size, sane=sane)
    backward = None
    if (args.only in ("all", "bwd") and not args.no_bwd and args.head_size == 64
            and args.workload == "b8_t4096_h64" and not sane):
        backward = bwd_leg(args, device, stream, wkv7_gdn_bwd if gdn else wkv7_bwd, hbm_peak,
                           peak_kind, max_over_ranks, barrier, rank, gdn)
    cpu = None
    if (rank == 0 and world == 1 and not args.no_cpu and args.only == "all"
            and args.head_size == 64 and not sane):
        cpu = cpu_oracle_sample(gdn=gdn)

    if rank == 0:
        desc = fwd["desc"] if fwd else {"workload": "none"}
        line = {"metric": GDN_METRIC if gdn else SANE_METRIC if sane else METRIC,
                "value": fwd and fwd["value"],
                "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": fwd and fwd["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": fwd_config(desc, args.algo, world, args.head_size),
                "roofline": fwd and fwd["roofline"], "cpu_baseline": cpu,
                "e2e": fwd and fwd["e2e"], "gpu_launches": args.steps if fwd else 0,
                "clocks": fwd and fwd["clocks"], "decode": decode, "backward": backward}
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def fwd_workload(args, rank):
    """Synthetic inputs, tokens per step and algorithmic bytes per launch of a workload."""
    mask = cu = None
    if args.family == "gdn":
        if args.workload != "b8_t4096_h64":
            raise SystemExit("--family gdn runs the b8_t4096_h64 workload only")
        D = args.head_size
        B, T, H = args.batch, GDN_FWD["T"], GDN_FWD["H"] * 64 // D
        x = synth.gdn_inputs(B, T, H, K=D, V=D, dtype=torch.bfloat16,
                             seed=replicas.replica_seed(GDN_FWD["seed"], rank),
                             s0_std=GDN_FWD["s0_std"])
        tag = "" if D == 64 else f"_d{D}"
        return (x, None, None, B, T, H, B * T, gdn_fwd_algorithmic_bytes(B, T, H, D),
                {"workload": f"gdn_fwd_bf16_b{B}_t{T}_h{H}{tag}", "B": B, "T": T, "H": H})
    if args.head_size != 64 and args.workload != "b8_t4096_h64":
        raise SystemExit("--head-size applies to the b8_t4096_h64 workload only")
    if args.family == "sane":
        if args.workload != "b8_t4096_h64":
            raise SystemExit("--family sane runs the b8_t4096_h64 workload only")
        D = args.head_size
        B, T, H = args.batch, FWD["T"], FWD["H"] * 64 // D
        seed = replicas.replica_seed(FWD["seed"], rank)
        x = synth.fwd_inputs(B, T, H, K=D, V=D, dtype=torch.bfloat16, seed=seed,
                             s0_std=FWD["s0_std"])
        x["tau"] = synth.sane_tau(B, T // 16, H, seed)
        tag = "" if D == 64 else f"_d{D}"
        nbytes = fwd_algorithmic_bytes(B, T, H, D) + x["tau"].numel() * 4
        return (x, None, None, B, T, H, B * T, nbytes,
                {"workload": f"sane_fwd_bf16_b{B}_t{T}_h{H}{tag}", "B": B, "T": T, "H": H,
                 "sane": "clip after every 16-token chunk"})
    if args.workload == "b8_t4096_h64":
        D = args.head_size
        B, T, H = args.batch, FWD["T"], FWD["H"] * 64 // D
        x = synth.fwd_inputs(B, T, H, K=D, V=D, dtype=torch.bfloat16,
                             seed=replicas.replica_seed(FWD["seed"], rank), s0_std=FWD["s0_std"])
        tokens = B * T
        nbytes = fwd_algorithmic_bytes(B, T, H, D)
        tag = "" if D == 64 else f"_d{D}"
        desc = {"workload": f"fwd_bf16_b{B}_t{T}_h{H}{tag}", "B": B, "T": T, "H": H}
    elif args.workload == "masked_b16_t4096_h32":
        p = synth.WORKLOADS["fwd_bf16_masked_b16_t4096_h32"]
        B, T, H = p["B"], p["T"], p["H"]
        x = synth.fwd_inputs(B, T, H, dtype=torch.bfloat16,
                             seed=replicas.replica_seed(p["seed"], rank), s0_std=p["s0_std"])
        mask = synth.padding_mask(B, T, seed=replicas.replica_seed(p["seed"], rank))
        kept = int(mask.sum())
        tokens = B * T
        # masked tokens only need r in and o out; the mask itself is read once
        nbytes = (kept * H * TOKEN_HEAD_BYTES + (B * T - kept) * H * 2 * 64 * 2 + B * T
                  + 2 * B * H * STATE_BYTES)
        desc = {"workload": "fwd_bf16_masked_b16_t4096_h32", "B": B, "T": T, "H": H,
                "masked_fraction": 1 - kept / (B * T)}
    else:
        p = synth.WORKLOADS["fwd_bf16_varlen_64seq_h32"]
        lengths = synth.varlen_lengths(p["n_seqs"], p["lo"], p["hi"],
                                       seed=replicas.replica_seed(p["seed"], rank))
        H = p["H"]
        x = synth.varlen_inputs(lengths, H, dtype=torch.bfloat16,
                                seed=replicas.replica_seed(p["seed"], rank), s0_std=p["s0_std"])
        cu = x.pop("cu_seqlens")
        B, T = 1, int(lengths.sum())
        tokens = T
        nbytes = T * H * TOKEN_HEAD_BYTES + 2 * lengths.numel() * H * STATE_BYTES
        desc = {"workload": "fwd_bf16_varlen_64seq_h32", "n_seqs": lengths.numel(),
                "total_tokens": T, "max_len": int(lengths.max()), "H": H}
    return x, mask, cu, B, T, H, tokens, nbytes, desc


def fwd_leg(args, device, stream, wkv7_fwd, hbm_peak, peak_kind, max_over_ranks, barrier,
            rank, world):
    """K timed forward launches on resident inputs, then the host-buffer e2e pass."""
    x, mask, cu, B, T, H, tokens_per_step, fwd_bytes, desc = fwd_workload(args, rank)
    xd = {k: v.to(device) for k, v in x.items()}
    maskd = None if mask is None else mask.to(device)
    cud = None if cu is None else cu.to(device)
    N = xd["s0"].shape[0]
    D = xd["v"].shape[-1]
    o = torch.empty(B, T, H, D, dtype=torch.bfloat16, device=device)
    sT = torch.empty(N, H, D, D, dtype=torch.float32, device=device)

    if args.family == "gdn":
        def step():
            wkv7_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], s0=xd["s0"],
                     algo=args.algo, o=o, sT=sT)
    elif args.family == "sane":
        def step():
            wkv7_fwd(xd["r"], xd["w"], xd["k"], xd["v"], xd["a"], xd["b"], xd["tau"],
                     s0=xd["s0"], o=o, sT=sT)
    else:
        def step():
            wkv7_fwd(xd["r"], xd["w"], xd["k"], xd["v"], xd["a"], xd["b"], s0=xd["s0"],
                     mask=maskd, cu_seqlens=cud, algo=args.algo, o=o, sT=sT)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    barrier()
    torch.cuda.synchronize(device)
    clocks = ClockSampler(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    clock_info = clocks.stop()
    barrier()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1))
    ms_step = ms_total / args.steps
    value = world * tokens_per_step * args.steps / (ms_total / 1e3)

    achieved = fwd_bytes / (ms_step / 1e3) / 1e9
    kernel = "chunked" if args.algo in ("auto", "chunked") and D == 64 else "recurrent"
    if args.family == "gdn":
        kernel = "gdn_" + kernel
    elif args.family == "sane":
        kernel = "sane_recurrent"
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "peak_kind": f"{peak_kind} burst copy",
                "kernel": kernel,
                "traffic": profiled_traffic(f"fwd_{kernel}_{args.workload}"
                                            + ("" if D == 64 else f"_d{D}")),
                "algorithmic_bytes_per_launch": fwd_bytes}

    # End to end through the public call with host buffers: pinned H2D of every
    # input, the forward, D2H of o and the final state, every step.
    host = {k: v.pin_memory() for k, v in x.items()}
    dev = dict(xd)
    if mask is not None:
        host["mask"], dev["mask"] = mask.pin_memory(), maskd
    if cu is not None:
        host["cu_seqlens"], dev["cu_seqlens"] = cu.pin_memory(), cud
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    s_host = torch.empty(sT.shape, dtype=sT.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = o.numel() * o.element_size() + sT.numel() * sT.element_size()

    def e2e_step():
        for k in host:
            dev[k].copy_(host[k], non_blocking=True)
        step()
        o_host.copy_(o, non_blocking=True)
        s_host.copy_(sT, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(device)
    barrier()
    ev0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1)) / args.e2e_steps
    e2e = {"value": world * tokens_per_step / (ms_e2e / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e}
    return {"value": value, "ms_per_step": ms_step, "roofline": roofline, "e2e": e2e,
            "clocks": clock_info, "desc": desc}


def bwd_leg(args, device, stream, bwd_fn, hbm_peak, peak_kind, max_over_ranks, barrier, rank,
            gdn=False):
    """wkv7_bwd (or wkv7_gdn_bwd) on the B=8, T=4096, H=64 bf16 forward workload (random
    dL/do and dL/dS_T), inputs and workspace resident; up to 20 timed launches."""
    B, T, H = args.batch, FWD["T"], FWD["H"]
    if gdn:
        x = synth.gdn_inputs(B, T, H, dtype=torch.bfloat16,
                             seed=replicas.replica_seed(GDN_FWD["seed"], rank),
                             s0_std=GDN_FWD["s0_std"])
        names = ("q", "k", "v", "g", "beta")
    else:
        x = synth.fwd_inputs(B, T, H, dtype=torch.bfloat16,
                             seed=replicas.replica_seed(FWD["seed"], rank), s0_std=FWD["s0_std"])
        names = ("r", "w", "k", "v", "a", "b")
    gen = torch.Generator().manual_seed(replicas.replica_seed(620, rank))
    dout = torch.randn(B, T, H, 64, generator=gen).to(torch.bfloat16).to(device)
    dsT = (torch.randn(B, H, 64, 64, generator=gen) * 0.1).to(device)
    xd = {k: v.to(device) for k, v in x.items()}
    if gdn:
        from linear_attention_rnn_wkv7_b200 import library
        nbytes = int(library().wkv7_gdn_bwd_workspace_bytes(B, T, H, 64, 64, B, 0, 0))
    else:
        nbytes = wkv7_bwd_workspace_nbytes(B, T, H)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def step():
        bwd_fn(*(xd[n] for n in names), dout, s0=xd["s0"], dsT=dsT, workspace=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize(device)
    barrier()
    steps = max(1, min(args.steps, 20))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1)) / steps
    # WKV7: r,w,k,v,a,b and dout read, six gradients written (bf16); Gated DeltaNet:
    # q,k,v,dout read and dq,dk,dv written (bf16 vectors), g,beta read and dg,dbeta
    # written (bf16 scalars); s0 and dsT read and ds0 written (fp32).  The workspace
    # (checkpoints, u, and for Gated DeltaNet the fp32 substituted inputs) is not counted.
    per_th = (7 * 64 * 2 + 4 * 2) if gdn else 13 * 64 * 2
    nbytes = B * T * H * per_th + 3 * B * H * STATE_BYTES
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": ("gdn_" if gdn else "") + f"bwd_bf16_b{B}_t{T}_h{H}", "steps": steps,
            "ms_per_step": ms,
            "tokens/s": B * T / (ms / 1e3), "algorithmic_bytes_per_step": nbytes, "GB/s": gbs,
            "peak": hbm_peak, "frac": gbs / hbm_peak, "peak_kind": f"{peak_kind} burst copy",
            "workspace_bytes": ws.numel(), "gpu_launches": 4 * steps,
            "kernels": ("gdn_map_kernel + ckpt_kernel (forward, checkpoints) + bwd_kernel "
                        "(reverse) + gdn_chain_kernel" if gdn else
                        "prep_kernel + chunked_kernel (forward, state checkpoints) + "
                        "chunked_kernel (state gradient over the reversed sequences, dv) + "
                        "grad_kernel (per-chunk gradients)")}


def wkv7_bwd_workspace_nbytes(B, T, H):
    """The workspace of the kernel family wkv7_bwd picks for bf16 inputs."""
    from linear_attention_rnn_wkv7_b200.wkv7 import wkv7_bwd_workspace_bytes
    return wkv7_bwd_workspace_bytes(B, T, H, dtype=torch.bfloat16, algo="auto")


def decode_leg(device, stream, wkv7_step, hbm_peak, peak_kind, max_over_ranks, barrier, rank,
               gdn=False, D=64, sane=False):
    """256 consecutive wkv7_step (or wkv7_gdn_step, wkv7_sane_step) calls over 1024 x 32
    fp32 states (512 MiB, > L2).  Step inputs: 32 independently drawn step sets, used in
    turn; SANE clips every state after every 16th step (do_sane = step % 16 == 15)."""
    p = GDN_DEC if gdn else DEC
    B, H, steps = p["B"], p["H"] * 64 // D, p["steps"]
    state = synth.decode_state(B, H, K=D, V=D, seed=replicas.replica_seed(p["seed"], rank),
                               std=p["s0_std"]).to(device)
    sets = []
    names = ("q", "k", "v", "g", "beta") if gdn else ("r", "w", "k", "v", "a", "b")
    draw = synth.gdn_step_inputs if gdn else synth.decode_step_inputs
    for i in range(32):
        x = draw(B, H, K=D, V=D, dtype=torch.bfloat16,
                 seed=replicas.replica_seed(p["seed"], rank), step=i)
        sets.append(tuple(x[n].to(device) for n in names))
    o = torch.empty(B, H, D, dtype=torch.bfloat16, device=device)
    tau = synth.sane_tau(B, 1, H, replicas.replica_seed(p["seed"], rank))[:, 0].contiguous().to(device)

    def run(n):
        for i in range(n):
            if sane:
                wkv7_step(*sets[i % len(sets)], tau, i % 16 == 15, state, o=o)
            else:
                wkv7_step(*sets[i % len(sets)], state, o=o)

    run(3)
    torch.cuda.synchronize(device)
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    run(steps)
    ev1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1)) / steps
    nbytes = gdn_step_algorithmic_bytes(B, H, D) if gdn else step_algorithmic_bytes(B, H, D)
    if sane:
        nbytes += B * H * 4  # tau
    gbs = nbytes / (ms / 1e3) / 1e9
    tag = "" if D == 64 else f"_d{D}"
    fam = "gdn_" if gdn else "sane_" if sane else ""
    return {"workload": fam + f"step_bf16_b{B}_h{H}_256steps{tag}",
            "steps": steps,
            "us_per_step": 1e3 * ms,
            "algorithmic_bytes_per_step": nbytes, "GB/s": gbs, "peak": hbm_peak,
            "frac": gbs / hbm_peak, "peak_kind": f"{peak_kind} burst copy",
            "tokens/s": B / (ms / 1e3), "gpu_launches": steps,
            "traffic": profiled_traffic(fam + f"step_b{B}_h{H}{tag}")}


if __name__ == "__main__":
    main()
