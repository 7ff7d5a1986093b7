#!/usr/bin/env python3
"""Benchmark of the B200 KDA forward (prefill) library.

One step = one kda_fwd call over the whole workload (every chunk of every
sequence and head: gate cumsums, decayed K.K^T / Q.K^T blocks, UT transform,
W/U pseudo-values, the sequential fp32 state scan and the fused output).

Default workload: the 1M-token prefill (B = 1, T = 1,048,576, H = 32, d = 128,
C = 64, fp32 final state), inputs resident in HBM before the timed region
(52 GB, far larger than the 126 MB L2, so no flush is needed between steps).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--workload NAME] [--no-cpu-baseline] [--no-e2e]

Prints ONE JSON line on rank 0. Multi-GPU runs (torchrun, one rank per GPU;
``--gpus N`` without torchrun starts the N ranks itself) give each rank its own
independent workload (weak scaling), or with ``--split heads`` share one
workload's heads between the ranks (strong scaling). Either way there is no
collective on the data path: NCCL carries only the barrier and the
max-over-ranks time.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

D, C = 128, 64
# algorithmic HBM bytes per token and head: q, k, v, out (bf16 x 128 each),
# g (fp32 x 128), beta (fp32)
BYTES_PER_TOKEN_HEAD = 4 * 2 * D + 4 * D + 4
FLOPS_PER_TOKEN_HEAD = 6 * D * D + 3 * C * D + C * C   # the pages' count


def pages_flops(tokens: int, H: int) -> float:
    return float(tokens) * H * FLOPS_PER_TOKEN_HEAD


def decode_unit_bytes(state_dtype: str) -> int:
    """Algorithmic HBM bytes of one decode step for one (request, head): the 128 x 128 state
    read and written, q, k, v and out (bf16), g (fp32) and beta."""
    esz = 4 if state_dtype == "fp32" else 2
    return 2 * D * D * esz + 4 * D * 2 + D * 4 + 4


def bwd_flops_per_token_head(C: int = 16) -> float:
    """FLOPs per token and head of the backward's chunk algebra (kda_bwd, chunks of C
    tokens), each dense product counted once (the kernel's recomputation not counted):
    X, S, dQd, dKt, dD (state part), dKd and dS's two products at C x D x D each; dGl and
    the decay of dS at D x D; B, Aqk, dAqk and the four decayed products of dK and dQ at
    C (C + 1) / 2 x D; D, dD (intra part), dTp, dX at C x C x D; dAkk at 2 C^3."""
    fma = (8 * C * D * D + 2 * D * D + 7 * (C * (C + 1) // 2) * D + 4 * C * C * D + 2 * C ** 3)
    return 2.0 * fma / C


# algorithmic HBM bytes per token and head of the backward: q, k, v, dout read (bf16),
# g (fp32) and beta read; dq, dk, dv, dg (fp32) and dbeta written; the 64 KiB state
# checkpoint per 64 tokens written once and read once
BWD_BYTES_PER_TOKEN_HEAD = 4 * 2 * D + 4 * D + 4 + 4 * 4 * D + 4 + 2 * (4 * D * D) // 64


def fp32_alu_peak_tflops(sm_max_mhz: float, sms: int = 148) -> float:
    """fp32 FMA peak of the CUDA cores: 128 lanes per SM, 2 FLOP per FMA, at the SM clock."""
    return sms * 128 * 2 * sm_max_mhz * 1e6 / 1e12


def state_bytes(N, H, init_dt, final_dt) -> int:
    b = 0
    for dt in (init_dt, final_dt):
        if dt is not None:
            b += N * H * D * D * (4 if str(dt).endswith("float32") else 2)
    return b


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm_gbs=float(j["hbm_gbs"]), bf16_tflops=float(j["bf16_tflops"]),
                    bf16_tflops_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# the sources the timed kernel is compiled from
KERNEL_SOURCES = ("kda_fwd_tc.cu", "kda_internal.h", "sm100_ptx.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kimi_delta_attention_27_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode()); h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(token_heads: int):
    """DRAM bytes per launch from the committed ncu summary, scaled to this
    launch by token-heads; None when the kernel sources changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        j = json.load(f)
    if j.get("kernel_source_hash") != kernel_source_hash():
        return None, j.get("kernel")
    return float(j["dram_bytes_per_token_head"]) * token_heads, j.get("kernel")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu_index = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of every rank's ``x`` (the slowest rank's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Tokens/s of the whole job: every rank's tokens over the slowest rank's step time."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s workload: each rank processes its own independent
    batch (weak scaling), never a copy of another rank's."""
    return base_seed + 1000 * rank


def head_range(H: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of rank ``rank`` when ``world`` ranks share H heads (strong scaling):
    contiguous blocks, the first H % world ranks one head more."""
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def take_heads(inp: dict, h0: int, h1: int) -> dict:
    """The workload restricted to heads [h0, h1) (contiguous copies)."""
    d = dict(inp)
    for key in ("q", "k", "v", "g", "beta"):
        d[key] = inp[key][:, :, h0:h1].contiguous()
    if inp["h0"] is not None:
        d["h0"] = inp["h0"][:, h0:h1].contiguous()
    d["H"] = h1 - h0
    return d


def cpu_baseline_run(inp, tokens_per_step, steps=1, warmup=0):
    """Time the fp64 oracle, as it stands, on the host cores over the first
    ``tokens_per_step`` tokens of the workload (all heads). The last run's output
    is returned too (``out``), so that the timed GPU output can be compared with it."""
    import oracle
    sample = {}
    for name in ("q", "k", "v", "g", "beta"):
        sample[name] = inp[name][:1, :tokens_per_step].cpu().float().contiguous()
    if sample["g"].dim() == 3:   # one decay per token and head: the same on every channel
        sample["g"] = sample["g"][..., None].expand(*sample["g"].shape, D).contiguous()
    h0 = None if inp["h0"] is None else inp["h0"][:1].cpu().double()
    threads = os.cpu_count() or 1
    times = []
    eo = None
    for i in range(warmup + steps):
        t = time.perf_counter()
        eo, _ = oracle.kda_oracle(sample["q"], sample["k"], sample["v"], sample["g"], sample["beta"],
                                  inp["scale"], h0=h0, nthreads=threads)
        dt = time.perf_counter() - t
        if i >= warmup:
            times.append(dt)
    H = inp["H"]
    used = min(threads, H)  # the oracle runs one (sequence, head) unit per thread
    return dict(seconds=times, tokens=tokens_per_step, heads=H, threads=used, out=eo)


def parity_of_sample(out_gpu, inp, r) -> dict:
    """max|d out| / max|out| of the timed GPU output against the CPU-baseline oracle run
    ``r`` (the first tokens of row 0, all heads; for a packed batch only the tokens of
    its first sequence, where the oracle's single-sequence sample is the same problem)."""
    import numpy as np
    n = r["tokens"]
    if inp["cu_seqlens"] is not None:
        n = min(n, int(inp["lengths"][0]))
    ref = np.asarray(r["out"])[:, :n]
    got = out_gpu[:1, :n].float().cpu().numpy()
    err = float(np.abs(got - ref).max() / max(float(np.abs(ref).max()), 1e-30))
    return {"out_rel_err": err, "bar": 1e-2, "tokens": n, "heads": r["heads"],
            "sample": f"first {n} tokens of row 0, every head, against the fp64 oracle "
                      "(the CPU-baseline run)"}


def reference_arm(args, world, rank):
    """The oracle, timed on this machine's host cores, on a bounded sample of the
    same workload per step."""
    if rank != 0:
        return 0
    from kimi_delta_attention_27_b200.inputs import make_inputs
    cfg_name = args.workload
    tokens = args.ref_tokens
    # a bounded sample of the workload: its first ``tokens`` tokens, every head
    inp = make_inputs(cfg_name, device="cpu", T=tokens, B=1, lengths=None)
    r = cpu_baseline_run(inp, tokens, steps=args.steps, warmup=args.warmup)
    per_step = statistics.mean(r["seconds"])
    value = tokens / per_step
    sample = f"first {tokens} tokens of all {r['heads']} heads of {cfg_name}, fp64 oracle"
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": workload_config(cfg_name, world, note="oracle sample per step: " + sample),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["threads"],
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "tflops": pages_flops(tokens, r["heads"]) / per_step / 1e12,
    }
    print(json.dumps(line), flush=True)
    return 0


METRIC = "KDA fwd prefill tokens/s and TFLOP/s (6Td^2+3TCd+TC^2) vs B200 bf16 peak"

WORKLOAD_TEXT = {
    "t1m_h32": "1M-token prefill: B=1, T=1048576, H=32, d=128, C=64, fp32 final state",
    "t4k_h32": "B=1, T=4096, H=32, d=128, C=64, fp32 initial and final state",
    "varlen16_h32": "varlen: 16 sequences U[512,16384] via cu_seqlens, H=32, d=128, fp32 states",
    "b8_t8k_h32": "B=8, T=8192, H=32, d=128, bf16 initial and final state, slow decay",
    "t256_h1": "B=1, T=256, H=1, d=128, fp32 final state",
}


def workload_config(name, world, note=None, split="none"):
    from kimi_delta_attention_27_b200.inputs import CONFIGS
    c = CONFIGS[name]
    strong = split == "heads"
    per = c["B"] if c.get("lengths") is None else c["lengths"][0]
    cfg = {"workload": WORKLOAD_TEXT.get(name, name), "name": name,
           "global_batch": per if strong else per * world,
           "seq_len": c["T"], "heads": c["H"], "head_dim": D, "chunk": C,
           "parallelism": (f"heads split over {world} ranks" if strong else f"dp{world}") if world > 1
           else "single-gpu",
           "l2": "inputs larger than L2 (no flush needed)"}
    if note:
        cfg["note"] = note
    return cfg


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default="t1m_h32")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=4096,
                    help="tokens (all heads) in the oracle's CPU-baseline sample")
    ap.add_argument("--ref-tokens", type=int, default=8192,
                    help="tokens (all heads) per reference-arm step")
    ap.add_argument("--e2e-slice", type=int, default=1 << 16,
                    help="tokens per host->device slice in the end-to-end measurement")
    ap.add_argument("--split", default="none", choices=["none", "heads"],
                    help="none: each rank runs its own copy of the workload (weak scaling); "
                         "heads: the ranks share the workload's heads (strong scaling)")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward pass (kda_bwd) on the workload instead; prints its own line")
    ap.add_argument("--segmented", type=int, default=0, metavar="TOKENS",
                    help="time kda_fwd_segmented with pieces of TOKENS tokens instead of kda_fwd")
    ap.add_argument("--heads", type=int, default=0, help="override the workload's number of heads")
    ap.add_argument("--gate", default="fp32", choices=["fp32", "bf16", "per_token"],
                    help="gate input of the timed forward (kda_fwd_ex for bf16 and per_token)")
    ap.add_argument("--decode", default=None, metavar="BxH[:bf16]",
                    help="time the single-token decode step instead (e.g. 256x32 or 256x32:bf16); "
                         "prints its own line, not the prefill metric")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.decode:
        return decode_main(args)
    if args.bwd:
        return bwd_main(args)

    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_under_torchrun(args.gpus)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        if rank == 0:
            print(f"bench.py: --gpus {args.gpus} but {world} ranks were started; no line printed",
                  file=sys.stderr)
        return 2
    if args.impl == "reference":
        return reference_arm(args, world, rank)

    import torch
    world, rank, local = dist_setup()
    import kimi_delta_attention_27_b200 as kda
    from kimi_delta_attention_27_b200.inputs import CONFIGS, make_inputs

    name = args.workload
    cfg = dict(CONFIGS[name])
    strong = args.split == "heads"
    if strong:
        # one workload (the same seed on every rank), this rank's heads of it
        full = make_inputs(name, device="cuda")
        h_lo, h_hi = head_range(full["H"], world, rank)
        inp = take_heads(full, h_lo, h_hi)
        H_all = full["H"]
        del full
        torch.cuda.empty_cache()
    else:
        over = {"H": args.heads} if args.heads else {}
        inp = make_inputs(name, device="cuda", seed=rank_seed(cfg["seed"], rank), **over)
        H_all = inp["H"]
    if args.gate == "bf16":
        inp["g"] = inp["g"].to(torch.bfloat16)
    elif args.gate == "per_token":
        inp["g"] = inp["g"][..., 0].contiguous()
    H, N, tokens = inp["H"], inp["N"], inp["B"] * inp["T"]
    final_dt = inp["final_dtype"]
    out = torch.empty_like(inp["v"])
    hT = None if final_dt is None else torch.empty((N, H, D, D), dtype=final_dt, device="cuda")
    stream = torch.cuda.current_stream()

    seg_ws = None
    if args.segmented:
        seg_ws = torch.empty(max(1, kda.segmented_workspace_bytes(inp["B"], inp["T"], H, args.segmented)),
                             dtype=torch.uint8, device="cuda")

    def step():
        if args.segmented:
            kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], args.segmented,
                                  inp["scale"], initial_state=inp["h0"], final_state=hT, out=out,
                                  workspace=seg_ws)
        else:
            kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["scale"],
                        cu_seqlens=inp["cu_seqlens"], initial_state=inp["h0"], final_state=hT,
                        out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    sampler = current_gpu_sampler() if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True); t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    t_start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    ms_per_step = total_ms / args.steps
    # weak: every rank processed its own tokens; strong: the ranks shared one workload's tokens
    value = (tokens / (ms_per_step / 1e3)) if strong else whole_job_value(world, tokens, ms_per_step)
    flops = pages_flops(tokens, H_all) if strong else world * pages_flops(tokens, H)
    peaks = load_peaks()
    # a bf16 gate saves 256 B per token-head, a per-token one 508 B
    bytes_th = BYTES_PER_TOKEN_HEAD - {"fp32": 0, "bf16": 2 * D, "per_token": 4 * D - 4}[args.gate]
    alg_bytes = tokens * H * bytes_th + state_bytes(
        N, H, None if inp["h0"] is None else inp["h0"].dtype, final_dt)
    avg_launch_s = statistics.mean(launch_ms) / 1e3
    achieved_gbs = alg_bytes / avg_launch_s / 1e9
    traffic, prof_kernel = profiled_traffic(tokens * H)
    if args.segmented or args.gate != "fp32":
        # the committed DRAM counters are the plain kernel's
        traffic = None
        prof_kernel = ("kda_fwd_segmented (affine run, scan, forward run)" if args.segmented
                       else f"kda_fwd_ex ({args.gate} gate)")

    # ---- end to end: pinned host buffers -> device -> kda_fwd -> host, per step
    e2e = None
    if not args.no_e2e and args.gate == "fp32" and not args.segmented:
        e2e = e2e_run(args, inp, world, rank, strong=strong)

    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # size the sample for roughly 10-30 s of host work: probe, then scale up
        ntok = min(args.cpu_tokens, tokens)
        r = cpu_baseline_run(inp, ntok)
        secs = r["seconds"][0]
        if secs < 8.0 and ntok < tokens:
            ntok = int(min(tokens, ntok * max(1.0, 12.0 / max(secs, 1e-3))))
            ntok = max(64, ntok // 64 * 64)
            r = cpu_baseline_run(inp, ntok)
            secs = r["seconds"][0]
        cpu = {"value": r["tokens"] / secs, "unit": "tokens/s", "cores": r["threads"],
               "kind": "oracle",
               "sample": f"first {r['tokens']} tokens of all {r['heads']} heads of the workload "
                         f"({secs:.1f} s, {os.cpu_count()} host cores, one thread per head)"}
        parity = parity_of_sample(out, inp, r)

    del inp
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "strong" if strong else "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(name, world, split=args.split), heads=H_all, gate=args.gate,
                           **({"segment_len": args.segmented} if args.segmented else {})),
            "tflops": flops / (ms_per_step / 1e3) / 1e12,
            "frac_bf16_peak": flops / (ms_per_step / 1e3) / 1e12 / peaks["bf16_tflops"] / world,
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
                         "traffic": traffic, "peak_source": peaks["source"],
                         "kernel": prof_kernel or "kda_fwd",
                         "alg_bytes_per_launch": alg_bytes,
                         "avg_launch_ms": avg_launch_s * 1e3},
            "cpu_baseline": cpu, "e2e": e2e, "parity": parity,
            "gpu_launches": args.steps * (3 if args.segmented else 1),
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def current_gpu_sampler():
    """A ClockSampler for this process's GPU, named by UUID so that nvidia-smi's
    numbering cannot pick another GPU."""
    import torch
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    uuid = str(getattr(props, "uuid", ""))
    return ClockSampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else
                        (uuid or torch.cuda.current_device()))


def bwd_main(args):
    """The backward pass (kda_bwd) on one GPU over the workload (default: the 4K-token one),
    with seeded bf16 output gradients and an fp32 final-state gradient."""
    import torch
    import kimi_delta_attention_27_b200 as kda
    from kimi_delta_attention_27_b200.inputs import make_inputs
    name = args.workload if args.workload != "t1m_h32" else "t4k_h32"
    over = {"H": args.heads} if args.heads else {}
    inp = make_inputs(name, device="cuda", **over)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(77)
    dout = torch.randn(inp["v"].shape, generator=gen, device="cuda").to(torch.bfloat16)
    dhT = torch.randn((inp["N"], inp["H"], D, D), generator=gen, device="cuda")
    H, tokens = inp["H"], inp["B"] * inp["T"]
    ws = torch.empty(kda.bwd_workspace_bytes(tokens, inp["N"], H), dtype=torch.uint8, device="cuda")

    def step():
        return kda.kda_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], dout, inp["scale"],
                           cu_seqlens=inp["cu_seqlens"], initial_state=inp["h0"], dfinal_state=dhT, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = current_gpu_sampler()
    sampler.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True); t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1) / args.steps
    peaks = load_peaks()
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else io.StringIO("{}") as f:
        sm_max = float(json.load(f).get("sm_max_mhz", 1965.0))
    flops = tokens * H * bwd_flops_per_token_head()
    achieved = flops / (ms / 1e3) / 1e12
    peak = fp32_alu_peak_tflops(sm_max)
    line = {
        "metric": "KDA bwd tokens/s (dq, dk, dv, dg, dbeta, dh0)", "value": tokens / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "dtype": "f32", "data": "synthetic",
        "config": dict(workload_config(name, 1), heads=H),
        "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None, "kernel": "kda::bwd::kda_bwd_kernel",
                     "flops_per_token_head": bwd_flops_per_token_head(),
                     "peak_source": f"derived: 148 SMs x 128 fp32 lanes x 2 x {sm_max:.0f} MHz",
                     "hbm_bytes_per_token_head": BWD_BYTES_PER_TOKEN_HEAD,
                     "hbm_gbs": tokens * H * BWD_BYTES_PER_TOKEN_HEAD / (ms / 1e3) / 1e9,
                     "hbm_peak_gbs": peaks["hbm_gbs"]},
        "gpu_launches": args.steps * 1, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def decode_main(args):
    """The decode step (kda_decode) on one GPU: B requests x H heads, one token per
    request per step, states updated in place. Bound by HBM: each (request, head)
    reads and writes its 128 x 128 state."""
    import torch
    import kimi_delta_attention_27_b200 as kda
    from kimi_delta_attention_27_b200.inputs import make_inputs
    spec, _, sdt = args.decode.partition(":")
    B, H = (int(x) for x in spec.lower().split("x"))
    sdt = sdt or "fp32"
    steps = args.steps
    # one token per request per step; inputs for all timed and warm-up steps are made up front
    nstep = args.warmup + steps
    inp = make_inputs({"B": B, "T": nstep, "H": H, "lengths": None, "g_mu": 3.0, "init": sdt,
                       "final": sdt, "seed": 90}, device="cuda")
    toks = [tuple(inp[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta")) for t in range(nstep)]
    S = inp["h0"]
    out = torch.empty((B, H, D), dtype=torch.bfloat16, device="cuda")
    del inp
    stream = torch.cuda.current_stream()

    def step(t):
        q, k, v, g, beta = toks[t]
        kda.kda_decode(q, k, v, g, beta, state_in=S, state_out=S, out=out)

    for t in range(args.warmup):
        step(t)
    torch.cuda.synchronize()
    sampler = current_gpu_sampler()
    sampler.start()
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True); t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    t0.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        step(args.warmup + i)
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    clocks = sampler.stop()
    ms_per_step = t0.elapsed_time(t1) / steps
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    unit_bytes = decode_unit_bytes(sdt)
    alg_bytes = B * H * unit_bytes
    peaks = load_peaks()
    achieved = alg_bytes / (launch_ms / 1e3) / 1e9
    line = {
        "metric": "KDA decode step tokens/s (one token per request, all heads)", "value": B / (ms_per_step / 1e3),
        "unit": "tokens/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "dtype": "f32" if sdt == "fp32" else "bf16", "data": "synthetic",
        "config": {"workload": f"decode step: {B} requests x {H} heads, {sdt} states updated in place",
                   "requests": B, "heads": H, "state_dtype": sdt,
                   "l2": "states larger than L2 (no flush needed)" if alg_bytes > 126e6 else "states fit in L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None, "peak_source": peaks["source"],
                     "kernel": f"kda_decode_kernel<{'true' if sdt == 'fp32' else 'false'}>",
                     "alg_bytes_per_launch": alg_bytes, "bytes_per_unit": unit_bytes, "avg_launch_ms": launch_ms},
        "gpu_launches": steps, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def relaunch_under_torchrun(n: int) -> int:
    """``--gpus N`` started without torchrun: run this command again as N ranks (one per
    GPU, rendezvous on 127.0.0.1) and return their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.call(cmd)


def e2e_run(args, inp, world, rank, strong=False):
    """Same metric through the public API with host buffers: every step streams
    the whole sequence through the device in slices (chunked prefill, state
    carried between slices), copying each slice's inputs host->device from
    pinned memory and its output device->host inside the timed region. The
    host holds one slice of synthetic data, reused for every slice (the
    sequence is periodic; the work per token is the same)."""
    import torch
    import kimi_delta_attention_27_b200 as kda
    if inp["cu_seqlens"] is not None or inp["B"] != 1:
        return None
    T, H = inp["T"], inp["H"]
    Ls = min(args.e2e_slice, T)
    nsl = T // Ls
    host = {}
    for key in ("q", "k", "v", "g", "beta"):
        host[key] = inp[key][:, :Ls].cpu().pin_memory()
    out_h = torch.empty((1, Ls, H, D), dtype=torch.bfloat16).pin_memory()
    dev = [{k: torch.empty_like(v, device="cuda") for k, v in host.items()} for _ in range(2)]
    out_d = [torch.empty((1, Ls, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    state = [torch.zeros((1, H, D, D), dtype=torch.float32, device="cuda") for _ in range(2)]
    copy_s = torch.cuda.Stream()
    back_s = torch.cuda.Stream()
    comp_s = torch.cuda.current_stream()
    h2d = sum(t.numel() * t.element_size() for t in host.values()) * nsl
    d2h = out_h.numel() * out_h.element_size() * nsl

    def one_step():
        ready = [torch.cuda.Event() for _ in range(nsl)]
        computed = [torch.cuda.Event() for _ in range(nsl)]
        done = [torch.cuda.Event() for _ in range(nsl)]
        with torch.cuda.stream(copy_s):
            for key in host:
                dev[0][key].copy_(host[key], non_blocking=True)
            ready[0].record(copy_s)
        for i in range(nsl):
            b = i % 2
            if i + 1 < nsl:
                with torch.cuda.stream(copy_s):
                    if i >= 1:
                        copy_s.wait_event(done[i - 1])
                    for key in host:
                        dev[1 - b][key].copy_(host[key], non_blocking=True)
                    ready[i + 1].record(copy_s)
            comp_s.wait_event(ready[i])
            kda.kda_fwd(dev[b]["q"], dev[b]["k"], dev[b]["v"], dev[b]["g"], dev[b]["beta"],
                        inp["scale"], initial_state=None if i == 0 else state[(i - 1) % 2],
                        final_state=state[i % 2], out=out_d[b])
            computed[i].record(comp_s)
            with torch.cuda.stream(back_s):
                back_s.wait_event(computed[i])
                out_h.copy_(out_d[b], non_blocking=True)
                done[i].record(back_s)
            if i >= 1:
                comp_s.wait_event(done[i - 1])   # out_d[1 - b] is free again
        comp_s.wait_event(done[nsl - 1])
        torch.cuda.current_stream().synchronize()

    one_step()  # warm-up
    steps = max(1, min(args.steps, 3))
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True); t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp_s)
    for _ in range(steps):
        one_step()
    t1.record(comp_s)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world) / steps
    return {"value": (1 if strong else world) * nsl * Ls / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": steps, "slice_tokens": Ls,
            "how": "public binding kda_fwd over the sequence in slices with state carry; "
                   "pinned host inputs copied per slice on a copy stream (double-buffered), "
                   "output copied back per slice. The host holds one slice of the workload's "
                   "synthetic inputs and streams it for every slice: the bytes copied and the work "
                   "per slice are the full sequence's, the values are not the workload's own"}


if __name__ == "__main__":
    sys.exit(main())
