#!/usr/bin/env python
"""Benchmark of the FP8 x MXFP4 MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl cuda|reference]

A step is one whole layer forward (router, top-k + gates, dispatch + E4M3
quantisation, grouped linear1 + SwiGLU + requant, grouped linear2, combine) over
one batch of T synthetic tokens already resident in HBM.  The default workload
is the DeepSeek-V3-shaped large-batch prefill (T=32768, H=7168, I=2048, E=256
routed + 1 shared, k=8); the same run also times the metric's other batch points
(T=1, T=512 and the Zipf-skewed T=8192 layer) on the same expert weights and
reports them under "per_T".  With N > 1
(launched by torchrun) every rank runs an independent replica on its own GPU and
its own token batch: the layer has no exchange step on one device, so there is
no collective on the data path (weak scaling); ranks only meet for the timing
barrier and the max-over-ranks reduction.

`--impl reference` times the CPU oracle (float64 numpy, oracle/) on a bounded
token sample of the same workload, on rank 0.
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

from fp8_fp4_moe_b200 import inputs as I  # noqa: E402

METRIC = "MoE-layer tokens/s and TFLOPS (% FP8 peak / % HBM) at T=1/512/8192/32768"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CPU_SAMPLE_TOKENS = {"tiny": 64, "mixtral": 8, "dsv3_t1": 1, "dsv3_t512": 2, "dsv3_t8192_zipf": 2,
                     "dsv3_t32768": 2}
REF_STEP_TOKENS = {"tiny": 64, "mixtral": 1, "dsv3_t1": 1, "dsv3_t512": 1, "dsv3_t8192_zipf": 1,
                   "dsv3_t32768": 1}


def kernels_per_forward(w) -> int:
    """router, top-k, column scan, expert scan, scatter, linear1, linear2, combine; with at
    most 32 tokens top-k and the two scans are one kernel, and with at most 32 (token, 256-channel
    slice) items the scatter runs in it too (prepare is skipped: weights static)."""
    if w.T <= 32:
        return 5 if w.T * ((w.H + 255) // 256) <= 32 else 6
    return 8


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="dsv3_t32768", choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-t", action="store_true",
                    help="time only the named workload (by default the T = 32768 headline also times the "
                         "T = 1 / 512 / 8192 points of the metric on the same weights)")
    ap.add_argument("--no-graph", action="store_true", help="launch kernels one by one (no CUDA graph replay)")
    ap.add_argument("--opt", action="append", default=[], metavar="NAME=VALUE",
                    help="plan option, e.g. SWAP_ROWS=64 or MAX_SMS=74 (MOE_OPT_<NAME>); repeatable")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (smaller cases of the same kernels, e.g. for ncu captures)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (with --tokens: a decode-shaped case with fewer experts in HBM)")
    return ap.parse_args()


def workload(args) -> I.Workload:
    w = I.WORKLOADS[args.workload]
    if args.experts is not None:
        w = w.with_experts(args.experts)
    return w if args.tokens is None else w.with_tokens(args.tokens)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """Hash of the files the grouped GEMM kernels are compiled from (their code, helpers and
    argument layout): a recorded DRAM-traffic figure is used only while it matches."""
    h = hashlib.sha256()
    for name in ("gemm_sm100.cu", "common.cuh", "kernels.h"):
        with open(os.path.join(ROOT, "fp8_fp4_moe_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if still current."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(f"{kernel}@{workload}")
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return float(ent["bytes_per_launch"])


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_ids):
        self.gpu_ids = gpu_ids
        self.proc = None
        # raw samples (the JSON line carries their summary); MOE_BENCH_CLOCKS_DIR keeps them
        out_dir = os.environ.get("MOE_BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"moe_bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", ",".join(map(str, self.gpu_ids)), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1])]
        mx = max((num(r[2]) or 0) for r in rows)
        loaded = [s for s in sm if s > 0.5 * mx] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- helpers

def algorithmic_counts(w: I.Workload, counts):
    """FLOPs and bytes of the layer and of each GEMM launch for the routed counts."""
    touched = int(np.count_nonzero(counts))
    rows = int(np.sum(counts))
    H, I_ = w.H, w.I
    w1_bytes = 2 * I_ * H // 2 + 2 * I_ * H // 32
    w2_bytes = H * I_ // 2 + H * I_ // 32
    return {
        "layer_flops": w.flops(),
        "layer_bytes": touched * (w1_bytes + w2_bytes) + w.E * H * 4 + w.T * H * 2 * 2,
        "linear1_flops": 2.0 * rows * H * 2 * I_,
        "linear1_bytes": touched * w1_bytes + rows * H + rows * I_,
        "linear2_flops": 2.0 * rows * I_ * H,
        "linear2_bytes": touched * w2_bytes + rows * I_ + rows * H * 2,
        "touched_experts": touched,
    }


def cpu_baseline(w: I.Workload, n_tokens: int):
    """The oracle as it stands, on all host cores, on a token sample of the workload."""
    from threadpoolctl import threadpool_info

    from oracle import moe as M
    x, W_r, bias = I.make_routing_inputs(w, 0)
    rng = np.random.default_rng(0)
    tokens = np.sort(rng.choice(w.T, size=min(n_tokens, w.T), replace=False))
    x_np = x.view(torch.int16).numpy().view(np.uint16)
    # expert weights of only the experts the sample touches (the rest are never read)
    ids, _, _ = M.route(x_np[tokens], W_r.numpy(), bias.numpy(), w.k)
    need = sorted(set(ids.ravel().tolist()) | ({w.E} if w.shared else set()))
    W1, W1s, W2, W2s = I.make_expert_weights(w, 0, device="cpu", experts=need)
    t0 = time.perf_counter()
    M.forward(x_np, W_r.numpy(), bias.numpy(), W1.numpy(), W1s.numpy(), W2.numpy(), W2s.numpy(), k=w.k,
              shared=w.shared, tokens=tokens)
    dt = time.perf_counter() - t0
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    return {"value": len(tokens) / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{w.name}: routing + dispatch of all {w.T} tokens, expert FFN + combine of "
                      f"{len(tokens)} sampled tokens ({len(need)} experts), float64 numpy; {dt:.1f} s"}


# ----------------------------------------------------------------------------- ranks

def token_seed(rank: int) -> int:
    """Seed of a rank's token batch: rank 0 times the workload's own tokens, the other replicas
    distinct batches of the same shape (weights and router are shared)."""
    return 0 if rank == 0 else 1000 + rank


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of the ranks' values (every rank calls it, in the same order)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def init_ranks(world: int, local_rank: int, need_gpu: bool) -> None:
    """One process per GPU over NCCL; without a GPU (the CPU reference arm) over gloo."""
    if world <= 1:
        return
    import datetime
    timeout = datetime.timedelta(seconds=120)
    if need_gpu or torch.cuda.is_available():
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local_rank))
    else:
        torch.distributed.init_process_group("gloo", timeout=timeout)


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return None
    from threadpoolctl import threadpool_info

    from oracle import moe as M
    w = workload(args)
    x, W_r, bias = I.make_routing_inputs(w, 0)
    x_np = x.view(torch.int16).numpy().view(np.uint16)
    n_tok = REF_STEP_TOKENS[args.workload]
    rng = np.random.default_rng(0)
    samples = [np.sort(rng.choice(w.T, size=min(n_tok, w.T), replace=False))
               for _ in range(args.steps + args.warmup)]
    need = set()
    for s in samples:
        ids, _, _ = M.route(x_np[s], W_r.numpy(), bias.numpy(), w.k)
        need |= set(ids.ravel().tolist())
    if w.shared:
        need.add(w.E)
    W1, W1s, W2, W2s = I.make_expert_weights(w, 0, device="cpu", experts=sorted(need))
    args_np = (x_np, W_r.numpy(), bias.numpy(), W1.numpy(), W1s.numpy(), W2.numpy(), W2s.numpy())
    for s in samples[:args.warmup]:
        M.forward(*args_np, k=w.k, shared=w.shared, tokens=s)
    t0 = time.perf_counter()
    done = 0
    for s in samples[args.warmup:]:
        M.forward(*args_np, k=w.k, shared=w.shared, tokens=s)
        done += len(s)
    dt = time.perf_counter() - t0
    value = done / dt
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.description, "T": w.T, "tokens_per_step": n_tok,
                   "parallelism": "none (CPU oracle, rank 0)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{w.name}: per step routing + dispatch of all {w.T} tokens and the expert "
                                   f"FFN + combine of {n_tok} sampled token(s), float64 numpy"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


# ----------------------------------------------------------------------------- CUDA arm

# The metric is quoted at T = 1 / 512 / 8192 / 32768 on the DeepSeek-V3-shaped layer (the "Mega
# MoE" batch points).  The headline line times the largest of them; the other three share its
# expert weights (same H, I, E, k, shared expert and weight seed) and are timed in the same run.
COMPANIONS = {"dsv3_t32768": ["dsv3_t1", "dsv3_t512", "dsv3_t8192_zipf"]}
# short points run more steps so that the timed region is long enough to read the clocks from
MIN_TIMED_S = 0.25
MAX_POINT_STEPS = 2000


def make_weights(w: I.Workload, dev):
    W1, W1s, W2, W2s = I.make_expert_weights(w, 0, device=dev)
    torch.cuda.empty_cache()        # return the quantiser's temporaries: only live tensors stay on the device
    return dict(W1=W1, W1_scales=W1s, W2=W2, W2_scales=W2s)


def roofline_of(w, alg, avg, fused, peaks, peak_src, bf16_key, workload_key, resized):
    """Roofline of the dominant kernel from the per-kernel CUDA-event times `avg` (ms)."""
    fp8 = 2.0 * peaks[bf16_key]
    hbm = peaks["hbm_gbs"]
    dominant = max(avg, key=avg.get)
    dom_ms = avg[dominant]
    if fused:
        # one persistent kernel for the whole forward: its time is reported as the first phase
        dominant, dom_ms = "fused_forward", sum(avg.values())
    if dominant in ("linear1", "linear2", "fused_forward"):
        flops = alg[f"{dominant}_flops"] if not fused else w.flops()
        byts = alg[f"{dominant}_bytes"] if not fused else alg["layer_bytes"]
        if flops / byts > fp8 * 1e12 / (hbm * 1e9):
            roof = {"bound": "tensor", "achieved": flops / (dom_ms * 1e-3) / 1e12, "peak": fp8,
                    "unit": "TFLOP/s", "algorithmic": flops}
        else:
            roof = {"bound": "hbm", "achieved": byts / (dom_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                    "algorithmic": byts}
    else:
        byts = alg["layer_bytes"]
        roof = {"bound": "hbm", "achieved": byts / (dom_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                "algorithmic": byts}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dominant
    roof["kernel_ms"] = dom_ms
    roof["peak_source"] = (f"{peak_src} MEASURED_PEAKS.json: 2 x {bf16_key} (FP8 = 2 x BF16 dense)"
                           if roof["unit"] == "TFLOP/s" else f"{peak_src} MEASURED_PEAKS.json hbm_gbs")
    roof["traffic"] = ncu_traffic(dominant, workload_key) if not resized else None
    return roof


def measure(w: I.Workload, weights: dict, args, rank, world, dev, steps: int, resized: bool, workload_key: str):
    """Time `steps` forwards of workload `w` (inputs resident in HBM, L2 flushed between steps),
    then the per-kernel event pass and the end-to-end pass.  Every rank calls it in the same order
    (barriers and max-over-ranks reductions).  Returns rank 0's record (None elsewhere)."""
    from fp8_fp4_moe_b200 import binding
    _, W_r, bias = I.make_routing_inputs(w, 0)
    x, _, _ = I.make_routing_inputs(w, token_seed(rank))
    d = dict(x=x.to(dev), W_router=W_r.to(dev), bias=bias.to(dev), **weights)
    del x
    plan = binding.Plan(w.T, w.H, w.I, w.E, w.k, w.shared, device=dev)
    # launch the forward's kernels as one recorded CUDA graph (per pointer set)
    plan.set_option(binding.MOE_OPT_GRAPH, 0 if args.no_graph else 1)
    for kv in args.opt:
        name, value = kv.split("=", 1)
        plan.set_option(getattr(binding, "MOE_OPT_" + name.upper()), int(value))
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # Expert weights are model state: their UE8M0 scales are re-laid out once
    # (timed here, reported separately) and reused by every timed forward.
    plan.set_option(binding.MOE_OPT_STATIC_WEIGHTS, 1)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    plan.prepare_weights(d["W1_scales"], d["W2_scales"])
    ev1.record(stream)
    ev1.synchronize()
    prepare_ms = ev0.elapsed_time(ev1)

    for _ in range(args.warmup):
        plan.forward(**d, out=out)
    code, detail = plan.check_status()
    if code != 0:
        raise RuntimeError(f"device status {code} {detail}")
    counts = plan.region("counts").cpu().numpy()

    sampler = ClockSampler(list(range(world)) if rank == 0 else [local_index(dev)])
    if rank == 0:
        sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    step_ms = []
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(1)                                   # L2 scrub between timed steps (not timed)
        ev[i][0].record(stream)
        plan.forward(**d, out=out)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if rank == 0 else None
    code, detail = plan.check_status()
    if code != 0:
        raise RuntimeError(f"device status {code} {detail}")
    total_ms = max_over_ranks(sum(step_ms), world, dev)

    # Per-kernel times for the roofline: CUDA events recorded on the forward's stream
    # between its kernels (graph replay is off while the events are on).
    plan.set_option(binding.MOE_OPT_PHASE_EVENTS, 1)
    phases = []
    for _ in range(min(steps, 20)):
        flush.fill_(1)
        plan.forward(**d, out=out)
        phases.append(plan.phase_times())
    plan.set_option(binding.MOE_OPT_PHASE_EVENTS, 0)
    plan.set_option(binding.MOE_OPT_GRAPH, 0 if args.no_graph else 1)
    for kv in args.opt:
        name, value = kv.split("=", 1)
        plan.set_option(getattr(binding, "MOE_OPT_" + name.upper()), int(value))

    # end to end through the public API: pinned host x -> device, forward, out -> pinned host
    # Every step copies its tokens host -> device, runs the layer and copies the
    # output back.  Steps are pipelined over three streams (copy in, compute,
    # copy out) with double-buffered device tensors, as a serving loop would.
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(w, plan, d, args, world, dev, stream, steps)
    del flush
    if rank != 0:
        del plan, d, out
        torch.cuda.empty_cache()
        return None

    tile_rows = plan.get_option(binding.MOE_OPT_TILE_ROWS)
    zero_pad = plan.get_option(binding.MOE_OPT_ZERO_PAD)
    l2_rows = plan.get_option(binding.MOE_OPT_L2_TILE_ROWS)
    alg = algorithmic_counts(w, counts)
    avg = {k: statistics.mean(p[k] for p in phases) for k in phases[0]}
    ms = total_ms / steps
    fused = any(o.replace(" ", "").upper() == "FUSED=1" for o in args.opt)
    peaks, peak_src = load_peaks()
    # Tensor peak: measured bf16 x the nominal FP8:BF16 dense ratio of 2.  The burst
    # figure when the SM clock stayed at its maximum during the timed steps, the
    # sustained (power-capped) figure otherwise.
    at_max = bool(clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz")
                  and clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"])
    bf16_key = "bf16_tflops" if at_max else "bf16_tflops_sustained"
    fp8 = 2.0 * peaks[bf16_key]
    hbm = peaks["hbm_gbs"]
    roof = roofline_of(w, alg, avg, fused, peaks, peak_src, bf16_key, workload_key, resized)
    rec = {
        "workload": w.description + ("" if not resized else f" (resized to T={w.T}, E={w.E})"),
        "T": w.T,
        "steps": steps,
        "ms_per_step": ms,
        "tokens_per_s": world * w.T / (ms * 1e-3),
        "tflops": w.flops() / (ms * 1e-3) / 1e12,
        "tflops_frac_fp8": w.flops() / (ms * 1e-3) / 1e12 / fp8,
        "fp8_peak_tflops": fp8,
        "hbm_gbs": alg["layer_bytes"] / (ms * 1e-3) / 1e9,
        "hbm_frac": alg["layer_bytes"] / (ms * 1e-3) / 1e9 / hbm,
        "layer_flops": alg["layer_flops"],
        "layer_bytes": alg["layer_bytes"],
        "phases_ms": avg,
        "roofline": roof,
        "e2e": e2e,
        # the fused option is one kernel per forward
        "gpu_launches": (1 if fused else kernels_per_forward(w)) * steps,
        "clocks": clocks,
        "max_expert_load_ratio": float(counts[:w.E].max() / (w.T * w.k / w.E)),
        "touched_experts": alg["touched_experts"],
        "weight_scales_prepare_ms": prepare_ms,
        "gemm_tiles": {"rows": tile_rows, "zero_padded": zero_pad == 1, "linear2_weight_rows": l2_rows},
    }
    del plan, d, out
    torch.cuda.empty_cache()
    return rec


def local_index(dev) -> int:
    return dev.index if dev.index is not None else 0


def measure_e2e(w, plan, d, args, world, dev, stream, steps):
    nbuf = 2
    x_host = d["x"].cpu().pin_memory()
    out_host = [torch.empty(w.T, w.H, dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
    x_dev = [torch.empty_like(d["x"]) for _ in range(nbuf)]
    out_dev = [torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev) for _ in range(nbuf)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_done = [torch.cuda.Event() for _ in range(nbuf)]
    fwd_done = [torch.cuda.Event() for _ in range(nbuf)]
    out_done = [torch.cuda.Event() for _ in range(nbuf)]
    d_e2e = dict(d)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(s_in)
    stream.wait_event(t_start)
    s_out.wait_event(t_start)
    for i in range(steps):
        b = i % nbuf
        if i >= nbuf:
            s_in.wait_event(fwd_done[b])           # x_dev[b] no longer read
        with torch.cuda.stream(s_in):
            x_dev[b].copy_(x_host, non_blocking=True)
        in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if i >= nbuf:
            stream.wait_event(out_done[b])         # out_dev[b] already copied out
        d_e2e["x"] = x_dev[b]
        plan.forward(**d_e2e, out=out_dev[b], stream=stream)
        fwd_done[b].record(stream)
        s_out.wait_event(fwd_done[b])
        with torch.cuda.stream(s_out):
            out_host[b].copy_(out_dev[b], non_blocking=True)
        out_done[b].record(s_out)
    t_end.record(s_out)
    t_end.synchronize()
    e2e_total = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    code, detail = plan.check_status()
    if code != 0:
        raise RuntimeError(f"device status {code} {detail}")
    return {"value": world * w.T * steps / (e2e_total / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
            "d2h_bytes_per_step": int(out_host[0].numel() * out_host[0].element_size()),
            "ms_per_step": e2e_total / steps, "steps": steps,
            "pipelining": "copy-in / compute / copy-out on 3 streams, double-buffered"}


def point_steps(ms_estimate: float, steps: int) -> int:
    """Steps of a companion point: at least `steps`, enough for MIN_TIMED_S of timed forwards."""
    want = int(MIN_TIMED_S * 1e3 / max(ms_estimate, 1e-3)) + 1
    return max(steps, min(want, MAX_POINT_STEPS))


def run_cuda(args, rank, world, local_rank):
    w = workload(args)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    resized = args.tokens is not None or args.experts is not None
    weights = make_weights(w, dev)
    head = measure(w, weights, args, rank, world, dev, args.steps, resized, args.workload)
    per_t = None
    companions = [] if (resized or args.no_per_t) else COMPANIONS.get(args.workload, [])
    if companions:
        per_t = {}
        for name in companions:
            wc = I.WORKLOADS[name]
            assert (wc.H, wc.I, wc.E, wc.k, wc.shared, wc.weight_std) == (w.H, w.I, w.E, w.k, w.shared, w.weight_std)
            # a short untimed run sizes the step count so every point's timed region is long enough
            est = measure_estimate(wc, weights, dev)
            est = max_over_ranks(est, world, dev)
            rec = measure(wc, weights, args, rank, world, dev, point_steps(est, args.steps), False, name)
            if rank == 0:
                per_t[f"T={wc.T}"] = rec
        head_key = f"T={w.T}"
        if rank == 0:
            per_t = {head_key: {k: v for k, v in head.items()}, **per_t}
            per_t = dict(sorted(per_t.items(), key=lambda kv: kv[1]["T"]))
    if rank != 0:
        return None

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, CPU_SAMPLE_TOKENS[args.workload])

    ms = head["ms_per_step"]
    value = world * w.T * args.steps / (ms * args.steps / 1e3)
    fused = any(o.replace(" ", "").upper() == "FUSED=1" for o in args.opt)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8e4m3 x fp4e2m1 (fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": head["workload"],
                   "T": w.T, "H": w.H, "I": w.I, "E": w.E, "k": w.k,
                   "shared": w.shared, "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MB write)",
                   "launch": ("one persistent cooperative kernel (MOE_OPT_FUSED)" if fused else
                              "kernels launched one by one" if args.no_graph else
                              f"CUDA graph replay of the {kernels_per_forward(w)} kernels (MOE_OPT_GRAPH)"),
                   "phase_times": "separate pass, CUDA events between kernels, 20 steps",
                   "weight_scales": f"re-laid out once before timing ({head['weight_scales_prepare_ms']:.3f} ms), "
                                    "reused (MOE_OPT_STATIC_WEIGHTS)",
                   "parallelism": f"replicas x{world} (token-sharded, no collective)",
                   "options": args.opt,
                   "per_T": ("the T = 1 / 512 / 8192 (Zipf-skewed) DeepSeek-V3-shaped layers on the same "
                             "expert weights, each timed in this run with its own steps, clocks, roofline "
                             "and end-to-end pass" if per_t else None)},
        "tflops": head["tflops"],
        "tflops_frac_fp8": head["tflops_frac_fp8"],
        "fp8_peak_tflops": head["fp8_peak_tflops"],
        "hbm_gbs": head["hbm_gbs"],
        "hbm_frac": head["hbm_frac"],
        "phases_ms": head["phases_ms"],
        "roofline": head["roofline"],
        "cpu_baseline": cpu,
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "max_expert_load_ratio": head["max_expert_load_ratio"],
        "per_T": per_t,
    }
    return line


def measure_estimate(w, weights, dev) -> float:
    """Milliseconds of one forward of `w` (untimed sizing run: 3 forwards, the last one timed)."""
    from fp8_fp4_moe_b200 import binding
    x, W_r, bias = I.make_routing_inputs(w, 0)
    d = dict(x=x.to(dev), W_router=W_r.to(dev), bias=bias.to(dev), **weights)
    plan = binding.Plan(w.T, w.H, w.I, w.E, w.k, w.shared, device=dev)
    plan.set_option(binding.MOE_OPT_STATIC_WEIGHTS, 1)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(2):
        plan.forward(**d, out=out)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    plan.forward(**d, out=out)
    b.record(stream)
    b.synchronize()
    ms = a.elapsed_time(b)
    del plan, d, out
    torch.cuda.empty_cache()
    return ms


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    init_ranks(world, local_rank, need_gpu=args.impl != "reference")
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_cuda(args, rank, world, local_rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
