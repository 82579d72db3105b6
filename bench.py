"""Benchmark of one DHSA prefill layer (mask construction + sparse attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole hot path on one synthetic layer: pool(Q),
pool(K), chunk score + top-k, block-CSR build and the sparse attention
kernel, all on one stream, inputs resident in HBM. At N = 1 the workload is
the 128K Llama-3.1-8B-shaped layer (the context length the metric is quoted
at). With N > 1 (torchrun, one process per GPU) every rank runs its own
independent layer: DHSA shards by head groups with no exchange, so ranks are
replicas and the scaling is weak.

Prints one JSON line on rank 0. `value` = amortised ms per layer over the
whole job (max-over-ranks device time of K steps / (K * N)).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

# The CPU legs (the oracle) use exactly the host cores this process may run
# on: BLAS and OpenMP thread pools are sized before numpy loads.
CORES = len(os.sched_getaffinity(0))
for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_v, str(CORES))

import numpy as np  # noqa: E402

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms per layer (mask+attn) and TFLOP/s on kept pairs at 128K, % of roofline"
ATTN_SRC = os.path.join(ROOT, "long_context_prefill_dhsa_b200", "csrc", "attn_fwd.cu")
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attention
# launch from an ncu capture of the 32K layer, scaled by tokens (x4) to the
# 128K layer; only valid for the kernel source it was measured on (the sha256
# of the kernel's constants and body, see kernel_region_sha).
ATTN_TRAFFIC = {"sha256_prefix": "bd13c5fab5760317",
                "bytes_per_launch": {"llama3.1-8b-32k": 6.427e8, "llama3.1-8b-128k": 2.571e9},
                "source": "ncu --set full capture of the 32K layer; 128K scaled x4 by tokens"}
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama8b-128k")
    ap.add_argument("--impl", default="dhsa", choices=["dhsa", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    # selection rule: top-k (default), or a token budget per row with a recent
    # window and a chunk cap; --budget-spread gives every row its own seeded
    # budget, uniform in budget * [1 - spread, 1 + spread] (query-dependent budgets)
    ap.add_argument("--budget", type=int, default=None)
    ap.add_argument("--recent", type=int, default=0)
    ap.add_argument("--kmax", type=int, default=None)
    ap.add_argument("--budget-spread", type=float, default=0.0)
    # query-tile policy of the attention: 0 = 128-row tiles (default, fastest);
    # 1 = chunk tails of at most 64 rows on the 64-row kernel; 2 = 64-row tiles only
    ap.add_argument("--short-tiles", type=int, default=0, choices=[0, 1, 2])
    # pooling and the top-k selection as one cooperative launch (top-k rule only)
    ap.add_argument("--fused-routing", action="store_true")
    return ap.parse_args()


def selection_rule(args, w, nmax):
    """(k passed to the layer, budget argument, recent, description) for the CLI options."""
    if args.budget is None:
        return w.k, None, 0, {"rule": "top-k", "k": w.k}
    k_max = args.kmax if args.kmax is not None else 4 * w.k
    desc = {"rule": "token budget", "budget": args.budget, "recent": args.recent, "k_max": k_max}
    if args.budget_spread > 0:
        rng = np.random.default_rng(1234)
        lo, hi = args.budget * (1 - args.budget_spread), args.budget * (1 + args.budget_spread)
        vec = rng.integers(int(lo), int(hi) + 1, (w.B, w.Hq, nmax)).astype(np.int32)
        desc["budget_spread"] = args.budget_spread
        return k_max, vec, args.recent, desc
    return k_max, args.budget, args.recent, desc


def kernel_region_sha(path=ATTN_SRC):
    """sha256 prefix of the attention kernel's device code: from its
    constants (`using namespace ptx;`) through the kernel's closing brace.
    Host-side launch code after the kernel does not enter it."""
    import hashlib
    s = open(path).read()
    a = s.index("using namespace ptx;")
    b = s.index("\n}\n", s.index("__global__", a)) + 3
    return hashlib.sha256(s[a:b].encode()).hexdigest()[:16]


def attn_traffic(workload_name):
    sha = kernel_region_sha()
    if sha != ATTN_TRAFFIC["sha256_prefix"]:
        return None, "kernel changed since the ncu capture"
    v = ATTN_TRAFFIC["bytes_per_launch"].get(workload_name)
    return v, ATTN_TRAFFIC["source"] if v is not None else "no capture for this workload"


def peaks():
    try:
        p = json.load(open(PEAKS_PATH))
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every
    20 ms while the timed region runs (read-only queries)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []
        self.sm_max = None
        self.error = None
        self._stop = threading.Event()

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.cuda_index)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
            except Exception:
                pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = int(vis.split(",")[self.cuda_index]) if vis and vis.split(",")[0].isdigit() else self.cuda_index
        return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def __enter__(self):
        try:
            import pynvml
            h = self._handle()
            self.sm_max = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                             int(get_reasons(h))))
                    except Exception as e:  # keep sampling; report the error
                        self.error = repr(e)[:120]
                    time.sleep(0.02)

            self.th = threading.Thread(target=run, daemon=True)
            self.th.start()
        except Exception as e:
            self.error = repr(e)[:120]
        return self

    def __exit__(self, *a):
        self._stop.set()
        if hasattr(self, "th"):
            self.th.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": ["no samples"], "error": self.error}
        reasons = sorted({name for _, r in self.samples for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(c for c, _ in self.samples), "sm_max_mhz": self.sm_max,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml, 20 ms"}


# ----------------------------------------------------------------- ranks
def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank timing over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_layer(max_total_ms: float, steps: int, world: int) -> float:
    """Whole-job amortised ms per layer: each of `world` ranks runs one layer per step."""
    return max_total_ms / steps / world


# ----------------------------------------------------------------- helpers
def kept_pair_count(off, n_chunks, sel, n_sel):
    """Kept token pairs of the layer from the GPU selection (host arithmetic)."""
    import torch
    B, Hq, nmax, stride = sel.shape
    lens = torch.diff(off.long(), dim=1)                                 # [B, Nmax]
    total = 0
    for b in range(B):
        n = int(n_chunks[b])
        lb = lens[b, :n]
        s = sel[b, :, :n].long()
        valid = s >= 0
        lj = torch.where(valid, lb[s.clamp(min=0)], torch.zeros_like(s))
        row_keys = lj.sum(-1) - lb[None, :]                               # earlier kept chunks
        total += int((lb[None, :] * row_keys).sum() + (Hq * (lb * (lb + 1) // 2).sum()))
    return total


def routing_bytes(w, nmax, k):
    """Algorithmic HBM bytes of the routing stages (one layer)."""
    d = 128
    x = w.B * (w.Hq + w.Hkv) * w.L * d * 2                 # read Q and K once
    pooled = w.B * (w.Hq + w.Hkv) * nmax * d * 4           # write Qp/Kp
    reread = pooled                                         # read them again for scoring
    stride = min(k, nmax - 1) + 1
    sel = w.B * w.Hq * nmax * (stride + 1) * 4 * 2          # write sel/n_sel, read in CSR build
    csr = w.B * w.Hq * nmax * (stride + 3) * 4              # row_ptr, col_idx, cost
    return x + pooled + reread + sel + csr


def attn_bytes(w):
    """Compulsory attention HBM bytes: Q, K, V read once, O written once."""
    return w.B * (2 * w.Hq + 2 * w.Hkv) * w.L * 128 * 2


# ----------------------------------------------------------------- oracle (CPU) leg
def cpu_oracle_sample(d, w, seconds, rule=None):
    """Time the CPU oracle on a bounded sample of the layer and extrapolate
    to ms per layer. Sample: pooling of one query head + its kv head, the
    chunk scores/selection of that head, and the attention of as many of its
    query chunks (in a fixed shuffled order) as fit in the time budget."""
    from oracle import dhsa as ora
    off, nc = d["off"], d["n_chunks"]
    nmax = off.shape[1] - 1
    cores = int(os.environ.get("OPENBLAS_NUM_THREADS", CORES))
    t0 = time.perf_counter()
    Qp = ora.chunk_pool(ora.bf16_to_f64(d["Q"][:, :1]), off, nc, nmax)
    Kp = ora.chunk_pool(ora.bf16_to_f64(d["K"][:, :1]), off, nc, nmax)
    t_pool = time.perf_counter() - t0
    t0 = time.perf_counter()
    S = ora.chunk_scores(Qp, Kp, nc)
    if rule is None or rule[1] is None:
        sel = ora.select(S, nc, w.k)
    else:
        k_max, bud, recent = rule[0], rule[1], rule[2]
        sel = ora.select_budget(S, off, nc, bud if np.isscalar(bud) else bud[:, :1], recent, k_max)
    t_route = time.perf_counter() - t0
    Q = ora.bf16_to_f64(d["Q"][0, 0]).astype(np.float32)
    K = ora.bf16_to_f64(d["K"][0, 0]).astype(np.float32)
    V = ora.bf16_to_f64(d["V"][0, 0]).astype(np.float32)
    n = int(nc[0])
    order = np.random.default_rng(0).permutation(n)
    done, t_attn = 0, 0.0
    t0 = time.perf_counter()
    for i in order:
        ora.attn_chunk(Q, K, V, off[0], sel[0][0][i], int(i), 1.0 / math.sqrt(128), np.float32)
        done += 1
        t_attn = time.perf_counter() - t0
        if t_attn > seconds:
            break
    heads = w.B * w.Hq
    kv_frac = w.Hkv / w.Hq
    est_route = t_pool * (1 + kv_frac) / 2 * heads + t_route * heads
    est_attn = t_attn * (n / done) * heads
    est = est_route + est_attn
    return {"value": est * 1e3, "unit": "ms", "cores": cores, "kind": "oracle",
            "routing_ms": est_route * 1e3, "attention_ms": est_attn * 1e3,
            "sample": (f"oracle on (b=0, hq=0): pooling of Q and K, all {n} score/selection rows, attention of "
                       f"{done}/{n} query chunks; extrapolated x{heads} heads"
                       f"{' x' + str(round(n / done, 2)) + ' chunks' if done < n else ''}")}


def workload_config(args, w, nmax, sel_desc):
    """The `config` object of both arms: what the workload is (no results,
    no kernel choices), so the GPU arm and the reference arm print the same."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "head_dim": 128, "k": w.k,
            "selection": sel_desc, "chunk_len": f"{w.length_kind}[{w.length_lo},{w.length_hi}]",
            "n_chunks": nmax, "parallelism": f"replicas x{args.gpus} (independent layers, no collective)",
            "l2": "inputs larger than L2 (Q+K+V = %.2f GB)" % (attn_bytes(w) / 2 / 1e9)}


# ----------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from long_context_prefill_dhsa_b200 import inputs as I
    w = I.WORKLOADS[args.workload]
    d = I.make_inputs(w)
    k_sel, bud, recent, sel_desc = selection_rule(args, w, d["off"].shape[1] - 1)
    rule = (k_sel, bud, recent)
    # every step (warm-up included) is the oracle on one whole head: pooling,
    # all score/selection rows and the attention of every query chunk; the
    # layer time is that head's time x the layer's heads (labelled)
    for _ in range(args.warmup):
        cpu_oracle_sample(d, w, math.inf, rule)
    vals = []
    res = None
    for _ in range(args.steps):
        res = cpu_oracle_sample(d, w, math.inf, rule)
        vals.append(res["value"])
    v = statistics.median(vals)
    res["value"] = v
    res["steps_ms"] = vals
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "ms", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": v, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args, w, d["off"].shape[1] - 1, sel_desc),
        "cpu_baseline": res, "e2e": {"value": v, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ----------------------------------------------------------------- main arm
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    from long_context_prefill_dhsa_b200 import binding, inputs as I
    binding.load()
    w = I.WORKLOADS[args.workload]
    d = I.make_inputs(w)
    dev = torch.device("cuda", local)
    host = {x: torch.from_numpy(d[x]).view(torch.bfloat16).pin_memory() for x in "QKV"}
    host_off = torch.from_numpy(d["off"]).pin_memory()
    host_nc = torch.from_numpy(d["n_chunks"]).pin_memory()
    Q, K, V = (host[x].to(dev) for x in "QKV")
    off, nc = host_off.to(dev), host_nc.to(dev)
    k_sel, bud, recent, sel_desc = selection_rule(args, w, d["off"].shape[1] - 1)
    bud_arg = torch.from_numpy(bud).to(dev) if isinstance(bud, np.ndarray) else bud
    layer = binding.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, off, nc, k_sel, device=dev, budget=bud_arg, recent=recent,
                                short_tiles=args.short_tiles, fused_routing=args.fused_routing)
    stream = torch.cuda.current_stream()

    ev = lambda: torch.cuda.Event(enable_timing=True)
    # pool (Q and K), key norms + score tiles + select, CSR scan + fill, work list + attention
    # (tile policy 1 launches both attention kernels)
    n_launch_per_step = 8 + (1 if args.short_tiles == 1 else 0) - (3 if args.fused_routing else 0)

    def step(timed_stages=None):
        if timed_stages is None:
            return layer.run(Q, K, V)
        e0, e1, e2 = ev(), ev(), ev()
        e0.record(stream)
        layer.routing(Q, K)
        e1.record(stream)
        layer.attention(Q, K, V)
        e2.record(stream)
        timed_stages.append((e0, e1, e2))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    binding.check_device_status()

    stages = []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0, t1 = ev(), ev()
        t0.record(stream)
        for _ in range(args.steps):
            step(stages)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(t0.elapsed_time(t1), dev)
    flags = binding.check_device_status()
    route_ms = statistics.median(a.elapsed_time(b) for a, b, _ in stages)
    attn_ms = statistics.median(b.elapsed_time(c) for _, b, c in stages)
    layer_ms = [a.elapsed_time(c) for a, _, c in stages]
    ms_step = total_ms / args.steps

    nmax = d["off"].shape[1] - 1
    pairs = kept_pair_count(off.cpu(), nc.cpu(), layer.sel.cpu(), layer.n_sel.cpu())
    flop = 4.0 * 128 * pairs
    hbm_peak, tc_peak, peak_kind = peaks()
    attn_tflops = flop / (attn_ms * 1e-3) / 1e12
    rbytes = routing_bytes(w, nmax, k_sel)
    traffic, traffic_src = attn_traffic(w.name)
    if args.short_tiles:
        traffic, traffic_src = None, "captured for the 128-row tile policy only"

    # end to end through the public API with host buffers (pinned), on this rank:
    # every step copies that layer's Q, K, V in from pinned host memory and its
    # O back out; HostStreamedPrefill overlaps the copies of neighbouring
    # layers with the compute (the chunk offsets of the sequence stay resident)
    e2e = None
    if not args.no_e2e:
        out_host = torch.empty(host["Q"].shape, dtype=torch.bfloat16).pin_memory()
        h2d = sum(host[x].numel() * 2 for x in "QKV")
        d2h = out_host.numel() * 2
        runner = binding.HostStreamedPrefill(layer)
        for _ in range(2):
            runner.submit(host["Q"], host["K"], host["V"], out_host)
        runner.synchronize()
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record(runner.s_in)
        for _ in range(args.steps):
            runner.submit(host["Q"], host["K"], host["V"], out_host)
        b.record(runner.s_out)
        runner.synchronize()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b), dev)
        e2e = {"value": job_ms_per_layer(e2e_ms, args.steps, world), "unit": "ms",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "overlap": "copy-in of step s+1 and copy-out of step s-1 run during step s"}
        del runner

    # dense comparisons (not part of the timed value): the same kernels with
    # k = all causal chunks, and torch SDPA dense causal attention
    dense = {}
    if not args.no_dense and rank == 0:
        try:
            dl = binding.DHSAPrefill(w.B, w.Hq, w.Hkv, w.L, off, nc, 1 << 30, device=dev)
            dl.run(Q, K, V)
            torch.cuda.synchronize()
            a, b = ev(), ev()
            a.record(stream)
            dl.run(Q, K, V)
            b.record(stream)
            torch.cuda.synchronize()
            dense["dhsa_k_all_ms"] = a.elapsed_time(b)
            del dl
            import torch.nn.functional as F
            Kr = K.repeat_interleave(w.G, dim=1)
            Vr = V.repeat_interleave(w.G, dim=1)
            F.scaled_dot_product_attention(Q, Kr, Vr, is_causal=True)
            torch.cuda.synchronize()
            a, b = ev(), ev()
            a.record(stream)
            F.scaled_dot_product_attention(Q, Kr, Vr, is_causal=True)
            b.record(stream)
            torch.cuda.synchronize()
            dense["torch_sdpa_causal_ms"] = a.elapsed_time(b)
            dense["speedup_vs_sdpa"] = dense["torch_sdpa_causal_ms"] / ms_step
            dense["speedup_vs_k_all"] = dense["dhsa_k_all_ms"] / ms_step
        except Exception as e:  # measurement only; never fails the bench
            dense["error"] = repr(e)[:200]

    cpu = None
    if not args.no_cpu and rank == 0 and world == 1:
        cpu = cpu_oracle_sample(d, w, args.cpu_seconds, (k_sel, bud, recent))

    if rank == 0:
        line = {
            "metric": METRIC, "value": job_ms_per_layer(total_ms, args.steps, world), "unit": "ms",
            "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(args, w, nmax, sel_desc),
            "kernels": {"query_tiles": ["128 rows", "128 rows, tails <= 64 rows on the 64-row kernel",
                                        "64 rows"][args.short_tiles],
                        "routing_launches": "fused (one cooperative launch up to the selection)"
                                            if args.fused_routing else "separate"},
            "kept_density": pairs / (w.B * w.Hq * w.L * (w.L + 1) / 2),
            "ms_per_step_median": statistics.median(layer_ms),
            "ms_per_step_protocol": "value = mean over the timed steps (total / steps); the median of the "
                                    "per-step layer times is ms_per_step_median",
            "stages_ms": {"routing": route_ms, "attention": attn_ms},
            "tflops_kept_pairs": flop / (ms_step * 1e-3) / 1e12,
            "roofline": {"bound": "tensor", "achieved": attn_tflops,
                         "kernel": ["sparse_attn_fwd_kernel", "sparse_attn_fwd_kernel + sparse_attn_short_kernel",
                                    "sparse_attn_short_kernel"][args.short_tiles],
                         "peak": tc_peak, "unit": "TFLOP/s", "frac": attn_tflops / tc_peak,
                         "peak_kind": f"{peak_kind} bf16 dense (burst)", "traffic": traffic,
                         "traffic_source": traffic_src, "flop_per_launch": flop},
            "routing_roofline": {"bound": "hbm", "achieved": rbytes / (route_ms * 1e-3) / 1e9, "peak": hbm_peak,
                                 "unit": "GB/s", "frac": rbytes / (route_ms * 1e-3) / 1e9 / hbm_peak,
                                 "bytes_per_layer": rbytes},
            "gpu_launches": n_launch_per_step * args.steps,
            "device_flags": flags,
            "clocks": clk.summary(),
            "e2e": e2e,
            "dense": dense,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
