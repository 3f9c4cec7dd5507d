"""Benchmark of the hybrid dense / 2:4 linear layer (PATCH) on B200.

Default workload: every linear of a Llama-3.2-1B-shaped model (16 layers x
q, k, v, o, gate, up, down) at M = 4096 tokens, bf16, 128x128 tiles, 90% of
tiles 2:4 overall (45% sparsity), each linear's 2:4 fraction drawn in
[0.8, 1.0] and adjusted to the exact global count. One step runs all 112
linears once on their synthetic inputs; weights and activations are already
resident in HBM. The step's working set (about 2 GB of packed weights) is far
larger than L2, so no flush is needed between steps.

Reported (one JSON line from rank 0):
  value        dense-equivalent TFLOP/s = 2*M*sum(N*K) / step time, all ranks
  speedup_vs_dense  step time of the same kernel on the all-dense packing of
               the same weights / hybrid step time
  sweep        the same step at 2:4 fractions 0 / 0.5 / 0.7 / 0.9 / 1.0
  roofline     tensor-pipe work (2*M*kept weights of each stored slab) per
               second of the tensor-core kernel, against the measured
               sustained bf16 peak
  e2e          the same metric through patch_linear_host (host buffers, copies
               inside the timed region)
  cpu_baseline the CPU oracle on a bounded sample of the same workload
  decode       the decode kernel on Llama-2-7B shapes at M = 1, 4, 16 (GB/s)

Multi-GPU (torchrun): every rank runs the whole workload on its own GPU with
its own tokens (data-parallel M split, weak scaling); no collective touches
the data path; the time is the max over ranks.

`--impl reference` times the CPU oracle (the only reference this method has)
on a bounded sample of the same workload.
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
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

FRACS_SWEEP = [0.0, 0.5, 0.7, 0.9, 1.0]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------- clocks ---

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            os.makedirs(os.path.join(ROOT, "gpurun_out"), exist_ok=True)
            self.path = os.path.join(ROOT, "gpurun_out", f"clocks_{os.getpid()}.csv")
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [r for r in rows if r[2] > 300] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in busy:
            for name, flag in zip(names, r[3][1:]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in busy), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(busy), "power_w_max": max(r[2] for r in rows), "reasons": sorted(reasons)}


# -------------------------------------------------------------- workload ---

def model_linears(n_layers: int):
    out = []
    for layer in range(n_layers):
        for l in synth.llama32_1b():
            out.append((layer, l))
    return out


def build_model(hsg, n_layers: int, frac: float, M: int, seed: int, lo=0.8, hi=1.0, rank=0):
    """Packs every linear of the model at global 2:4 fraction `frac`. Returns
    (list of (PackedLinear, K, N, kept_elems), inputs by K, outputs)."""
    lins = model_linears(n_layers)
    T = [(l.N // 128) * (l.K // 128) for _, l in lins]
    if frac in (0.0, 1.0):
        counts = [int(round(frac * t)) for t in T]
    else:
        counts = synth.split_fraction(T, frac, max(0.0, lo - (0.9 - frac)), min(1.0, hi - (0.9 - frac)),
                                      "model", seed, frac)
    packed = []
    for (layer, l), cnt in zip(lins, counts):
        p = synth.make_problem(l.N, l.K, 0, R=128, C=128, n_sparse=cnt, seed=seed,
                               device="cuda", tag=f"L{layer}-{l.name}")
        lin = hsg.PackedLinear.pack(p.W, p.bits, p.flags.cpu())
        info = lin.info()
        kept = (info.slabs_total - info.slabs_sparse) * 128 * 64 + info.slabs_sparse * 128 * 32
        packed.append((lin, l.K, l.N, kept, info.packed_bytes))
        del p
    torch.cuda.synchronize()
    X = {}
    for K in sorted({l.K for _, l in lins}):
        X[K] = synth.normal_bf16((M, K), 1.0, "cuda", "X", seed, rank, M, K)
    Y = {}
    for N in sorted({l.N for _, l in lins}):
        Y[N] = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    return packed, X, Y, sum(counts) / sum(T)


def run_step(hsg, model, X, Y, stream, path=0, events=None):
    for i, (lin, K, N, _, _) in enumerate(model):
        if events is not None:
            events[i][0].record(stream)
        hsg.patch_linear_path(lin.handle, X[K], Y[N], path, stream)
        if events is not None:
            events[i][1].record(stream)


def time_steps(hsg, model, X, Y, steps, warmup, stream, dist_on, per_launch=False):
    for _ in range(warmup):
        run_step(hsg, model, X, Y, stream)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    ev = None
    if per_launch:
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in model] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for s in range(steps):
        run_step(hsg, model, X, Y, stream, events=ev[s] if ev else None)
    end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    if dist_on:
        t = torch.tensor([ms], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    launch_ms = None
    if ev:
        launch_ms = [[a.elapsed_time(b) for a, b in row] for row in ev]
    return ms / steps, launch_ms


def flops_dense(model, M):
    return sum(2.0 * M * N * K for _, K, N, _, _ in model)


def cpu_sample(budget_s: float = 15.0, seed: int = 0, min_rows: int = 1):
    """The oracle on a bounded sample of the workload: token rows of the 7
    Llama-3.2-1B linears (one layer), as many rows as fit in about `budget_s`
    seconds. Returns (dense-equivalent TFLOP/s, threads, description)."""
    import oracle
    oracle.build()
    shapes = synth.llama32_1b()
    probs = [synth.make_problem(l.N, l.K, 64, R=128, C=128, frac=0.9, seed=seed, tag=f"cpu-{l.name}")
             for l in shapes]
    # calibrate on one row of every linear
    t0 = time.perf_counter()
    for p in probs:
        oracle.linear(p.X[:1], p.W, p.bits.numpy())
    t1 = time.perf_counter() - t0
    rows = max(min_rows, min(64, int(budget_s / max(t1, 1e-6))))
    flops = 0.0
    t0 = time.perf_counter()
    for l, p in zip(shapes, probs):
        oracle.linear(p.X[:rows], p.W, p.bits.numpy())
        flops += 2.0 * rows * l.N * l.K
    t = time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return flops / t / 1e12, threads, (f"oracle (expand mask, zero pruned weights, naive fp32 loop, OpenMP) "
                                       f"on {rows} token rows x the 7 Llama-3.2-1B linears of one layer, "
                                       f"{t:.1f} s")


def decode_bench(hsg, stream, steps=20):
    """Decode kernel, Llama-2-7B layer shapes, 70% 2:4 tiles, 4 layers of
    weights rotated so each launch streams its weights from HBM."""
    shapes = synth.llama2_7b()
    layers = []
    for L in range(4):
        row = []
        for l in shapes:
            p = synth.make_problem(l.N, l.K, 0, R=128, C=128, frac=0.7, seed=L, device="cuda",
                                   tag=f"dec{L}-{l.name}")
            lin = hsg.PackedLinear.pack(p.W, p.bits, p.flags.cpu())
            row.append((lin, l.K, l.N, lin.info().packed_bytes))
            del p
        layers.append(row)
    out = {}
    for M in (1, 4, 16):
        X = {K: synth.normal_bf16((M, K), 1.0, "cuda", "decX", M, K) for K in (4096, 11008)}
        Y = {N: torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for N in (4096, 11008)}
        for _ in range(3):
            for row in layers:
                for lin, K, N, _ in row:
                    hsg.patch_linear_path(lin.handle, X[K], Y[N], 2, stream)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        nbytes = 0
        for _ in range(steps):
            for row in layers:
                for lin, K, N, pb in row:
                    hsg.patch_linear_path(lin.handle, X[K], Y[N], 2, stream)
                    nbytes += pb + M * K * 2 + M * N * 2
        e.record(stream)
        torch.cuda.synchronize()
        ms = s.elapsed_time(e)
        out[f"M{M}"] = {"GB_s": nbytes / (ms / 1e3) / 1e9, "us_per_layer": ms * 1e3 / (steps * len(layers))}
    for row in layers:
        for lin, *_ in row:
            lin.free()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=16)
    ap.add_argument("--M", type=int, default=4096)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    workload = (f"Llama-3.2-1B linears (16 layers x q,k,v,o,gate,up,down), M={args.M} tokens, "
                f"bf16, 128x128 tiles, 90% 2:4 tiles (45% sparsity), per-linear fraction in [0.8,1.0]")

    if args.impl == "reference":
        if rank != 0:
            return
        steps_v = []
        for _ in range(min(args.warmup, 1)):
            cpu_sample(budget_s=2.0)
        for _ in range(args.steps):
            v, threads, desc = cpu_sample(budget_s=5.0)
            steps_v.append(v)
        val = statistics.median(steps_v)
        print(json.dumps({
            "impl": "reference", "metric": "hybrid dense/2:4 GEMM dense-equiv TFLOP/s", "value": val,
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
            "data": "synthetic", "config": {"workload": workload, "sample": "token rows of one layer per step"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return

    import hybrid_sparse_gemm_b200 as hsg

    dist_on = world > 1
    if dist_on:
        torch.cuda.set_device(local_rank)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    peaks = load_peaks()
    M = args.M

    with torch.cuda.stream(stream):
        model, X, Y, frac_real = build_model(hsg, args.layers, 0.9, M, seed=0, rank=rank)
        dense_model, _, _, _ = build_model(hsg, args.layers, 0.0, M, seed=0, rank=rank)
    torch.cuda.synchronize()
    F = flops_dense(model, M)
    exec_flops = sum(2.0 * M * kept for _, _, _, kept, _ in model)

    with ClockSampler(torch.cuda.current_device()) as clk:
        ms_h, launch_ms = time_steps(hsg, model, X, Y, args.steps, args.warmup, stream, dist_on,
                                     per_launch=False)
    clocks = clk.summary()
    ms_d, _ = time_steps(hsg, dense_model, X, Y, args.steps, args.warmup, stream, dist_on)
    # per-launch durations for the roofline (separate pass, events between launches)
    _, launch_ms = time_steps(hsg, model, X, Y, max(2, args.steps // 2), 1, stream, dist_on, per_launch=True)
    kern_ms = statistics.mean(sum(row) for row in launch_ms)
    achieved = exec_flops / (kern_ms / 1e3) / 1e12
    n_launch = len(model)
    value = world * F / (ms_h / 1e3) / 1e12

    sweep = None
    if not args.no_sweep:
        sweep = {}
        for f in FRACS_SWEEP:
            if f == 0.0:
                t = ms_d
            elif f == 0.9:
                t = ms_h
            else:
                with torch.cuda.stream(stream):
                    mdl, _, _, _ = build_model(hsg, args.layers, f, M, seed=0, rank=rank)
                t, _ = time_steps(hsg, mdl, X, Y, args.steps, args.warmup, stream, dist_on)
                for lin, *_ in mdl:
                    lin.free()
                del mdl
            sweep[str(f)] = {"tflops": world * F / (t / 1e3) / 1e12, "speedup_vs_dense": ms_d / t,
                             "ms_per_step": t}

    e2e = None
    if not args.no_e2e:
        Xh = {K: X[K].cpu().pin_memory() for K in X}
        Yh = {N: torch.empty(Y[N].shape, dtype=torch.bfloat16).pin_memory() for N in Y}
        h2d = sum(M * K * 2 for _, K, _, _, _ in model)
        d2h = sum(M * N * 2 for _, _, N, _, _ in model)
        e2e_steps = max(1, min(args.steps, 3))
        for lin, K, N, _, _ in model:  # warm-up
            hsg.patch_linear_host(lin.handle, Xh[K], Yh[N], stream)
        if dist_on:
            torch.distributed.barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        s.record(stream)
        for _ in range(e2e_steps):
            for lin, K, N, _, _ in model:
                hsg.patch_linear_host(lin.handle, Xh[K], Yh[N], stream)
        e.record(stream)
        torch.cuda.synchronize()
        ms_e = s.elapsed_time(e) / e2e_steps
        if dist_on:
            t = torch.tensor([ms_e], device="cuda")
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            ms_e = float(t.item())
        e2e = {"value": world * F / (ms_e / 1e3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ms_e}

    decode = None
    if not args.no_decode:
        for lin, *_ in dense_model:
            lin.free()
        dense_model = []
        decode = decode_bench(hsg, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        v, threads, desc = cpu_sample()
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": "hybrid dense/2:4 GEMM dense-equiv TFLOP/s and speedup vs dense bf16, per sparsity",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_h, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload, "M": M, "layers": args.layers, "linears": len(model),
                       "frac_2to4": frac_real, "tile": "128x128",
                       "l2": "inputs larger than L2 (%.2f GB of packed weights per step)" %
                             (sum(pb for *_, pb in model) / 1e9),
                       "parallelism": f"dp{world} (M split, replicated weights)"},
            "speedup_vs_dense": ms_d / ms_h, "dense_ms_per_step": ms_d,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops_sustained"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops_sustained"],
                         "traffic": None,
                         "kernel": "hybrid_gemm2_kernel (CTA pair, 256x256 tiles)",
                         "work": "2*M*(kept weights of stored slabs) per launch; sparse slabs count half",
                         "peak_kind": f"bf16 sustained ({peaks['source']})"},
            "gpu_launches": n_launch * args.steps,
            "clocks": clocks,
            "sweep": sweep, "e2e": e2e, "decode": decode, "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    for lin, *_ in model:
        lin.free()
    if dist_on:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
