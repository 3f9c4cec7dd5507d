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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

FRACS_SWEEP = [0.0, 0.5, 0.7, 0.9, 1.0]
METRIC = "hybrid dense/2:4 GEMM dense-equiv TFLOP/s and speedup vs dense bf16, per sparsity"
# DRAM bytes (read + write) of one launch of a kernel on the default workload
# (one Llama-3.2-1B layer, M = 4096, 90 % 2:4 tiles), from an ncu capture, with
# the sha256 prefix of the kernel source it was taken on: reported only while
# that source is unchanged.
MEASURED_TRAFFIC = {
    "hybrid_gemm22_kernel": {"source": "hybrid_sparse_gemm_b200/csrc/gemm22.cu", "sha256": "fab2917e4fbf7991",
                             "workload": ("llama32-1b", 4096, "128x128"), "bytes_per_launch": 407.99e6},
}
KERNEL_NAMES = {4: "hybrid_gemm2_kernel (CTA pair, 256x256 tiles)",
                6: "hybrid_gemm22_kernel (CTA pair, two strips per CTA, 512x240 tiles)",
                3: "hybrid_gemm_kernel (single CTA, 128x128 tiles)"}


def measured_traffic(kernel_name: str, workload=("llama32-1b", 4096, "128x128")):
    """ncu DRAM bytes per launch for this kernel on this workload, or None if
    none was taken on the current source."""
    import hashlib
    for k, t in MEASURED_TRAFFIC.items():
        if kernel_name.startswith(k) and tuple(t["workload"]) == tuple(workload):
            with open(os.path.join(ROOT, t["source"]), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest()[:16] == t["sha256"]:
                    return t["bytes_per_launch"]
    return None


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

    def __init__(self, device_index: int, cmd=None):
        self.idx = device_index
        self.cmd = cmd or ["nvidia-smi", "-i", str(device_index), f"--query-gpu={self.FIELDS}",
                           "--format=csv,noheader,nounits", "-lms", "50"]
        self.proc = None
        self.path = None
        self.fh = None

    def __enter__(self):
        try:
            # PATCH_CLOCKS_CSV keeps the raw samples at a chosen path; by default
            # they go to a temporary file that is summarised into the JSON line.
            self.path = os.environ.get("PATCH_CLOCKS_CSV") or os.path.join(
                tempfile.gettempdir(), f"patch_clocks_{os.getpid()}.csv")
            d = os.path.dirname(self.path)
            if d:
                os.makedirs(d, exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(self.cmd, stdout=self.fh, stderr=subprocess.DEVNULL)
            # nvidia-smi needs a few hundred ms to start; hold the timed region
            # until its first sample is on disk (at most 5 s).
            t0 = time.time()
            while time.time() - t0 < 5.0 and self.proc.poll() is None:
                if os.path.getsize(self.path) > 0:
                    break
                time.sleep(0.02)
        except Exception:
            self.proc = None
            if self.fh is not None:
                self.fh.close()
                self.fh = None
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
        with open(self.path) as f:
            lines = f.readlines()
        if not os.environ.get("PATCH_CLOCKS_CSV"):
            os.remove(self.path)  # the temporary file; its summary goes into the JSON line
        for line in lines:
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

# Model shapes the bench can run: (shape function, default tokens M, default layers).
WORKLOADS = {
    "llama32-1b": (synth.llama32_1b, 4096, 16, "Llama-3.2-1B"),
    "llama2-7b": (synth.llama2_7b, 2048, 8, "Llama-2-7B"),
    "llama2-13b": (synth.llama2_13b, 8192, 2, "Llama-2-13B"),
}


def model_linears(n_layers: int, shapes=synth.llama32_1b):
    out = []
    for layer in range(n_layers):
        for l in shapes():
            out.append((layer, l))
    return out


ROLE_INPUT = {"q": "attn", "k": "attn", "v": "attn", "o": "o", "gate": "mlp", "up": "mlp", "down": "down"}


def build_model(hsg, n_layers: int, frac: float, M: int, seed: int, lo=0.8, hi=1.0, rank=0, group=True,
                shapes=synth.llama32_1b, R=128, C=128):
    """Packs every linear of the model at global 2:4 fraction `frac`.

    Returns (layers, X, Y, frac): layers is a list of per-layer launch lists;
    each launch is (callable, [(PackedLinear, K, N, kept_weights, packed_bytes)]).
    q/k/v read one input, gate/up another, o and down their own; every linear
    writes its own output."""
    lins = model_linears(n_layers, shapes)
    T = [(l.N // R) * (l.K // C) for _, l in lins]
    if frac in (0.0, 1.0):
        counts = [int(round(frac * t)) for t in T]
    else:
        counts = synth.split_fraction(T, frac, max(0.0, lo - (0.9 - frac)), min(1.0, hi - (0.9 - frac)),
                                      "model", seed, frac)
    X = {}
    for _, l in lins[:7]:
        role = ROLE_INPUT[l.name]
        if role not in X:
            X[role] = synth.normal_bf16((M, l.K), 1.0, "cuda", "X", seed, rank, M, role)
    per_layer = {}
    for (layer, l), cnt in zip(lins, counts):
        p = synth.make_problem(l.N, l.K, 0, R=R, C=C, n_sparse=cnt, seed=seed,
                               device="cuda", tag=f"L{layer}-{l.name}")
        lin = hsg.PackedLinear.pack(p.W, p.bits, p.flags.cpu(), R, C)
        info = lin.info()
        kept = (info.slabs_total - info.slabs_sparse) * 128 * 64 + info.slabs_sparse * 128 * 32
        Yt = torch.empty((M, l.N), dtype=torch.bfloat16, device="cuda")
        per_layer.setdefault(layer, []).append((lin, l.K, l.N, kept, info.packed_bytes, X[ROLE_INPUT[l.name]], Yt))
        del p
    torch.cuda.synchronize()
    layers = []
    for layer in sorted(per_layer):
        members = per_layer[layer]
        if group:
            g = hsg.LinearGroup([m[0] for m in members])
            layers.append((g, members))
        else:
            for m in members:
                layers.append((None, [m]))
    return layers, X, None, sum(counts) / sum(T)


def free_model(layers):
    for g, members in layers:
        if g is not None:
            g.free()
        for m in members:
            m[0].free()


def run_step(hsg, model, X, Y, stream, path=0, events=None):
    for i, (g, members) in enumerate(model):
        if events is not None:
            events[i][0].record(stream)
        if g is not None:
            g([m[5] for m in members], [m[6] for m in members], path=path, stream=stream)
        else:
            m = members[0]
            hsg.patch_linear_path(m[0].handle, m[5], m[6], path, stream)
        if events is not None:
            events[i][1].record(stream)


def time_steps(hsg, model, X, Y, steps, warmup, stream, dist_on, per_launch=False, path=0):
    from hybrid_sparse_gemm_b200 import dist as hdist
    for _ in range(warmup):
        run_step(hsg, model, X, Y, stream, path)
    torch.cuda.synchronize()
    hdist.barrier(dist_on)
    ev = None
    if per_launch:
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in model] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for s in range(steps):
        run_step(hsg, model, X, Y, stream, path, events=ev[s] if ev else None)
    end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    ms = hdist.max_over_ranks(ms, dist_on, device="cuda")
    launch_ms = None
    if ev:
        launch_ms = [[a.elapsed_time(b) for a, b in row] for row in ev]
    return ms / steps, launch_ms


def members(model):
    return [m for _, ms in model for m in ms]


def flops_dense(model, M):
    return sum(2.0 * M * m[2] * m[1] for m in members(model))


class OracleSample:
    """The oracle on a bounded sample of the workload: token rows of the 7
    linears of one layer. Building the inputs and calibrating the cost model
    happen once; `run(rows)` is one timed sample."""

    def __init__(self, workload: str = "llama32-1b", M: int = 4096, R: int = 128, C: int = 128, seed: int = 0):
        import oracle
        oracle.build()
        self.oracle = oracle
        shape_fn, _, _, self.model_name = WORKLOADS[workload]
        self.M = M
        self.shapes = shape_fn()
        self.probs = [synth.make_problem(l.N, l.K, M, R=R, C=C, frac=0.9, seed=seed, tag=f"cpu-{l.name}")
                      for l in self.shapes]
        self.bits = [p.bits.numpy() for p in self.probs]
        # calibrate: time 4 and 16 rows of every linear (after one untimed call
        # that starts the thread pool) and fit time = fixed + rows * per_row; the
        # fixed part (mask expansion over the whole weight) does not shrink with rows
        oracle.linear(self.probs[0].X[:1], self.probs[0].W, self.bits[0])
        t4, t16 = self.run(4)[1], self.run(16)[1]
        self.per_row = max((t16 - t4) / 12.0, 1e-6)
        self.fixed = max(t4 - 4 * self.per_row, 0.0)
        self.threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))

    def rows_for(self, budget_s: float, min_rows: int = 1) -> int:
        return max(min_rows, min(self.M, int((budget_s - self.fixed) / self.per_row)))

    def run(self, rows: int):
        """One pass over the 7 linears on `rows` token rows; returns
        (dense-equivalent TFLOP/s, seconds)."""
        flops = 0.0
        t0 = time.perf_counter()
        for l, p, b in zip(self.shapes, self.probs, self.bits):
            self.oracle.linear(p.X[:rows], p.W, b)
            flops += 2.0 * rows * l.N * l.K
        t = time.perf_counter() - t0
        return flops / t / 1e12, t

    def describe(self, rows: int, t: float) -> str:
        return (f"oracle (expand mask, zero pruned weights, naive fp32 loop, OpenMP) on {rows} token rows "
                f"x the 7 {self.model_name} linears of one layer, {t:.1f} s")


def cpu_sample(budget_s: float = 15.0, seed: int = 0, min_rows: int = 1, workload: str = "llama32-1b",
               M: int = 4096, R: int = 128, C: int = 128):
    """One bounded oracle sample of about `budget_s` seconds.
    Returns (dense-equivalent TFLOP/s, threads, description)."""
    s = OracleSample(workload, M, R, C, seed)
    rows = s.rows_for(budget_s, min_rows)
    v, t = s.run(rows)
    return v, s.threads, s.describe(rows, t)


def decode_bench(hsg, stream, peaks, steps=20):
    """Decode kernel on Llama-2-7B layer shapes, 70% 2:4 tiles: each layer's 7
    linears in one grouped launch, 4 layers rotated (about 1.1 GB of weights,
    far above L2) so every launch streams its weights from HBM. Bytes counted
    are the ones the decode path must read: per-strip records (16 KB per dense
    slab, 8 KB per 2:4 slab), metadata blocks, X and Y."""
    shapes = synth.llama2_7b()
    layers = []
    for L in range(4):
        mem = []
        for l in shapes:
            p = synth.make_problem(l.N, l.K, 0, R=128, C=128, frac=0.7, seed=L, device="cuda",
                                   tag=f"dec{L}-{l.name}")
            lin = hsg.PackedLinear.pack(p.W, p.bits, p.flags.cpu())
            info = lin.info()
            algo = ((info.slabs_total - info.slabs_sparse) * 16384 + info.slabs_sparse * 8192
                    + info.meta_blocks * 2048)
            mem.append((lin, l.K, l.N, algo))
            del p
        layers.append((hsg.LinearGroup([m[0] for m in mem]), mem))
    out = {}
    for M in (1, 4, 16):
        X = {K: synth.normal_bf16((M, K), 1.0, "cuda", "decX", M, K) for K in (4096, 11008)}
        Y = [[torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _, _, N, _ in mem] for _, mem in layers]
        res = {}
        for name, path in (("tc", 2), ("simt", 5)):
            def step():
                for (g, mem), ys in zip(layers, Y):
                    g([X[K] for _, K, _, _ in mem], ys, path=path, stream=stream)
            for _ in range(3):
                step()
            torch.cuda.synchronize()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            for _ in range(steps):
                step()
            e.record(stream)
            torch.cuda.synchronize()
            ms = s.elapsed_time(e)
            nbytes = steps * sum(a + M * K * 2 + M * N * 2 for _, mem in layers for _, K, N, a in mem)
            gbs = nbytes / (ms / 1e3) / 1e9
            res[name] = {"GB_s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                         "us_per_layer": ms * 1e3 / (steps * len(layers))}
        out[f"M{M}"] = res
    for g, mem in layers:
        g.free()
        for m in mem:
            m[0].free()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama32-1b", choices=sorted(WORKLOADS),
                    help="model whose linears one step runs (default: Llama-3.2-1B, M = 4096)")
    ap.add_argument("--layers", type=int, default=None, help="layers per step (default per workload)")
    ap.add_argument("--M", type=int, default=None, help="tokens (default per workload)")
    ap.add_argument("--tile", default="128x128", choices=["128x128", "128x64", "64x128", "64x64"],
                    help="mask tile shape")
    ap.add_argument("--no-group", action="store_true", help="one launch per linear instead of per layer")
    ap.add_argument("--path", default="auto", choices=["auto", "pair", "wide"],
                    help="tensor-core kernel for the timed steps (auto: the library's choice)")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    shape_fn, default_M, default_layers, model_name = WORKLOADS[args.workload]
    if args.M is None:
        args.M = default_M
    if args.layers is None:
        args.layers = default_layers
    R, C = (int(v) for v in args.tile.split("x"))
    workload = (f"{model_name} linears ({args.layers} layers x q,k,v,o,gate,up,down), M={args.M} tokens, "
                f"bf16, {R}x{C} tiles, 90% 2:4 tiles (45% sparsity), per-linear fraction in [0.8,1.0]")

    if args.impl == "reference":
        if rank != 0:
            return
        # each step is one bounded sample, sized so that all K steps take
        # about a minute and a half of CPU time (0.25 s to 5 s per step)
        samp = OracleSample(args.workload, args.M, R, C)
        rows = samp.rows_for(max(0.25, min(5.0, 90.0 / max(1, args.steps))))
        for _ in range(min(args.warmup, 1)):
            samp.run(rows)
        steps_v, secs = [], []
        for _ in range(args.steps):
            v, t = samp.run(rows)
            steps_v.append(v)
            secs.append(t)
        val = statistics.median(steps_v)
        threads, desc = samp.threads, samp.describe(rows, statistics.median(secs)) + " per step"
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": val,
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
            "data": "synthetic", "config": {"workload": workload, "M": args.M, "layers": args.layers,
                                            "tile": args.tile, "path": "cpu oracle",
                                            "sample": "token rows of one layer per step"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return

    import hybrid_sparse_gemm_b200 as hsg
    from hybrid_sparse_gemm_b200 import dist as hdist

    torch.cuda.set_device(local_rank if world > 1 else 0)
    dist_on = hdist.init("nccl")
    stream = torch.cuda.Stream()
    peaks = load_peaks()
    gpath = {"auto": hsg.PATH_AUTO, "pair": hsg.PATH_GEMM_PAIR, "wide": hsg.PATH_GEMM_WIDE}[args.path]
    M = args.M
    group = not args.no_group

    with torch.cuda.stream(stream):
        model, X, _, frac_real = build_model(hsg, args.layers, 0.9, M, seed=0, rank=rank, group=group,
                                             shapes=shape_fn, R=R, C=C)
        dense_model, _, _, _ = build_model(hsg, args.layers, 0.0, M, seed=0, rank=rank, group=group,
                                           shapes=shape_fn, R=R, C=C)
    torch.cuda.synchronize()
    F = flops_dense(model, M)
    exec_flops = sum(2.0 * M * m[3] for m in members(model))
    n_launch = len(model)

    nvtx = torch.cuda.nvtx  # phase markers for profilers; nothing inside the timed loops
    with ClockSampler(torch.cuda.current_device()) as clk, nvtx.range("hybrid steps"):
        ms_h, _ = time_steps(hsg, model, X, None, args.steps, args.warmup, stream, dist_on, path=gpath)
    clocks = clk.summary()
    with nvtx.range("dense steps"):
        ms_d, _ = time_steps(hsg, dense_model, X, None, args.steps, args.warmup, stream, dist_on, path=gpath)
    # per-launch durations for the roofline (separate pass, events around each launch)
    with nvtx.range("per-launch timing"):
        _, launch_ms = time_steps(hsg, model, X, None, max(2, args.steps // 4), 1, stream, dist_on,
                                  per_launch=True, path=gpath)
    kern_ms = statistics.mean(sum(row) for row in launch_ms)
    kernel_name = KERNEL_NAMES.get(model[0][0].path(M, gpath) if model[0][0] is not None else hsg.PATH_GEMM_PAIR,
                                   "tensor-core GEMM")
    achieved = exec_flops / (kern_ms / 1e3) / 1e12
    value = hdist.job_rate(F, world, ms_h) / 1e12

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
                    mdl, _, _, _ = build_model(hsg, args.layers, f, M, seed=0, rank=rank, group=group,
                                               shapes=shape_fn, R=R, C=C)
                with nvtx.range(f"sweep f={f}"):
                    t, _ = time_steps(hsg, mdl, X, None, args.steps, args.warmup, stream, dist_on, path=gpath)
                free_model(mdl)
                del mdl
            sweep[str(f)] = {"tflops": hdist.job_rate(F, world, t) / 1e12, "speedup_vs_dense": ms_d / t,
                             "ms_per_step": t}

    e2e = None
    if not args.no_e2e:
        mem = members(model)
        Xh = {id(m[5]): m[5].cpu().pin_memory() for m in mem}
        Yh = [torch.empty(m[6].shape, dtype=torch.bfloat16).pin_memory() for m in mem]
        h2d = sum(M * m[1] * 2 for m in mem)
        d2h = sum(M * m[2] * 2 for m in mem)
        e2e_steps = max(1, min(args.steps, 3))
        for m, yh in zip(mem, Yh):  # warm-up
            hsg.patch_linear_host(m[0].handle, Xh[id(m[5])], yh, stream)
        hdist.barrier(dist_on)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        s.record(stream)
        for _ in range(e2e_steps):
            for m, yh in zip(mem, Yh):
                hsg.patch_linear_host(m[0].handle, Xh[id(m[5])], yh, stream)
        e.record(stream)
        torch.cuda.synchronize()
        ms_e = s.elapsed_time(e) / e2e_steps
        ms_e = hdist.max_over_ranks(ms_e, dist_on, device="cuda")
        e2e = {"value": hdist.job_rate(F, world, ms_e) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ms_e}

    free_model(dense_model)
    dense_model = []
    decode = None
    if not args.no_decode:
        with nvtx.range("decode"):
            decode = decode_bench(hsg, stream, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        v, threads, desc = cpu_sample(workload=args.workload, M=args.M, R=R, C=C)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank == 0:
        packed_gb = sum(m[4] for m in members(model)) / 1e9
        line = {
            "metric": METRIC,
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_h, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload, "M": M, "layers": args.layers, "linears": len(members(model)),
                       "launches_per_step": n_launch, "grouped": group,
                       "frac_2to4": frac_real, "tile": args.tile,
                       "l2": "inputs larger than L2 (%.2f GB of packed weights per step)" % packed_gb,
                       "parallelism": f"dp{world} (M split, replicated weights)", "path": args.path},
            "speedup_vs_dense": ms_d / ms_h, "dense_ms_per_step": ms_d,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops_sustained"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops_sustained"],
                         "traffic": measured_traffic(kernel_name, (args.workload, M, args.tile)),
                         "kernel": kernel_name,
                         "work": "2*M per kept weight of every loaded slab (a 2:4 slab counts half)",
                         "peak_kind": f"bf16 sustained ({peaks['source']})"},
            "gpu_launches": n_launch * args.steps,
            "clocks": clocks,
            "sweep": sweep, "e2e": e2e, "decode": decode, "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    free_model(model)
    hdist.shutdown(dist_on)


if __name__ == "__main__":
    main()
