"""Benchmark of the hybrid dense / 2:4 linear layer (PATCH) on B200.

Default workload: every linear of a Llama-2-7B-shaped model (32 layers x q, k,
v, o, gate, up, down) at M = 2048 tokens, bf16, 128x128 tiles. The headline
point is 90% of tiles 2:4 overall (45% sparsity), each linear's 2:4 fraction
drawn in [0.8, 1.0] and adjusted to the exact global count; the sweep repeats
the step at 2:4 fractions 0 / 0.5 / 0.7 / 0.9 / 1.0 (sparsity 0 / 25 / 35 /
45 / 50%). One step runs all 224 linears once on their synthetic inputs, one
grouped launch per layer; weights and activations are already resident in HBM.
The step's working set (about 9 GB of packed weights) is far larger than L2,
so no flush is needed between steps.

Reported (one JSON line from rank 0):
  value        dense-equivalent TFLOP/s = 2*M*sum(N*K) / step time, all ranks
  speedup_vs_dense  step time of the same kernel on the all-dense packing of
               the same weights / hybrid step time
  sweep        the same step at each 2:4 fraction of the sweep
  roofline     the method's tensor work (2*M per kept weight: a 2:4 tile
               counts half) per second of the step, whose only launches are
               the large-M kernel, against the measured bf16 peak (burst for
               a timed region under 2 s, sustained for longer ones under the
               power cap)
  llama2_13b   Llama-2-13B linears at M = 8192, 45% sparsity, for each of the
               four tile shapes, with its own dense run
  cublas_bf16  torch.matmul (cuBLAS) on the dense weights of the same shapes,
               context only (not on the measured path)
  e2e          the same metric through patch_group_linear_host (host buffers,
               copies inside the timed region)
  cpu_baseline the CPU oracle on a bounded sample of the same workload, on all
               host cores and on one
  decode       on Llama-2-7B layer shapes (GB/s of the bytes that must be read):
               the tensor-core decode kernel and the CUDA-core one at M = 1, 4,
               16; the decode kernel and the single-CTA GEMM at M = 32, 64; the
               automatic choice at M = 128

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
# (one Llama-2-7B layer, M = 2048, 90 % 2:4 tiles), from an ncu capture, with
# the sha256 prefix of the kernel source it was taken on: reported only while
# that source is unchanged.
MEASURED_TRAFFIC = {
    "hybrid_gemm22_kernel": {"source": "hybrid_sparse_gemm_b200/csrc/gemm22.cu", "sha256": "a31ae1d85c04c402",
                             "workload": ("llama2-7b", 2048, "128x128"), "bytes_per_launch": 630.15e6},
}
KERNEL_NAMES = {4: "hybrid_gemm2_kernel (CTA pair, 256x256 tiles)",
                6: "hybrid_gemm22_kernel (CTA pair, two strips per CTA, 512x240 tiles)",
                7: "hybrid_gemm22_kernel (CTA pair, two strips per CTA, 512x240 tiles; pure 2:4 instance)",
                3: "hybrid_gemm_kernel (single CTA, 128x128 tiles)"}


def measured_traffic(kernel_name: str, workload=("llama2-7b", 2048, "128x128")):
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
    "llama2-7b": (synth.llama2_7b, 2048, 32, "Llama-2-7B"),
    "llama32-1b": (synth.llama32_1b, 4096, 16, "Llama-3.2-1B"),
    "llama2-13b": (synth.llama2_13b, 8192, 2, "Llama-2-13B"),
}
DEFAULT_WORKLOAD = "llama2-7b"
TILES = ["128x128", "128x64", "64x128", "64x64"]


def model_linears(n_layers: int, shapes=synth.llama2_7b):
    out = []
    for layer in range(n_layers):
        for l in shapes():
            out.append((layer, l))
    return out


ROLE_INPUT = {"q": "attn", "k": "attn", "v": "attn", "o": "o", "gate": "mlp", "up": "mlp", "down": "down"}


class Member:
    """One packed linear of the model with its input and output buffers.

    kept: weights the method multiplies (N*K minus the mask's zeros);
    executed: weights the tensor-core kernel multiplies (a 2:4 slab whose
    partner strip's slab is dense runs from its dense image)."""

    def __init__(self, lin, K, N, info, X, Y):
        self.lin, self.K, self.N, self.X, self.Y = lin, K, N, X, Y
        self.kept = N * K - int(info.pruned)
        self.executed = (int(info.slabs_total) - int(info.slabs_pair_sparse)) * 128 * 64 + \
            int(info.slabs_pair_sparse) * 128 * 32
        self.packed_bytes = int(info.packed_bytes)
        self.sparse_area = int(info.tiles_sparse) * int(info.tile_rows) * int(info.tile_cols)
        self.pair_sparse_area = int(info.slabs_pair_sparse) * 128 * 64


def build_model(hsg, n_layers: int, frac: float, M: int, seed: int, lo=0.8, hi=1.0, rank=0, group=True,
                shapes=synth.llama2_7b, R=128, C=128):
    """Packs every linear of the model at global 2:4 fraction `frac`.

    Returns (layers, X, frac): layers is a list of per-layer launches, each
    (LinearGroup or None, [Member]). q/k/v read one input, gate/up another,
    o and down their own; every linear writes its own output."""
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
        Yt = torch.empty((M, l.N), dtype=torch.bfloat16, device="cuda")
        per_layer.setdefault(layer, []).append(Member(lin, l.K, l.N, lin.info(), X[ROLE_INPUT[l.name]], Yt))
        del p
    torch.cuda.synchronize()
    layers = []
    for layer in sorted(per_layer):
        mem = per_layer[layer]
        if group:
            layers.append((hsg.LinearGroup([m.lin for m in mem]), mem))
        else:
            for m in mem:
                layers.append((None, [m]))
    return layers, X, sum(counts) / sum(T)


def free_model(layers):
    for g, mem in layers:
        if g is not None:
            g.free()
        for m in mem:
            m.lin.free()


def run_step(hsg, model, stream, path=0):
    for g, mem in model:
        if g is not None:
            g([m.X for m in mem], [m.Y for m in mem], path=path, stream=stream)
        else:
            m = mem[0]
            hsg.patch_linear_path(m.lin.handle, m.X, m.Y, path, stream)


def time_steps(hsg, model, steps, warmup, stream, dist_on, path=0):
    """Mean device time of one step (ms) over `steps` timed steps, max over
    ranks: CUDA events on the launching stream, a barrier and a device
    synchronisation on both sides."""
    from hybrid_sparse_gemm_b200 import dist as hdist
    for _ in range(warmup):
        run_step(hsg, model, stream, path)
    torch.cuda.synchronize()
    hdist.barrier(dist_on)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(steps):
        run_step(hsg, model, stream, path)
    end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    hdist.barrier(dist_on)
    return hdist.max_over_ranks(ms, dist_on, device="cuda") / steps


def members(model):
    return [m for _, mem in model for m in mem]


def flops_dense(model, M):
    return sum(2.0 * M * m.N * m.K for m in members(model))


def flops_kept(model, M):
    return sum(2.0 * M * m.kept for m in members(model))


def flops_executed(model, M):
    return sum(2.0 * M * m.executed for m in members(model))


def choose_peak(peaks, timed_s: float, clocks) -> tuple[float, str]:
    """The measured bf16 peak of the clock regime the timed region ran in: the
    burst figure while the SM clock stays near its maximum; the sustained one
    (a loop held under the 1 kW power cap) when the power cap was active and
    the median SM clock sat well below the maximum (under 95 %), or when the
    region ran for seconds under the cap."""
    reasons = clocks.get("reasons") or []
    capped = "sw_power_cap" in reasons
    mhz, max_mhz = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    throttled = capped and mhz is not None and max_mhz and mhz < 0.95 * max_mhz
    if throttled or (capped and timed_s >= 2.0):
        why = (f"median SM clock {mhz:.0f} of {max_mhz:.0f} MHz under the power cap" if throttled
               else f"{timed_s:.1f} s under the power cap")
        return peaks["bf16_tflops_sustained"], f"bf16 sustained ({peaks['source']}): {why}"
    return peaks["bf16_tflops"], f"bf16 burst ({peaks['source']}): timed region {timed_s:.2f} s"


def roofline(model, M, ms_per_step, launches_per_step, peak, peak_kind, kernel_name, traffic, peaks=None):
    """The step's launches are all the large-M kernel, back to back, so the
    kernel's average launch time is the step time over its launches."""
    algo = flops_kept(model, M)
    achieved = algo / (ms_per_step / 1e3) / 1e12
    peaks_cache = peaks or {"bf16_tflops": peak, "bf16_tflops_sustained": peak}
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "frac_of_burst": achieved / peaks_cache["bf16_tflops"],
            "frac_of_sustained": achieved / peaks_cache["bf16_tflops_sustained"],
            "traffic": traffic, "kernel": kernel_name, "peak_kind": peak_kind,
            "kernel_ms_per_launch": ms_per_step / launches_per_step,
            "work": "2*M per kept weight (N*K minus the mask's zeros) of every linear, per launch",
            "executed_frac": flops_executed(model, M) / (ms_per_step / 1e3) / 1e12 / peak}


# ------------------------------------------------------------ CPU oracle ---

def _libgomp():
    import ctypes
    try:
        return ctypes.CDLL("libgomp.so.1")
    except OSError:
        return None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


class OracleSample:
    """The oracle on a bounded sample of the workload: token rows of the 7
    linears of one layer. Building the inputs and calibrating the cost model
    happen once; `run(rows)` is one timed sample."""

    def __init__(self, workload: str = DEFAULT_WORKLOAD, M: int | None = None, R: int = 128, C: int = 128,
                 seed: int = 0, threads: int | None = None):
        import oracle
        oracle.build()
        self.oracle = oracle
        shape_fn, default_M, _, self.model_name = WORKLOADS[workload]
        self.M = M or default_M
        self.shapes = shape_fn()
        self.probs = [synth.make_problem(l.N, l.K, self.M, R=R, C=C, frac=0.9, seed=seed, tag=f"cpu-{l.name}")
                      for l in self.shapes]
        self.bits = [p.bits.numpy() for p in self.probs]
        gomp = _libgomp()
        if gomp is not None and threads:
            gomp.omp_set_num_threads(int(threads))
        self.threads = int(gomp.omp_get_max_threads()) if gomp is not None else (os.cpu_count() or 1)
        # calibrate: time 4 and 16 rows of every linear (after one untimed call
        # that starts the thread pool) and fit time = fixed + rows * per_row; the
        # fixed part (mask expansion over the whole weight) does not shrink with rows
        oracle.linear(self.probs[0].X[:1], self.probs[0].W, self.bits[0])
        t4, t16 = self.run(4)[1], self.run(16)[1]
        self.per_row = max((t16 - t4) / 12.0, 1e-6)
        self.fixed = max(t4 - 4 * self.per_row, 0.0)

    def set_threads(self, n: int):
        gomp = _libgomp()
        if gomp is not None:
            gomp.omp_set_num_threads(int(n))
            self.threads = int(gomp.omp_get_max_threads())
            return True
        return False

    def rows_for(self, budget_s: float, min_rows: int = 1, per_row: float | None = None) -> int:
        per_row = per_row or self.per_row
        return max(min_rows, min(self.M, int((budget_s - self.fixed) / per_row)))

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


def cpu_sample(budget_s: float = 15.0, seed: int = 0, min_rows: int = 1, workload: str = DEFAULT_WORKLOAD,
               M: int | None = None, R: int = 128, C: int = 128, one_core_s: float = 0.0):
    """One bounded oracle sample of about `budget_s` seconds on all host
    threads, then (if one_core_s > 0) one of about `one_core_s` seconds on one
    thread. Returns a cpu_baseline dict (value in dense-equivalent TFLOP/s)."""
    s = OracleSample(workload, M, R, C, seed)
    rows = s.rows_for(budget_s, min_rows)
    v, t = s.run(rows)
    out = {"value": v, "unit": "TFLOP/s", "cores": s.threads, "kind": "oracle", "sample": s.describe(rows, t),
           "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    if one_core_s > 0 and s.set_threads(1):
        # the per-row cost grows about with the thread count
        rows1 = s.rows_for(one_core_s, 1, per_row=s.per_row * max(1, out["cores"]))
        v1, t1 = s.run(rows1)
        out["value_1core"] = v1
        out["sample_1core"] = s.describe(rows1, t1) + ", 1 thread"
    return out


# ----------------------------------------------------------- context runs ---

def cublas_bf16(shapes, M: int, stream, layers: int = 4, steps: int = 10):
    """torch.matmul (cuBLAS) on dense bf16 weights of the same shapes, layers
    rotated so that the weights stream from HBM. Context only: the measured
    path never calls it."""
    Ws = [[synth.normal_bf16((l.N, l.K), 0.02, "cuda", "cublas", L, l.name) for l in shapes()] for L in range(layers)]
    Xs = {l.K: synth.normal_bf16((M, l.K), 1.0, "cuda", "cublasX", l.K) for l in shapes()}
    Ys = [torch.empty((M, l.N), dtype=torch.bfloat16, device="cuda") for l in shapes()]
    with torch.cuda.stream(stream):
        def step():
            for W in Ws:
                for w, y in zip(W, Ys):
                    torch.matmul(Xs[w.shape[1]], w.t(), out=y)
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(steps):
            step()
        e.record(stream)
        torch.cuda.synchronize()
    ms_layer = s.elapsed_time(e) / (steps * layers)
    fl = sum(2.0 * M * l.N * l.K for l in shapes())
    del Ws, Xs, Ys
    return {"ms_per_layer": ms_layer, "tflops": fl / (ms_layer / 1e3) / 1e12, "layers_rotated": layers,
            "note": "context only: torch.matmul (cuBLAS) on dense bf16 weights, not on the measured path"}


def decode_bench(hsg, stream, peaks, steps=20, Ms=(1, 4, 16, 32, 64, 128)):
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
    for M in Ms:
        X = {K: synth.normal_bf16((M, K), 1.0, "cuda", "decX", M, K) for K in (4096, 11008)}
        Y = [[torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _, _, N, _ in mem] for _, mem in layers]
        res = {}
        # M <= 16: the tensor-core decode kernel (16-token MMAs) and the
        # CUDA-core one; 16 < M <= 64: the decode kernel's 64-token instance
        # and the single-CTA GEMM (one 128-token tile, so each weight record
        # is still read once, but no split-K); above: the library's choice
        if M <= 16:
            paths = (("tc", hsg.PATH_GEMV), ("simt", hsg.PATH_GEMV_SIMT))
        elif M <= 64:
            paths = (("tc", hsg.PATH_GEMV), ("gemm", hsg.PATH_GEMM_SINGLE))
        else:
            paths = (("auto", hsg.PATH_AUTO),)
        for name, path in paths:
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
                         "us_per_layer": ms * 1e3 / (steps * len(layers)),
                         "tflops": steps * sum(2.0 * M * K * N for _, mem in layers for _, K, N, _ in mem)
                         / (ms / 1e3) / 1e12}
        out[f"M{M}"] = res
    for g, mem in layers:
        g.free()
        for m in mem:
            m[0].free()
    return out


def kernel_label(hsg, model, M, gpath):
    g = model[0][0]
    p = g.path(M, gpath) if g is not None else hsg.PATH_GEMM_PAIR
    return KERNEL_NAMES.get(p, "tensor-core GEMM")


def llama2_13b_tiles(hsg, stream, peaks, steps, warmup, dist_on, rank, gpath, tiles=TILES, layers=2):
    """Llama-2-13B linears at M = 8192, 90% 2:4 tiles (45% sparsity), for each
    tile shape, each against the all-dense packing of the same shapes."""
    M = 8192
    with torch.cuda.stream(stream):
        dense, _, _ = build_model(hsg, layers, 0.0, M, seed=1, rank=rank, shapes=synth.llama2_13b)
    ms_d = time_steps(hsg, dense, steps, warmup, stream, dist_on, gpath)
    free_model(dense)
    del dense
    out = {"workload": f"Llama-2-13B linears ({layers} layers x q,k,v,o,gate,up,down), M={M} tokens, bf16, "
                       "90% 2:4 tiles (45% sparsity), per-linear fraction in [0.8,1.0]",
           "dense_ms_per_step": ms_d}
    for tile in tiles:
        R, C = (int(v) for v in tile.split("x"))
        with torch.cuda.stream(stream):
            mdl, _, frac = build_model(hsg, layers, 0.9, M, seed=1, rank=rank, shapes=synth.llama2_13b, R=R, C=C)
        ms = time_steps(hsg, mdl, steps, warmup, stream, dist_on, gpath)
        F = flops_dense(mdl, M)
        algo = flops_kept(mdl, M) / (ms / 1e3) / 1e12
        mem = members(mdl)
        out[tile] = {"tflops": F / (ms / 1e3) / 1e12, "speedup_vs_dense": ms_d / ms, "ms_per_step": ms,
                     "frac_2to4": frac, "roofline_frac_of_burst": algo / peaks["bf16_tflops"],
                     "roofline_frac_of_sustained": algo / peaks["bf16_tflops_sustained"],
                     "sparse_area_run_sparse": sum(m.pair_sparse_area for m in mem) /
                     max(1, sum(m.sparse_area for m in mem))}
        free_model(mdl)
        del mdl
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS),
                    help="model whose linears one step runs (default: Llama-2-7B, 32 layers, M = 2048)")
    ap.add_argument("--layers", type=int, default=None, help="layers per step (default per workload)")
    ap.add_argument("--M", type=int, default=None, help="tokens (default per workload)")
    ap.add_argument("--tile", default="128x128", choices=TILES, help="mask tile shape")
    ap.add_argument("--no-group", action="store_true", help="one launch per linear instead of per layer")
    ap.add_argument("--path", default="auto", choices=["auto", "pair", "wide"],
                    help="tensor-core kernel for the timed steps (auto: the library's choice)")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-13b", action="store_true", help="skip the Llama-2-13B tile-shape runs")
    ap.add_argument("--no-cublas", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-M", default="1,4,16,32,64,128",
                    help="token counts of the decode section, comma-separated")
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
                f"bf16, {R}x{C} tiles, 90% 2:4 tiles (45% sparsity), per-linear fraction in [0.8,1.0]; "
                f"sweep over 2:4 fractions {'/'.join(str(f) for f in FRACS_SWEEP)}")

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
                             "sample": desc, "cpu_model": cpu_model()},
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
    nvtx = torch.cuda.nvtx  # phase markers for profilers; nothing inside the timed loops

    with torch.cuda.stream(stream):
        model, X, frac_real = build_model(hsg, args.layers, 0.9, M, seed=0, rank=rank, group=group,
                                          shapes=shape_fn, R=R, C=C)
        dense_model, _, _ = build_model(hsg, args.layers, 0.0, M, seed=0, rank=rank, group=group,
                                        shapes=shape_fn, R=R, C=C)
    torch.cuda.synchronize()
    F = flops_dense(model, M)
    n_launch = len(model)

    with ClockSampler(torch.cuda.current_device()) as clk, nvtx.range("hybrid steps"):
        ms_h = time_steps(hsg, model, args.steps, args.warmup, stream, dist_on, path=gpath)
    clocks = clk.summary()
    with nvtx.range("dense steps"):
        ms_d = time_steps(hsg, dense_model, args.steps, args.warmup, stream, dist_on, path=gpath)
    kernel_name = kernel_label(hsg, model, M, gpath)
    peak, peak_kind = choose_peak(peaks, ms_h * args.steps / 1e3, clocks)
    roof = roofline(model, M, ms_h, n_launch, peak, peak_kind, kernel_name,
                    measured_traffic(kernel_name, (args.workload, M, args.tile)), peaks)
    roof["sm_mhz"] = clocks.get("sm_mhz")
    value = hdist.job_rate(F, world, ms_h) / 1e12

    sweep = None
    if not args.no_sweep:
        sweep = {}
        for f in FRACS_SWEEP:
            if f == 0.0:
                t, mdl = ms_d, dense_model
            elif f == 0.9:
                t, mdl = ms_h, model
            else:
                with torch.cuda.stream(stream):
                    mdl, _, _ = build_model(hsg, args.layers, f, M, seed=0, rank=rank, group=group,
                                            shapes=shape_fn, R=R, C=C)
                with nvtx.range(f"sweep f={f}"):
                    t = time_steps(hsg, mdl, args.steps, args.warmup, stream, dist_on, path=gpath)
            sweep[str(f)] = {"tflops": hdist.job_rate(F, world, t) / 1e12, "speedup_vs_dense": ms_d / t,
                             "ms_per_step": t, "sparsity": 0.5 * f,
                             "roofline_frac": flops_kept(mdl, M) / (t / 1e3) / 1e12 / peak}
            if f not in (0.0, 0.9):
                free_model(mdl)
                del mdl
    free_model(dense_model)
    dense_model = []

    e2e = None
    if not args.no_e2e and group:
        # Host memory in and out through patch_group_linear_host, one call per
        # layer: each layer uploads its distinct inputs (q, k, v share one) and
        # brings every output back, in token chunks whose copies overlap the
        # product and each other. Each layer has its own pinned input and
        # output buffers, as the activations of successive layers would.
        Xh, Yh = [], []
        for g, mem in model:
            cache = {}
            Xh.append([cache.setdefault(id(m.X), m.X.cpu().pin_memory()) for m in mem])
            Yh.append([torch.empty(m.Y.shape, dtype=torch.bfloat16).pin_memory() for m in mem])
        h2d = sum(sum(M * x.shape[1] * 2 for x in {id(x): x for x in xs}.values()) for xs in Xh)
        d2h = sum(M * m.N * 2 for m in members(model))
        e2e_steps = max(1, min(args.steps, 3))

        # Layers alternate between two streams: each call makes its stream wait
        # for its own copies back, so one stream would hold the next layer's
        # product behind them; with two, the copy engines stay busy.
        streams = [stream, torch.cuda.Stream()]

        def e2e_step():
            for i, ((g, mem), xs, ys) in enumerate(zip(model, Xh, Yh)):
                g.host(xs, ys, path=gpath, stream=streams[i % 2], sync=False)

        e2e_step()  # warm-up: staging buffers and copy streams
        torch.cuda.synchronize()
        hdist.barrier(dist_on)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        joined = torch.cuda.Event()
        torch.cuda.synchronize()
        s.record(stream)
        streams[1].wait_event(s)
        for _ in range(e2e_steps):
            e2e_step()
        joined.record(streams[1])
        stream.wait_event(joined)
        e.record(stream)
        torch.cuda.synchronize()
        ms_e = s.elapsed_time(e) / e2e_steps
        ms_e = hdist.max_over_ranks(ms_e, dist_on, device="cuda")
        e2e = {"value": hdist.job_rate(F, world, ms_e) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ms_e,
               "call": "patch_group_linear_host per layer, layers alternating over two streams (pinned host "
                       "buffers, chunked copies overlapped)"}
        del Xh, Yh

    packed_gb = sum(m.packed_bytes for m in members(model)) / 1e9
    linears = len(members(model))
    free_model(model)
    model = []

    big = None
    if args.workload == DEFAULT_WORKLOAD and not args.no_13b:
        with nvtx.range("llama2-13b tiles"):
            big = llama2_13b_tiles(hsg, stream, peaks, args.steps, args.warmup, dist_on, rank, gpath)

    cublas = None
    if rank == 0 and not args.no_cublas:
        with nvtx.range("cublas context"):
            cublas = cublas_bf16(shape_fn, M, stream)
            cublas["same_step_ms"] = cublas["ms_per_layer"] * args.layers

    decode = None
    if not args.no_decode:
        with nvtx.range("decode"):
            decode = decode_bench(hsg, stream, peaks, Ms=tuple(int(m) for m in args.decode_M.split(",")))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_sample(workload=args.workload, M=args.M, R=R, C=C, one_core_s=8.0)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_h, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload, "M": M, "layers": args.layers, "linears": linears,
                       "launches_per_step": n_launch, "grouped": group,
                       "frac_2to4": frac_real, "tile": args.tile,
                       "l2": "inputs larger than L2 (%.2f GB of packed weights per step)" % packed_gb,
                       "parallelism": f"dp{world} (M split, replicated weights)", "path": args.path},
            "speedup_vs_dense": ms_d / ms_h, "dense_ms_per_step": ms_d,
            "roofline": roof,
            "gpu_launches": n_launch * args.steps,
            "clocks": clocks,
            "sweep": sweep, "llama2_13b": big, "cublas_bf16": cublas,
            "e2e": e2e, "decode": decode, "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    hdist.shutdown(dist_on)


if __name__ == "__main__":
    main()
