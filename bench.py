"""Benchmark: GPTQ layer-wise quantization of one 7B-shaped linear layer per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = the whole hot path over one layer with its inputs resident in HBM:
  Hessian 2·XᵀX over the calibration tokens (tensor cores) -> damping -> act_order (if on) ->
  Cholesky + triangular inverse (U) -> blocked column loop with OBS compensation + lazy batch
  updates -> output assembly -> reconstruction loss -> group min-max RTN baseline of the same W.
Default workload ``mlp_up_7b``: W 11008x4096 fp16, X 262144x4096 fp16, INT4 g128 B128,
percdamp 0.01. value = weights quantized per second over all ranks (each rank quantizes its
own layer: weak scaling, no data-path collective).

Prints one JSON line on rank 0. ``--impl reference`` times the fp64 CPU checker on a bounded
sample of the same workload instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from post_weight_quantization_24_b200 import workloads  # noqa: E402

METRIC = "GPTQ weights quantized/s & calib tokens/s per layer; % roofline per stage"
UNIT = "weights/s"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
N_SM, FP32_LANES_PER_SM = 148, 128
TF32_PER_BF16 = round(1.1 / 2.25, 4)   # nominal dense tf32 : bf16 tensor rates on B200


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except (OSError, ValueError):
        p = dict(FALLBACK_PEAKS)
        p["source"] = "fallback"
        return p


# ------------------------------------------------------------------------------------------
# distributed plumbing (one process per GPU)
# ------------------------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local, backend="nccl"):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world > 1


def max_over_ranks(x: float, distributed: bool, device) -> float:
    if not distributed:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(name: str, rank: int) -> workloads.LayerWorkload:
    """Each rank quantizes its own layer of the named shape: the same recipe, seed + rank."""
    base = workloads.WORKLOADS[name]
    return base.replace(seed=base.seed + rank)


def job_value(world: int, steps: int, weights_per_step: int, total_ms_max: float) -> float:
    """Weights quantized per second by the whole job: every rank's units over the slowest
    rank's time (weak scaling: each rank does a fixed amount of work)."""
    return world * steps * weights_per_step / (total_ms_max / 1e3)


def barrier(distributed: bool):
    if distributed:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "timestamp")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", "GPU-" + uuid if not uuid.startswith("GPU-") else uuid]
        except Exception:
            sel = []
        self.sel = sel

    def start(self, wait_s: float = 5.0):
        """Start sampling every 20 ms and wait (up to wait_s) for the first sample, so that the
        sampler is running before the timed region begins."""
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", *self.sel], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < wait_s and os.path.getsize(self.path) == 0:
            time.sleep(0.01)

    def mark(self):
        """Wall-clock marks of the timed region (the samples' timestamps are wall clock)."""
        return time.time()

    def stop(self, t_begin=None, t_end=None):
        if self.proc is None:
            return None
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows, inside = [], []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                row = dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                           hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8])
            except ValueError:
                continue
            rows.append(row)
            try:
                import datetime
                ts = datetime.datetime.strptime(parts[9], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if t_begin is not None and t_begin - 0.05 <= ts <= t_end + 0.05:
                    inside.append(row)
            except ValueError:
                pass
        os.unlink(self.path)
        if inside:
            rows = inside
        if not rows:
            return None
        busy = [r for r in rows if r["power"] > 250.0] or rows
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in busy),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "power_w_max": max(r["power"] for r in rows),
                "samples": len(rows), "samples_under_load": len(busy),
                "samples_in_timed_region": len(inside),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------
# the committed ncu summary of the dominant kernel (traffic is null if the kernel changed)
# ------------------------------------------------------------------------------------------
def code_sha(source_file: str) -> str:
    """sha256 of a kernel source with comments and blank lines removed: an edit of comments
    alone leaves it unchanged, any edit of the code changes it."""
    src = os.path.join(ROOT, "post_weight_quantization_24_b200", "csrc", source_file)
    text = re.sub(r"/\*.*?\*/", "", open(src).read(), flags=re.S)
    lines = [ln.split("//", 1)[0].rstrip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def ncu_traffic(summary_name: str, source_file: str):
    """DRAM bytes per full-size launch from a committed ncu summary, or None when the summary is
    missing or the kernel's code has changed since its capture."""
    path = os.path.join(ROOT, "profiles", summary_name)
    try:
        text = open(path).read()
    except OSError:
        return None, None
    m_h = re.search(r"kernel_code_sha256:\s*([0-9a-f]{64})", text)
    m_b = re.search(r"dram_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text)
    if not (m_h and m_b):
        return None, path
    if code_sha(source_file) != m_h.group(1):
        return None, path
    return float(m_b.group(1)), path


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------
class LayerStep:
    """All device buffers for one layer and the step that quantizes it."""

    def __init__(self, gptq, wl: workloads.LayerWorkload, device):
        self.gptq, self.wl, self.device = gptq, wl, device
        self.W = workloads.make_weights(wl, device=device)
        self.X = workloads.make_activations(wl, device=device)
        self.h = gptq.Hessian(wl.d_in)
        self.Hraw = self.h.raw()
        ng = wl.d_in // wl.group_size
        self.out = dict(codes=torch.empty(wl.d_out, wl.d_in, dtype=torch.uint8, device=device),
                        scales=torch.empty(wl.d_out, ng, dtype=torch.float16, device=device),
                        zeros=torch.empty(wl.d_out, ng, dtype=torch.float16, device=device),
                        g_idx=torch.empty(wl.d_in, dtype=torch.int32, device=device),
                        perm=torch.empty(wl.d_in, dtype=torch.int32, device=device))
        self.rtn_out = (torch.empty(wl.d_out, wl.d_in // 2 if wl.bits == 4 else wl.d_in,
                                    dtype=torch.uint8, device=device),
                        torch.empty(wl.d_out, ng, dtype=torch.float16, device=device),
                        torch.empty(wl.d_out, ng, dtype=torch.float16, device=device))
        nbytes = gptq.quantize_layer_workspace(wl.d_out, wl.d_in, wl.block_size)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.ev = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for k in ("hessian", "gptq", "rtn")}
        self.loss = None

    def run(self, timed=False):
        g, wl = self.gptq, self.wl
        e = self.ev
        if timed:
            e["hessian"][0].record()
        self.h.reset()
        self.h.accumulate(self.X)
        if timed:
            e["hessian"][1].record()
            e["gptq"][0].record()
        res = g.quantize_layer(self.W, self.Hraw, bits=wl.bits, group_size=wl.group_size,
                               block_size=wl.block_size, percdamp=wl.percdamp,
                               act_order=wl.act_order, compute_loss=True, workspace=self.ws,
                               out=self.out)
        self.loss = res["loss"]
        if timed:
            e["gptq"][1].record()
            e["rtn"][0].record()
        g.rtn_minmax_quantize(self.W, wl.bits, wl.group_size, out=self.rtn_out)
        if timed:
            e["rtn"][1].record()

    def stage_ms(self):
        return {k: a.elapsed_time(b) for k, (a, b) in self.ev.items()}


def rtn_stack_measure(gptq, device, reps: int = 3):
    """Group min-max RTN (INT4, g128) over the weights of a 7B-shaped decoder stack: 32 layers x
    {q, k, v, o 4096x4096; gate, up 11008x4096; down 4096x11008}, 6.48e9 fp16 weights (13 GB),
    far larger than L2. The matrices of one input width are quantized as one row block (RTN is
    row-independent), so each repetition is two launches; CUDA events bracket back-to-back
    repetitions on the launching stream. Weights: N(0, 0.02) with 0.1% of input columns x20."""
    g = torch.Generator(device=device).manual_seed(1234)
    shapes = ((32 * (4 * 4096 + 2 * 11008), 4096), (32 * 4096, 11008))
    bufs = []
    for rows, cols in shapes:
        W = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float16)
        W.mul_(0.02)
        outl = torch.randperm(cols, generator=g, device=device)[:max(1, round(0.001 * cols))]
        W[:, outl] *= 20
        out = (torch.empty(rows, cols // 2, dtype=torch.uint8, device=device),
               torch.empty(rows, cols // 128, dtype=torch.float16, device=device),
               torch.empty(rows, cols // 128, dtype=torch.float16, device=device))
        bufs.append((W, out))
    n = sum(r * c for r, c in shapes)
    for W, out in bufs:                       # warm-up
        gptq.rtn_minmax_quantize(W, 4, 128, out=out)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        for W, out in bufs:
            gptq.rtn_minmax_quantize(W, 4, 128, out=out)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    nbytes = n * 2.5 + n // 128 * 4
    del bufs
    torch.cuda.empty_cache()
    return {"ms": ms, "weights": n, "bytes": nbytes, "gbs": nbytes / (ms / 1e3) / 1e9,
            "weights_per_s": n / (ms / 1e3), "launches": 2 * reps}


def gptq_flops(d_out: int, d: int, B: int, w_f16: bool = True) -> dict:
    """Algorithmic flops of one quantize_layer call, per stage (symmetric Hessian work is
    counted once; the loss denominator is the Gram matrix on the fp16 path)."""
    return {"factor": 2.0 * d ** 3 / 3.0,
            "column_loop": float(d_out) * d * B,
            "lazy_update": 2.0 * d_out * sum(B * max(0, d - j0 - B) for j0 in range(0, d, B)),
            "loss": float(d_out) * d * (d + 1) if w_f16 else 2.0 * d_out * d * d}


def peaks_for(peaks, clock_mhz):
    tc = peaks["bf16_tflops"]                            # fp16 MMA runs at the bf16 rate
    return {"tensor": tc, "tf32x3": tc * TF32_PER_BF16 / 3.0,
            "ffma": N_SM * FP32_LANES_PER_SM * 2 * clock_mhz * 1e6 / 1e12}


def stage_entry(ms, bound, flops=None, peak=None, note=None):
    out = {"ms": ms, "bound": bound}
    if flops is not None and ms > 0:
        out["tflops"] = flops / (ms / 1e3) / 1e12
        out["peak_tflops"] = peak
        out["frac"] = out["tflops"] / peak
    if note:
        out["peak_note"] = note
    return out


TF32X3_NOTE = f"tf32 = {TF32_PER_BF16} x measured bf16, / 3 MMA passes (3xTF32)"


def gptq_stage_table(hess_flops, hess_ms, lib_ms, fl, pk, clock_mhz, w_f16=True, n_tokens=None,
                     d=None):
    """Per-stage times and roofline fractions of one layer (or a sum of layers)."""
    st = {
        "hessian": stage_entry(hess_ms, "tensor", hess_flops, pk["tensor"],
                               "measured bf16 dense burst"),
        "prepare": {"ms": lib_ms["prepare"]},
        "factor": stage_entry(lib_ms["factor"], "tensor", fl["factor"], pk["tf32x3"],
                              TF32X3_NOTE + "; Cholesky and triangular inverse, two streams"),
        "images": {"ms": lib_ms["images"]},
        "column_loop": stage_entry(lib_ms["column_loop"], "alu", fl["column_loop"], pk["ffma"],
                                   f"FFMA 148 SM x 128 lanes x 2 at the sampled {clock_mhz:.0f} MHz"),
        "lazy_update": stage_entry(lib_ms["lazy_update"], "tensor", fl["lazy_update"],
                                   pk["tf32x3"], TF32X3_NOTE),
        "assemble": {"ms": lib_ms["assemble"]},
        "loss": stage_entry(lib_ms["loss"], "tensor", fl["loss"],
                            pk["tensor"] if w_f16 else pk["tf32x3"],
                            "Gram matrix on the fp16 path; measured bf16 dense burst" if w_f16
                            else TF32X3_NOTE),
    }
    if n_tokens is not None and hess_ms > 0:
        st["hessian"]["calib_tokens_per_s"] = n_tokens / (hess_ms / 1e3)
    if d is not None and lib_ms["column_loop"] > 0:
        st["column_loop"]["us_per_column_step"] = lib_ms["column_loop"] * 1e3 / d
    return st


def measure_config(gptq, wl, device, flush, steps, warmup, peaks, clock_mhz):
    """One timed line for a layer workload: the same step as the headline (Hessian, GPTQ with
    loss, RTN of the same W), with its per-stage roofline fractions."""
    step = LayerStep(gptq, wl, device)
    gptq.profile_enable(False)
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    tot, stage_tot = 0.0, {k: 0.0 for k in ("hessian", "gptq", "rtn")}
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step.run(timed=True)
        b.record()
        torch.cuda.synchronize()
        tot += a.elapsed_time(b)
        for k, v in step.stage_ms().items():
            stage_tot[k] += v
    lib_tot = {k: 0.0 for k in gptq.STAGES}
    gptq.profile_enable(True)
    for _ in range(steps):
        flush.zero_()
        step.run()
        torch.cuda.synchronize()
        for k, v in gptq.profile_read().items():
            lib_tot[k] += v
    gptq.profile_enable(False)
    ms = tot / steps
    d, n, d_out = wl.d_in, wl.n_tokens, wl.d_out
    pk = peaks_for(peaks, clock_mhz)
    fl = gptq_flops(d_out, d, wl.block_size, wl.w_dtype == "f16")
    hess_ms = stage_tot["hessian"] / steps
    st = gptq_stage_table(float(n) * d * (d + 1), hess_ms, {k: v / steps for k, v in lib_tot.items()},
                          fl, pk, clock_mhz, wl.w_dtype == "f16", n, d)
    rtn_ms = stage_tot["rtn"] / steps
    rtn_bytes = d_out * d * ((2 if wl.w_dtype == "f16" else 4) + (0.5 if wl.bits == 4 else 1.0)) \
        + d_out * (d // wl.group_size) * 4
    st["rtn"] = {"ms": rtn_ms, "bound": "hbm", "gbs": rtn_bytes / (rtn_ms / 1e3) / 1e9,
                 "frac": rtn_bytes / (rtn_ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
    out = {"workload": f"{wl.name}: W {d_out}x{d} {wl.w_dtype}, X {n}x{d} fp16, INT{wl.bits} "
                       f"g{wl.group_size} B{wl.block_size} act_order {wl.act_order}",
           "steps": steps, "warmup": warmup, "ms_per_step": ms,
           "weights_per_s": d_out * d / (ms / 1e3), "layers_per_s": 1e3 / ms,
           "calib_tokens_per_s": n / (hess_ms / 1e3), "loss": step.loss,
           "gptq_ms": stage_tot["gptq"] / steps, "stages": st}
    del step
    torch.cuda.empty_cache()
    return out


CONFIG_LINES = (("linear_512", {}), ("mlp_down_7b_int4", {"base": "mlp_down_7b", "bits": 4}),
                ("mlp_down_7b_int3", {"base": "mlp_down_7b", "bits": 3}),
                ("attn_o_70b", {}), ("mlp_down_70b", {}))


def configs_measure(gptq, device, flush, peaks, clock_mhz, steps=3, warmup=3):
    res = {}
    for name, kw in CONFIG_LINES:
        wl = workloads.WORKLOADS[kw.get("base", name)]
        if "bits" in kw:
            wl = wl.replace(bits=kw["bits"], name=name)
        try:
            res[name] = measure_config(gptq, wl, device, flush, steps, warmup, peaks, clock_mhz)
        except Exception as exc:                      # reported in the line, never fatal
            res[name] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
            torch.cuda.empty_cache()
    return res


def _events():
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def w4a16_measure(gptq, device, peaks, n_tokens=16384, d_in=4096, d_out=22016, reps=5):
    """The W4A16 layer on the 7B MLP-in shape (gate;up stacked: 22016 x 4096, INT4 g128) over
    16384 tokens, with and without the act_order gather. Algorithmic flops 2·n·d_out·d_in."""
    wl = workloads.WORKLOADS["mlp_up_7b"]
    W = workloads.make_weights(wl.replace(d_out=d_out, d_in=d_in), device=device)
    packed, scales, zeros = gptq.rtn_minmax_quantize(W, 4, 128)
    X = workloads.make_activations(wl.replace(d_in=d_in, n_tokens=n_tokens), device=device)
    Y = torch.empty(n_tokens, d_out, dtype=torch.float16, device=device)
    perm = torch.randperm(d_in, device=device).to(torch.int32)
    ws = torch.empty(gptq.lib().w4a16_linear_workspace(n_tokens, d_in, 1), dtype=torch.uint8,
                     device=device)
    out = {}
    flops = 2.0 * n_tokens * d_out * d_in
    for name, pm in (("plain", None), ("act_order_gather", perm)):
        for _ in range(2):
            gptq.w4a16_linear(X, packed, scales, zeros, 128, perm=pm, out=Y, workspace=ws)
        a, b = _events()
        a.record()
        for _ in range(reps):
            gptq.w4a16_linear(X, packed, scales, zeros, 128, perm=pm, out=Y, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        tf = flops / (ms / 1e3) / 1e12
        out[name] = {"ms": ms, "tflops": tf, "bound": "tensor", "peak_tflops": peaks["bf16_tflops"],
                     "frac": tf / peaks["bf16_tflops"]}
    out["workload"] = (f"X {n_tokens}x{d_in} fp16, W {d_out}x{d_in} INT4 g128 (7B gate;up), "
                       "fp32 accumulate, fp16 out")
    del W, X, Y, ws
    torch.cuda.empty_cache()
    return out


def sequential_measure(gptq, device, peaks, n_blocks=2, n_tokens=65536, d=4096, d_ff=11008):
    """Layer-by-layer GPTQ of `n_blocks` 7B-shaped gated-MLP blocks (gate;up 22016 x 4096,
    down 4096 x 11008, INT4 g128), each layer's Hessian from the W4A16 outputs of the layers
    before it, over 65536 calibration tokens."""
    from post_weight_quantization_24_b200 import sequential
    g = torch.Generator(device=device).manual_seed(77)
    blocks = []
    for _ in range(n_blocks):
        f = lambda r, c: (0.02 * torch.randn(r, c, generator=g, device=device)).to(torch.float16)
        blocks.append((f(d_ff, d), f(d_ff, d), f(d, d_ff)))
    X0 = workloads.make_activations(workloads.WORKLOADS["mlp_up_7b"].replace(
        d_in=d, n_tokens=n_tokens, seed=78), device=device)
    sequential.quantize_mlp_stack(X0, blocks)                # warm-up (the whole stack)
    torch.cuda.synchronize()
    passes = []                                              # (ms, stage timings, records)
    for _ in range(3):
        timings = {}
        a, b = _events()
        a.record()
        _, recs = sequential.quantize_mlp_stack(X0, blocks, timings=timings)
        b.record()
        torch.cuda.synchronize()
        passes.append((a.elapsed_time(b), timings, recs))
    passes.sort(key=lambda x: x[0])
    ms, timings, recs = passes[1]                            # the median pass
    w4_flops = n_blocks * 2.0 * n_tokens * (2 * d_ff * d + d * d_ff)
    h_flops = n_blocks * float(n_tokens) * (d * (d + 1) + d_ff * (d_ff + 1))
    out = {"blocks": n_blocks, "tokens": n_tokens, "ms": ms,
           "ms_passes": [x[0] for x in passes],
           "layers_per_s": 2 * n_blocks / (ms / 1e3),
           "weights_per_s": n_blocks * 3 * d * d_ff / (ms / 1e3),
           "stage_ms": timings,
           "w4a16_frac": w4_flops / (timings.get("w4a16", 1e-9) / 1e3) / 1e12 / peaks["bf16_tflops"],
           "hessian_frac": h_flops / (timings.get("hessian", 1e-9) / 1e3) / 1e12 / peaks["bf16_tflops"],
           "losses": {r["name"]: r["loss"] for r in recs},
           "workload": f"{n_blocks} gated-MLP blocks d={d} d_ff={d_ff}, {n_tokens} tokens, INT4 g128",
           "timing": "median of 3 passes after one untimed pass of the whole stack"}
    del blocks, X0, recs, passes
    torch.cuda.empty_cache()
    return out


def awq_clip_measure(gptq, device, peaks, reps=3):
    """AWQ-lite (11 alphas) and the RTN clip search (11 ratios, H criterion) on the mlp_up_7b
    weights, H from 65536 tokens of its activations."""
    wl = workloads.WORKLOADS["mlp_up_7b"]
    W = workloads.make_weights(wl, device=device)
    X = workloads.make_activations(wl.replace(n_tokens=65536), device=device)
    h = gptq.Hessian(wl.d_in)
    h.accumulate(X)
    H = h.get()
    sums = gptq.channel_abs_sum(X)
    res = {}
    for name, fn in (("awq_lite", lambda: gptq.awq_lite_search(W, sums, X.shape[0], H)),
                     ("rtn_clip_search", lambda: gptq.rtn_clip_search(W, 4, 128, H=H))):
        fn()
        torch.cuda.synchronize()
        a, b = _events()
        a.record()
        for _ in range(reps):
            r = fn()
        b.record()
        torch.cuda.synchronize()
        res[name] = {"ms": a.elapsed_time(b) / reps}
        if name == "awq_lite":
            res[name]["alpha"] = r["alpha"]
            d, n_a = wl.d_in, len(r["losses"])
            fl = n_a * 2.0 * wl.d_out * d * d       # the loss GEMMs, fp32-equivalent
            res[name]["loss_gemm_tflops_equiv"] = fl / (res[name]["ms"] / 1e3) / 1e12
    res["workload"] = "W 11008x4096 fp16 INT4 g128; H over 65536 tokens"
    del W, X, H, h
    torch.cuda.empty_cache()
    return res


def stack_measure(gptq, device, peaks, clock_mhz, n_layers=32, n_tokens=131072,
                  variants=((128, False), (128, True), (64, False), (64, True))):
    """GPTQ over a full 7B-shaped decoder stack, end to end: for each of `n_layers` layers,
    fresh synthetic inputs (four distinct inputs of `n_tokens` tokens, the 7B activation recipe)
    and fresh fp16 weights are generated, the four Hessians are accumulated, and the layer's
    linears are quantized (INT4, B128, loss on), q;k;v and gate;up each in one call on their
    row-stacked weights (rows are independent given the shared Hessian, so this is the same
    result as separate calls with one factorisation instead of three or two). Every quantize
    call synchronises once, as a user's would. Device time (CUDA events around the Hessians and
    the quantize calls of each layer, input synthesis excluded) and host wall time (synthesis
    included) are reported per variant, with per-stage times and roofline fractions summed over
    the stack."""
    hs = {k: gptq.Hessian(d) for k, d in workloads.DECODER_7B_INPUTS.items()}
    shapes = []
    for name, parts, d_in, src in workloads.DECODER_7B_FUSED:
        rows = sum(d_out for n_, d_out, _, _ in workloads.DECODER_7B_LINEARS if n_ in parts)
        shapes.append((name, rows, d_in, src))
    ws = torch.empty(max(gptq.quantize_layer_workspace(r, d) for _, r, d, _ in shapes),
                     dtype=torch.uint8, device=device)
    pk = peaks_for(peaks, clock_mhz)
    n_w = sum(r * d for _, r, d, _ in shapes)
    res = {}
    gptq.profile_enable(True)
    try:
        # one untimed layer per setting first: module loading and one-time kernel set-up
        inputs, fused = workloads.make_decoder_layer(n_layers, n_tokens, device=device)
        for k, X in inputs.items():
            hs[k].reset()
            hs[k].accumulate(X)
        for g, ao in variants:
            for name, W, src in fused:
                gptq.quantize_layer(W, hs[src].raw(), bits=4, group_size=g, block_size=128,
                                    act_order=ao, compute_loss=True, workspace=ws)
        del inputs, fused
        torch.cuda.synchronize()
        for g, ao in variants:
            outs = {name: dict(codes=torch.empty(r, d, dtype=torch.uint8, device=device),
                               scales=torch.empty(r, d // g, dtype=torch.float16, device=device),
                               zeros=torch.empty(r, d // g, dtype=torch.float16, device=device),
                               g_idx=torch.empty(d, dtype=torch.int32, device=device),
                               perm=torch.empty(d, dtype=torch.int32, device=device))
                    for name, r, d, _ in shapes}
            lib_ms = {k: 0.0 for k in gptq.STAGES}
            hess_ms = dev_ms = 0.0
            losses = {name: [] for name, _, _, _ in shapes}
            launches0 = gptq.launch_count()
            torch.cuda.synchronize()
            wall0 = time.perf_counter()
            for layer in range(n_layers):
                inputs, fused = workloads.make_decoder_layer(layer, n_tokens, device=device)
                a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                a.record()
                for k, X in inputs.items():
                    hs[k].reset()
                    hs[k].accumulate(X)
                b.record()
                for name, W, src in fused:
                    r = gptq.quantize_layer(W, hs[src].raw(), bits=4, group_size=g,
                                            block_size=128, act_order=ao, compute_loss=True,
                                            workspace=ws, out=outs[name])
                    losses[name].append(r["loss"])
                    for k, v in gptq.profile_read().items():
                        lib_ms[k] += v
                c.record()
                torch.cuda.synchronize()
                hess_ms += a.elapsed_time(b)
                dev_ms += a.elapsed_time(c)
                del inputs, fused
            wall_s = time.perf_counter() - wall0
            hess_flops = n_layers * sum(float(n_tokens) * d * (d + 1)
                                        for d in workloads.DECODER_7B_INPUTS.values())
            fl = {k: 0.0 for k in ("factor", "column_loop", "lazy_update", "loss")}
            for _, r, d, _ in shapes:
                for k, v in gptq_flops(r, d, 128).items():
                    fl[k] += n_layers * v
            st = gptq_stage_table(hess_flops, hess_ms, lib_ms, fl, pk, clock_mhz,
                                  n_tokens=4 * n_layers * n_tokens)
            res[f"g{g}_act_order_{'on' if ao else 'off'}"] = {
                "layers": n_layers, "tokens_per_input": n_tokens, "weights": n_layers * n_w,
                "device_s": dev_ms / 1e3, "wall_s": wall_s,
                "layers_per_s": n_layers / (dev_ms / 1e3),
                "weights_per_s": n_layers * n_w / (dev_ms / 1e3),
                "launches": gptq.launch_count() - launches0,
                "mean_loss": {k: float(np.mean(v)) for k, v in losses.items()},
                "stages": st}
            del outs
    finally:
        gptq.profile_enable(False)
        del hs, ws
        torch.cuda.empty_cache()
    return res


def run_ours(args):
    world, rank, local = dist_env()
    distributed = init_dist(world, local)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    from post_weight_quantization_24_b200 import gptq
    gptq.lib()
    peaks = load_peaks()

    # each rank quantizes its own layer (different seed): independent units, no collective
    wl = rank_workload(args.workload, rank)
    step = LayerStep(gptq, wl, device)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)   # > L2 (126 MB)

    gptq.profile_enable(False)   # no stage events inside the timed steps
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    stage_tot = {k: 0.0 for k in ("hessian", "gptq", "rtn")}
    lib_stage_tot = {k: 0.0 for k in gptq.STAGES}
    total_ms = 0.0
    barrier(distributed)
    torch.cuda.synchronize()
    sampler.start()
    t_mark0 = sampler.mark()
    launches0 = gptq.launch_count()
    t_wall0 = time.perf_counter()
    for _ in range(args.steps):
        flush.zero_()                                   # L2 flush, outside the timed events
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        step.run(timed=True)
        t1.record()
        torch.cuda.synchronize()
        total_ms += t0.elapsed_time(t1)
        for k, v in step.stage_ms().items():
            stage_tot[k] += v
    torch.cuda.synchronize()
    wall_s = time.perf_counter() - t_wall0
    launches = gptq.launch_count() - launches0
    clocks = sampler.stop(t_mark0, sampler.mark())
    barrier(distributed)
    # the library's per-stage breakdown, from as many further steps with its stage events on
    gptq.profile_enable(True)
    for _ in range(args.steps):
        flush.zero_()
        step.run()
        torch.cuda.synchronize()
        for k, v in gptq.profile_read().items():
            lib_stage_tot[k] += v
    gptq.profile_enable(False)
    K = args.steps
    total_ms_max = max_over_ranks(total_ms, distributed, device)
    ms_per_step = total_ms_max / K
    weights_per_step = wl.d_out * wl.d_in
    value = job_value(world, K, weights_per_step, total_ms_max)

    hess_ms = stage_tot["hessian"] / K
    rtn_ms = stage_tot["rtn"] / K
    lib_ms = {k: v / K for k, v in lib_stage_tot.items()}
    d, n, d_out = wl.d_in, wl.n_tokens, wl.d_out

    # ---- per-stage roofline ----
    clock_mhz = (clocks or {}).get("sm_mhz") or peaks.get("clocks_under_load", {}).get("sm_mhz_median", 1312.0)
    pk = peaks_for(peaks, clock_mhz)
    tc_peak = pk["tensor"]
    hess_flops = float(n) * d * (d + 1)                  # symmetric 2·XᵀX
    hess_tf = hess_flops / (hess_ms / 1e3) / 1e12
    w_f16 = wl.w_dtype == "f16"
    stages = gptq_stage_table(hess_flops, hess_ms, lib_ms, gptq_flops(d_out, d, wl.block_size, w_f16),
                              pk, clock_mhz, w_f16, n, d)
    rtn_bytes = d_out * d * (2 + (0.5 if wl.bits == 4 else 1.0)) + d_out * (d // wl.group_size) * 4
    stages["rtn"] = {"ms": rtn_ms, "bound": "hbm", "gbs": rtn_bytes / (rtn_ms / 1e3) / 1e9,
                     "frac": rtn_bytes / (rtn_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "note": "one call on this layer's W (90 MB, inside L2) right after a "
                             "synchronising call: includes the host submission gap; see "
                             "rtn_7b_stack"}

    # ---- outside the timed steps (1 GPU only): RTN over a 7B stack, every config, the stack ----
    extras = world == 1
    rtn_stack = None if (args.no_rtn_stack or not extras) else rtn_stack_measure(gptq, device)
    if rtn_stack is not None:
        stages["rtn_7b_stack"] = dict(rtn_stack, bound="hbm",
                                      frac=rtn_stack["gbs"] / peaks["hbm_gbs"],
                                      note="INT4 g128 RTN over a 7B decoder stack's 224 matrices "
                                           "(6.48e9 fp16 weights), outside the timed step")
    configs = None
    if extras and not args.no_configs:
        configs = configs_measure(gptq, device, flush, peaks, clock_mhz)
    more = {}
    if extras and not args.no_configs:
        for key, fn in (("w4a16", lambda: w4a16_measure(gptq, device, peaks)),
                        ("sequential_mlp_7b", lambda: sequential_measure(gptq, device, peaks)),
                        ("awq_clip", lambda: awq_clip_measure(gptq, device, peaks))):
            try:
                more[key] = fn()
            except Exception as exc:                  # reported in the line, never fatal
                more[key] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
                torch.cuda.empty_cache()
    stack = None
    if extras and not args.no_stack:
        try:
            stack = stack_measure(gptq, device, peaks, clock_mhz, n_layers=args.stack_layers)
        except Exception as exc:                      # reported in the line, never fatal
            stack = {"error": f"{type(exc).__name__}: {exc}"[:300]}
            torch.cuda.empty_cache()

    # the dominant kernel (largest stage) carries the roofline object
    traffic, _ = ncu_traffic("hessian_pair_kernel_mlp_up_7b.md", "hessian.cu")
    roof = {"kernel": "hessian_pair_kernel", "bound": "tensor", "achieved": hess_tf,
            "peak": tc_peak, "unit": "TFLOP/s", "frac": hess_tf / tc_peak,
            "traffic": traffic,
            "peak_note": "measured bf16 dense burst (fp16 MMA runs at the bf16 rate); of measured"
            if peaks["source"] == "measured" else "fallback"}
    # (the 7B-stack RTN measurement runs outside the step and does not compete)
    dom = max((k for k in stages if k != "rtn_7b_stack"
               and ("frac" in stages[k] or k == "hessian")),
              key=lambda k: stages[k]["ms"])
    if dom != "hessian":
        roof = {"kernel": dom, "bound": stages[dom]["bound"],
                "achieved": stages[dom].get("tflops", stages[dom].get("gbs")),
                "peak": stages[dom].get("peak_tflops", peaks["hbm_gbs"]),
                "unit": "TFLOP/s" if "tflops" in stages[dom] else "GB/s",
                "frac": stages[dom]["frac"], "traffic": None,
                "peak_note": stages[dom].get("peak_note", "")}

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(step, gptq, args, distributed, device, world)

    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": workload_config(wl),
        "arithmetic": "Hessian and loss Gram matrix fp16 x fp16 -> fp32 on tcgen05; "
                      "factorisation and lazy update fp32 as 3xTF32 on tcgen05; "
                      "column loop fp32 FFMA; group scalars fp64",
        "calib_tokens_per_s": world * n / (hess_ms / 1e3),
        "layer_loss": step.loss,
        "stages": stages,
        "configs": configs,
        "stack_7b": stack,
        "next_rows": more or None,
        "roofline": roof,
        "clocks": clocks,
        "gpu_launches": launches,
        "wall_s_timed": wall_s,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(step, wl)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if distributed:
        import torch.distributed as dist
        dist.destroy_process_group()


def workload_config(wl):
    """The `config` object of both arms' lines: the same workload, named the same way."""
    d_out, d, n = wl.d_out, wl.d_in, wl.n_tokens
    return {"workload": f"{wl.name}: W {d_out}x{d} {wl.w_dtype}, X {n}x{d} fp16 "
                        f"(lognormal channel scales, outliers), INT{wl.bits} g{wl.group_size} "
                        f"B{wl.block_size} percdamp {wl.percdamp} act_order {wl.act_order}",
            "per_rank": "one independent layer per GPU (seed = rank)",
            "l2": f"X ({n * d * 2 / 1e9:.1f} GB) larger than L2, plus a 512 MB L2 flush "
                  f"between steps"}


def run_e2e(step, gptq, args, distributed, device, world):
    """Same step, with the inputs copied in from pinned host memory and the results copied
    back inside the timed region."""
    wl = step.wl
    X_h = step.X.cpu().pin_memory()
    W_h = step.W.cpu().pin_memory()
    outs_h = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in step.out.items()}
    rtn_h = tuple(torch.empty_like(t, device="cpu").pin_memory() for t in step.rtn_out)
    h2d = X_h.numel() * X_h.element_size() + W_h.numel() * W_h.element_size()
    d2h = sum(t.numel() * t.element_size() for t in outs_h.values()) + \
        sum(t.numel() * t.element_size() for t in rtn_h) + 4   # + the loss (float)

    def one():
        step.X.copy_(X_h, non_blocking=True)
        step.W.copy_(W_h, non_blocking=True)
        step.run()
        for k, t in step.out.items():
            outs_h[k].copy_(t, non_blocking=True)
        for hst, dev in zip(rtn_h, step.rtn_out):
            hst.copy_(dev, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    barrier(distributed)
    total = 0.0
    K = max(1, min(args.steps, 10))
    for _ in range(K):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        one()
        b.record()
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
    total = max_over_ranks(total, distributed, device)
    return {"value": world * K * wl.d_out * wl.d_in / (total / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": total / K, "steps": K}


# ------------------------------------------------------------------------------------------
# CPU checker timings (the fp64 oracle as it stands, on a bounded sample)
# ------------------------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def oracle_sample(W_np, X_np, wl, n_tok, n_rows, n_rtn_rows, seed=0):
    """Time the oracle's stages on a sample; return (extrapolated full-step seconds, detail)."""
    from oracle import gptq as ogptq
    from oracle import hessian as ohess
    from oracle import loss as oloss
    from oracle import rtn as ortn
    rng = np.random.default_rng(seed)
    d, d_out, n = wl.d_in, wl.d_out, wl.n_tokens
    t = time.perf_counter()
    Hs = ohess.hessian(X_np[:n_tok])
    t_h = time.perf_counter() - t
    t = time.perf_counter()
    perm, U = ogptq.prepare_u(Hs, wl.percdamp, wl.act_order)
    t_u = time.perf_counter() - t
    rows = np.sort(rng.choice(d_out, n_rows, replace=False))
    Wn = W_np.astype(np.float64)
    t = time.perf_counter()
    out = ogptq.gptq_blocked_ref(Wn, Hs, wl.bits, wl.group_size, wl.block_size, wl.percdamp,
                                 wl.act_order, rows=rows, U=U)
    t_g = time.perf_counter() - t
    t = time.perf_counter()
    oloss.recon_loss(Wn[rows], out["What"], Hs)
    t_l = time.perf_counter() - t
    t = time.perf_counter()
    ortn.rtn_minmax(Wn[:n_rtn_rows], wl.bits, wl.group_size)
    t_r = time.perf_counter() - t
    full = (t_h * n / n_tok + t_u + (t_g + t_l) * d_out / n_rows + t_r * d_out / n_rtn_rows)
    measured = t_h + t_u + t_g + t_l + t_r
    detail = (f"oracle fp64 on a sample: Hessian over {n_tok} of {n} tokens (x{n / n_tok:.0f}), "
              f"U for the full d={d}, GPTQ + loss on {n_rows} of {d_out} rows "
              f"(x{d_out / n_rows:.1f}), RTN on {n_rtn_rows} rows (x{d_out / n_rtn_rows:.1f}); "
              f"sample took {measured:.1f} s, extrapolated full step {full:.1f} s")
    return full, measured, detail


# One oracle sample definition for both the cpu_baseline leg and the reference arm: the
# Hessian over the first 4096 tokens, the full factorisation (d_in = 4096), GPTQ and the loss
# on 64 rows, RTN on 1024 rows; each part is then scaled to the full layer.
SAMPLE = dict(n_tok=4096, n_rows=64, n_rtn_rows=1024)
THREAD_NOTE = ("numpy/LAPACK with its BLAS threads for the matrix products and factorisation; "
               "the oracle's column loop itself is a Python loop of numpy vector steps on one "
               "thread")


def cpu_baseline(step, wl):
    X_np = step.X[:SAMPLE["n_tok"]].cpu().numpy()
    W_np = step.W.float().cpu().numpy()
    full, measured, detail = oracle_sample(W_np, X_np, wl, **SAMPLE)
    return {"value": wl.d_out * wl.d_in / full, "unit": UNIT, "cores": _blas_threads(),
            "kind": "oracle", "sample": detail + "; " + THREAD_NOTE}


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return
    wl = workloads.WORKLOADS[args.workload]
    # the same generator recipe on the CPU (bounded: only what the sample touches)
    W = workloads.make_weights(wl, device="cpu").float().numpy()
    X = workloads.make_activations(wl, device="cpu", n_tokens=SAMPLE["n_tok"]).numpy()
    fulls, measured = [], 0.0
    for i in range(args.warmup + args.steps):
        full, m, detail = oracle_sample(W, X, wl, seed=i, **SAMPLE)
        if i >= args.warmup:
            fulls.append(full)
            measured += m
    full = statistics.mean(fulls)
    value = wl.d_out * wl.d_in / full
    cores = _blas_threads()
    res = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": full * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "impl": "reference",
           "config": workload_config(wl),
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                            "sample": detail + f"; {args.steps} timed samples; " + THREAD_NOTE},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def run_ncu_case(name: str):
    """Small invocations for ncu captures (inputs larger than L2, a few GB at most): the
    profile summaries under profiles/ name these commands."""
    from post_weight_quantization_24_b200 import gptq
    torch.cuda.set_device(0)
    wl = workloads.WORKLOADS["mlp_up_7b"]
    if name == "hessian":                        # X 16384 x 4096 fp16 = 134 MB; 3 launches
        X = workloads.make_activations(wl.replace(n_tokens=16384), device="cuda")
        h = gptq.Hessian(wl.d_in)
        for _ in range(3):
            h.accumulate(X)
    elif name == "gptq":                         # the timed layer's quantizer, 2 calls
        X = workloads.make_activations(wl.replace(n_tokens=8192), device="cuda")
        W = workloads.make_weights(wl, device="cuda")
        h = gptq.Hessian(wl.d_in)
        h.accumulate(X)
        ws = torch.empty(gptq.quantize_layer_workspace(wl.d_out, wl.d_in), dtype=torch.uint8,
                         device="cuda")
        for _ in range(2):
            gptq.quantize_layer(W, h.raw(), compute_loss=True, workspace=ws)
    elif name == "rtn":                          # W 11008 x 4096 fp16; 3 launches
        W = workloads.make_weights(wl, device="cuda")
        for _ in range(3):
            gptq.rtn_minmax_quantize(W, 4, 128)
    elif name == "w4a16":                        # X 16384 x 4096, W 22016 x 4096 INT4; 3 launches
        W = workloads.make_weights(wl.replace(d_out=22016), device="cuda")
        packed, scales, zeros = gptq.rtn_minmax_quantize(W, 4, 128)
        X = workloads.make_activations(wl.replace(n_tokens=16384), device="cuda")
        Y = torch.empty(16384, 22016, dtype=torch.float16, device="cuda")
        for _ in range(3):
            gptq.w4a16_linear(X, packed, scales, zeros, 128, out=Y)
    elif name == "factor":                       # d = 11008 (mlp_down_7b's H), 2 calls
        wd = workloads.WORKLOADS["mlp_down_7b"]
        X = workloads.make_activations(wd.replace(n_tokens=4096), device="cuda")
        h = gptq.Hessian(wd.d_in)
        h.accumulate(X)
        for _ in range(2):
            gptq.inverse_factor(h.raw(), act_order=True)
    elif name == "rtn_big":                      # 4 layers of 7B weights: 153600 x 4096 fp16
        W = workloads.make_weights(wl.replace(d_out=4 * (4 * 4096 + 2 * 11008)), device="cuda")
        for _ in range(3):                       # (1.26 GB, ten times L2)
            gptq.rtn_minmax_quantize(W, 4, 128)
    else:
        raise SystemExit(f"unknown ncu case {name}")
    torch.cuda.synchronize()
    print("ncu case done:", name)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="mlp_up_7b", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rtn-stack", action="store_true",
                    help="skip the RTN measurement over a 7B decoder stack (13 GB of weights)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the timed lines of the other layer workloads")
    ap.add_argument("--no-stack", action="store_true",
                    help="skip GPTQ over a full 7B decoder stack (4 variants)")
    ap.add_argument("--stack-layers", type=int, default=32)
    ap.add_argument("--ncu-case", choices=("hessian", "gptq", "rtn", "rtn_big", "w4a16", "factor"),
                    help="run one small case for an ncu capture and exit (no JSON line)")
    args = ap.parse_args(argv)
    if args.ncu_case:
        run_ncu_case(args.ncu_case)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
