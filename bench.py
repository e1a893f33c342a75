#!/usr/bin/env python
"""Benchmark of the QLoRA adapted linear layer (libqlora, B200).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward + backward pass of the adapted linear layer(s) of the
workload over one batch of M tokens: dequantisation of the frozen NF4 weight
inside the GEMMs, V = X A, Y, U = dY B^T, dX, dA, dB.  Quantisation and merge
are one-time operations of the method ("How it works" steps 1 and 5) and are
timed separately under "rows", with the small-M forward, the training step with
the fused Adam update, and the INT (one scale per 16 weights) base quantiser.
The Llama-7B stack workload (--workload llama7b_stack_m2048_r16) runs all 224
linears of the model per step and times the quantise pass over all of them.

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
synchronize on both sides, CUDA events on the launching stream, max over ranks.
Inputs rotate over several independent sets whose combined size exceeds the L2
cache, so every step reads its operands from HBM.  One JSON line on rank 0.

With --gpus N > 1 (launched by torch.distributed.run) every rank runs an
independent replica on its own GPU (the layer's data-parallel split has no
exchange in the forward; weak scaling), and the value is all ranks' tokens over
the slowest rank's time.

--impl reference times the float64 CPU oracle (the reference arm) on a bounded
sample of the same workload on the host cores.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# one Llama-7B decoder layer's projections, in order: q, k, v and o take 4096
# inputs; gate and up expand to 11008; down projects back.  q, k and v read the
# same input activations, as do gate and up (the model feeds them one tensor).
LLAMA7B_LAYER = (("q", 4096, 4096, "attn_in"), ("k", 4096, 4096, "attn_in"), ("v", 4096, 4096, "attn_in"),
                 ("o", 4096, 4096, "o_in"), ("gate", 4096, 11008, "mlp_in"), ("up", 4096, 11008, "mlp_in"),
                 ("down", 11008, 4096, "down_in"))

WORKLOADS = {
    # Llama-7B attention projection (the headline configuration)
    "attn4096_m4096_r16": dict(shapes=[(4096, 4096)], M=4096, r=16),
    # Llama-7B MLP projections, one gate/up and one down per step
    "mlp4096x11008_m8192_r64": dict(shapes=[(4096, 11008), (11008, 4096)], M=8192, r=64),
    # the smallest configuration (launch-bound)
    "linear256_m64_r8": dict(shapes=[(256, 256)], M=64, r=8),
    # the whole Llama-7B linear stack: 32 layers x 7 projections, 6.48e9 weights
    # quantised on the device, r = 16 on every linear; one step is the forward
    # and backward of all 224 linears
    "llama7b_stack_m2048_r16": dict(shapes=[(a, b) for _, a, b, _ in LLAMA7B_LAYER] * 32, M=2048, r=16,
                                    layer=LLAMA7B_LAYER, layers=32, steps=20, warmup=3),
}
DEFAULT_WORKLOAD = "llama7b_stack_m2048_r16"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures, reported beside the measured ones: dense bf16 tensor
# throughput and HBM3e bandwidth
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None, help="timed steps (default: 2000; 20 for the stack)")
    p.add_argument("--warmup", type=int, default=None, help="warm-up steps (default: 10; 3 for the stack)")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-rows", action="store_true", help="skip the per-kernel row measurements")
    p.add_argument("--rows", default=None,
                   help="comma-separated subset of the rows: quantize, dequantize, merge, gemv, train_step, int16 "
                        "(default: all of them; none for the stack, whose quantize pass is always measured)")
    p.add_argument("--rows-only", action="store_true",
                   help="measure only the rows (no headline step); prints {'rows': ...}")
    p.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    a = p.parse_args()
    wl = WORKLOADS[a.workload]
    if a.steps is None:
        a.steps = wl.get("steps", 2000)
    if a.warmup is None:
        a.warmup = wl.get("warmup", 10)
    if a.rows is None:
        a.rows = "all"
    return a


def workload_config(name):
    wl = WORKLOADS[name]
    c = {"workload": name, "M": wl["M"], "r": wl["r"]}
    if "layer" in wl:
        c.update(layers=wl["layers"], layer=[f"{n} {a}x{b}" for n, a, b, _ in wl["layer"]])
    else:
        c["shapes"] = wl["shapes"]
    return c


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gemm_peak(pk, timed_s, reasons):
    """The bf16 peak the headline's fused GEMM is measured against: the sustained
    figure (a seconds-long cuBLAS loop under the power cap) for a kernel timed
    inside a long step, that is a timed region of 2 s or more or one whose clock
    record shows the power cap holding the SM clock down; the burst figure
    otherwise.  Returns (peak TFLOP/s, sustained?, power-capped?)."""
    power_capped = "sw_power_cap" in (reasons or [])
    sustained = timed_s >= 2.0 or power_capped
    return (pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]), sustained, power_capped


def flops_fwd_bwd(n_in, n_out, M, r):
    """Algorithmic flops of one forward + backward: 4 M in out + 6 M r (in + out)."""
    return 4 * M * n_in * n_out + 6 * M * r * (n_in + n_out)


def flops_fwd_gemm(n_in, n_out, M, r):
    """The fused forward GEMM: X W (2 M in out) plus V B (2 M r out)."""
    return 2 * M * n_out * (n_in + r)


# the fused GEMM's source and every header it includes: traffic counters taken
# from an ncu capture stay valid only while these are unchanged
GEMM_SOURCES = ("gemm.cu", "sm100.cuh", "common.cuh")


def code_tokens(text: str) -> str:
    """C/C++/CUDA source with its comments removed and whitespace collapsed: what
    the compiler sees, so that a comment edit does not count as a kernel change."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":                          # string or character literal, kept whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def src_hash(*names):
    """Hash of the code (comments and whitespace aside) of the GEMM's sources."""
    h = hashlib.sha1()
    for n in names:
        with open(os.path.join(ROOT, "quantized_rank_fine_b200", "csrc", n), encoding="utf-8") as f:
            h.update(code_tokens(f.read()).encode())
    return h.hexdigest()[:12]


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled every ~2 ms by a thread
    polling NVML (read-only queries) while the timed region runs; `nvidia-smi`
    every 100 ms when NVML cannot be loaded.  A median needs samples inside the
    region, which for a short region only an in-process poll provides."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.002

    def __init__(self, index, uuid=None, pci_bus_id=None):
        self.index = index          # nvidia-smi index (fallback path)
        self.uuid = uuid            # CUDA device UUID, for NVML
        self.pci_bus_id = pci_bus_id
        self.proc = None
        self.thread = None
        self.samples = []           # (sm_mhz, reasons bitmask)
        self.sm_max = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        for how, key in ((pynvml.nvmlDeviceGetHandleByUUID, self.uuid),
                         (pynvml.nvmlDeviceGetHandleByPciBusId, self.pci_bus_id)):
            if key:
                try:
                    return pynvml, how(key)
                except Exception:
                    pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(self.index))

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            nv = None
        if nv is None:
            self.source = "nvidia-smi"
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None
            return
        self.source = "nvml"
        self._stop = threading.Event()

        def poll():
            while not self._stop.is_set():
                try:
                    self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                         int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
                except Exception:
                    pass
                time.sleep(self.PERIOD_S)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()

    def stop(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        if self.thread is not None:
            import pynvml as nv
            self._stop.set()
            self.thread.join(timeout=5)
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            sm = [s for s, _ in self.samples]
            reasons = sorted(n for n in names if any(r & bits[n] for _, r in self.samples))
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.sm_max,
                    "reasons": reasons, "samples": len(sm), "source": "nvml, 2 ms poll"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, 100 ms"}


def clock_sampler(local):
    """The sampler for this rank's GPU (NVML by the CUDA device's UUID)."""
    import torch
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    smi_id = vis.split(",")[local] if vis and len(vis.split(",")) > local else str(local)
    uuid = pci = None
    try:
        p = torch.cuda.get_device_properties(local)
        u = str(p.uuid)
        uuid = u if u.startswith("GPU-") else "GPU-" + u
        pci = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        pass
    return ClockSampler(smi_id, uuid, pci)


# ------------------------------------------------------------------ distributed plumbing

def dist_init(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value of x over all ranks (identity with one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ our arm

def build_sets(wl, nsets, seed_base):
    import torch
    import quantized_rank_fine_b200 as q
    import synth
    M, r = wl["M"], wl["r"]
    sets = []
    for s in range(nsets):
        layers = []
        for li, (n_in, n_out) in enumerate(wl["shapes"]):
            t = synth.layer_inputs(n_in, n_out, M, r, device="cuda", seed=seed_base + s, tag=f"bench{li}:")
            w = q.qlora_quantize_nf4(t["W0"])
            del t["W0"]
            out = {
                "Y": torch.empty((M, n_out), dtype=torch.bfloat16, device="cuda"),
                "V": torch.empty((M, r), dtype=torch.bfloat16, device="cuda"),
                "dX": torch.empty((M, n_in), dtype=torch.bfloat16, device="cuda"),
                "dA": torch.empty((n_in, r), dtype=torch.float32, device="cuda"),
                "dB": torch.empty((r, n_out), dtype=torch.float32, device="cuda"),
            }
            layers.append((w, t, out))
        sets.append(layers)
    torch.cuda.synchronize()
    return sets


def stack_weight(li, name, n_in, n_out, seed, device="cuda"):
    """W0 of projection `name` of layer li of the stack (fp32 0.02 N(0, 1))."""
    import torch
    import synth
    return synth.normal(f"stack{li}.{name}:W0", (n_in, n_out), 0.02, torch.float32, device, seed)


def stack_linear(li, name, n_in, n_out, x_key, M, r, seed, acts, device="cuda"):
    """W0 and the inputs of one linear of the stack, drawn on the device: its own
    adapters A, B and output gradient dY, and the input X of its key, drawn once
    per layer and key (`acts` holds the layer's drawn inputs)."""
    import torch
    import synth
    p = f"stack{li}.{name}:"
    W0 = stack_weight(li, name, n_in, n_out, seed, device)
    if x_key not in acts:
        acts[x_key] = synth.normal(f"stack{li}.{x_key}:X", (M, n_in), 1.0, torch.bfloat16, device, seed)
    t = {"X": acts[x_key],
         "A": synth.normal(p + "A", (n_in, r), 1.0 / math.sqrt(n_in), torch.bfloat16, device, seed),
         "B": synth.normal(p + "B", (r, n_out), 0.01, torch.bfloat16, device, seed),
         "dY": synth.normal(p + "dY", (M, n_out), 1.0, torch.bfloat16, device, seed)}
    return W0, t


def build_stack(wl, seed, pk):
    """The Llama-7B linear stack as one input set, and its quantize pass.

    Every linear gets its own W0, adapters and output gradient dY; q, k and v
    share one input X, gate and up another.  All 224 W0 (fp32, 26 GB) are drawn
    on the device first; the quantize pass quantises each into its NF4 weight,
    once to build the weights and then timed with CUDA events (identical
    results), each pass captured in a CUDA graph and replayed twice: through the
    batch call (qlora_quantize_nf4_batch, 32 weights per launch) and one call per
    weight, after which the W0 are freed."""
    import torch
    import quantized_rank_fine_b200 as q
    import synth
    M, r = wl["M"], wl["r"]
    W0s, plan = [], []
    for li in range(wl["layers"]):
        acts = {}
        for name, n_in, n_out, x_key in wl["layer"]:
            W0, t = stack_linear(li, name, n_in, n_out, x_key, M, r, seed, acts)
            W0s.append(W0)
            out = {
                "Y": torch.empty((M, n_out), dtype=torch.bfloat16, device="cuda"),
                "V": torch.empty((M, r), dtype=torch.bfloat16, device="cuda"),
                "dX": torch.empty((M, n_in), dtype=torch.bfloat16, device="cuda"),
                "dA": torch.empty((n_in, r), dtype=torch.float32, device="cuda"),
                "dB": torch.empty((r, n_out), dtype=torch.float32, device="cuda"),
            }
            plan.append((t, out))
    weights = q.qlora_quantize_nf4_batch(W0s)
    torch.cuda.synchronize()

    def timed_pass(fn):
        # the pass captured in a CUDA graph, as the other rows: device time only
        # (the host's argument checks and launches are not timed)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side, capture_error_mode="relaxed"):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        times = []
        for _ in range(2):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        del graph
        return min(times)

    def one_by_one():
        for W, w in zip(W0s, weights):
            q.qlora_quantize_nf4(W, out=w)

    ms = timed_pass(lambda: q.qlora_quantize_nf4_batch(W0s, outs=weights))
    ms_single = timed_pass(one_by_one)
    n = sum(W.numel() for W in W0s)
    del W0s
    torch.cuda.empty_cache()
    b = sum(a * o * (4 + 0.5 + 1 / 64) + 4 * math.ceil(a * o / 64 / 256) for a, o in wl["shapes"])
    single = hbm_fracs(b, ms_single, pk)
    row = {"ms": ms, "weights": n, "launches": math.ceil(len(weights) / 32), **hbm_fracs(b, ms, pk),
           "one_call_per_weight": {"ms": ms_single, "launches": len(weights), "gbs": single["gbs"],
                                   "frac_hbm": single["frac_hbm"]},
           "note": "all 224 W0 of the stack quantised (fp32 in, NF4 codes + absmax codes + scales out) by "
                   "the batch call, 32 weights per launch; the better of two replays of the pass captured "
                   "in a CUDA graph"}
    layers = [(w, t, o) for w, (t, o) in zip(weights, plan)]
    return [layers], row


def set_bytes(wl):
    """HBM bytes one step of one input set touches at least: NF4 weights, the
    adapters and their gradients, and the activations (X and dY read, Y and dX
    written), each distinct activation tensor counted once."""
    M, r = wl["M"], wl["r"]
    tot = 0
    for n_in, n_out in wl["shapes"]:
        n = n_in * n_out
        tot += n // 2 + n // 64 + 2 * r * (n_in + n_out) + 4 * r * (n_in + n_out)
        tot += 2 * M * (2 * n_out + n_in)          # dY read, Y written, dX written
        tot += 2 * M * n_in                        # X read (the stack shares some; below)
    if "layer" in wl:
        x_width = {key: n_in for _, n_in, _, key in wl["layer"]}      # one X per key
        counted = sum(n_in for _, n_in, _, _ in wl["layer"])
        tot -= 2 * M * (counted - sum(x_width.values())) * wl["layers"]
    return tot


def run_step(layers, ws):
    import quantized_rank_fine_b200 as q
    for w, t, o in layers:
        q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, Y=o["Y"], V=o["V"])
        q.qlora_linear_bwd(w, t["X"], o["V"], t["dY"], t["A"], t["B"], ws, dX=o["dX"], dA=o["dA"], dB=o["dB"])


ROW_NAMES = ("quantize", "dequantize", "merge", "gemv", "train_step", "int16", "mlp_m8192", "dense")


def time_rows(wl, pk, which="all"):
    """Per-kernel measurements of the other rows of the path (one GPU); `which`
    is "all" or a comma-separated subset of ROW_NAMES."""
    if not which:
        return {}
    want = set(ROW_NAMES) if which == "all" else set(which.split(","))
    unknown = want - set(ROW_NAMES)
    if unknown:
        raise SystemExit(f"unknown rows: {sorted(unknown)}")
    rows = {}
    if want & {"quantize", "dequantize", "merge"}:
        rows.update(time_weight_rows(wl, pk, want))
    if "gemv" in want:
        rows["gemv"] = time_gemv(pk)
    if "train_step" in want:
        # the stack's layers are too many for graph-captured sets: its training-step
        # row runs the attention projection (4096 x 4096, r = 16, M = 4096)
        rows["train_step_adam"] = time_train_step(WORKLOADS["attn4096_m4096_r16"] if "layer" in wl else wl)
    if "mlp_m8192" in want:
        rows["mlp_m8192"] = time_mlp_row(pk)
    if "int16" in want:
        try:
            rows["int16"] = time_int16_rows(wl, pk)
        except Exception as e:   # a secondary row never takes the headline down
            rows["int16"] = {"error": f"{type(e).__name__}: {e}"}
    if "dense" in want:
        try:
            rows["dense_context"] = time_dense_context(pk)
        except Exception as e:   # context only: never takes the headline down
            rows["dense_context"] = {"error": f"{type(e).__name__}: {e}"}
    return rows


def time_dense_context(pk):
    """Context, not the product: the unfused alternative to the fused forward.
    cuBLAS (torch.matmul, bf16) on the dequantised bf16 weight, and the same after
    qlora_dequantize each call, beside this library's forward (V = X A and the
    fused dequant GEMM) on the same weights, at the attention projection (M = 4096,
    r = 16) and the MLP projections (M = 8192, r = 64).  Device time per call of a
    CUDA graph of back-to-back calls over weights rotated past L2; TFLOP/s count
    2 M in out (the base product)."""
    import torch
    import quantized_rank_fine_b200 as q
    import synth
    out = {}
    iters = 20
    for n_in, n_out, M, r in ((4096, 4096, 4096, 16), (4096, 11008, 8192, 64), (11008, 4096, 8192, 64)):
        reps = max(3, math.ceil(3 * L2_BYTES / (n_in * n_out * 2)))
        wts = [q.qlora_quantize_nf4(synth.normal(f"denseW{i}", (n_in, n_out), 0.02, device="cuda"))
               for i in range(reps)]
        Ws = [q.qlora_dequantize(w, torch.bfloat16) for w in wts]
        X = synth.normal(f"denseX{M}", (M, n_in), 1.0, torch.bfloat16, "cuda")
        A = synth.normal("denseA", (n_in, r), 1 / math.sqrt(n_in), torch.bfloat16, "cuda")
        B = synth.normal("denseB", (r, n_out), 0.01, torch.bfloat16, "cuda")
        Y = torch.empty((M, n_out), dtype=torch.bfloat16, device="cuda")
        V = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
        ws = q.Workspace()
        torch.cuda.synchronize()

        def cublas(i):
            torch.matmul(X, Ws[i % reps], out=Y)

        def dequant_cublas(i):
            q.qlora_dequantize(wts[i % reps], torch.bfloat16, out=Ws[i % reps])
            torch.matmul(X, Ws[i % reps], out=Y)

        def fused(i):
            q.qlora_linear_fwd(wts[i % reps], X, A, B, ws, Y=Y, V=V)

        flops = 2.0 * M * n_in * n_out
        row = {}
        for name, fn in (("cublas_on_dequantised_bf16", cublas), ("dequantize_then_cublas", dequant_cublas),
                         ("libqlora_forward", fused)):
            t = graph_per_call(fn, iters)
            row[name] = {"ms": t, **tensor_fracs(flops, t, pk)}
        if ws.status() != 0:
            raise RuntimeError("a kernel wait timed out in the dense-context row")
        out[f"{n_in}x{n_out}_m{M}_r{r}"] = row
        del wts, Ws, X, Y, V, ws
        torch.cuda.synchronize()
    out["note"] = ("context only: cuBLAS through torch.matmul, not part of the path; TFLOP/s of the base "
                   "product 2 M in out")
    return out


def weight_row_shape(wl):
    """Weight shape of the quantize / dequantize / merge rows: the workload's first
    shape, or 4096 x 11008 (the largest matrix of a layer) for the stack."""
    return (4096, 11008) if "layer" in wl else wl["shapes"][0]


def hbm_fracs(b, ms, pk):
    """GB/s of b algorithmic bytes in ms, as fractions of the measured and the
    datasheet HBM bandwidth."""
    gbs = b / ms / 1e6
    return {"gbs": gbs, "frac_hbm": gbs / pk["hbm_gbs"], "frac_hbm_spec": gbs / SPEC_HBM_GBS}


def time_weight_rows(wl, pk, want):
    """Quantize, dequantize and merge on one weight (weight_row_shape)."""
    import torch
    import quantized_rank_fine_b200 as q
    import synth
    rows = {}
    n_in, n_out = weight_row_shape(wl)
    n = n_in * n_out
    reps = max(3, math.ceil(3 * L2_BYTES / (4 * n)))
    W0s = [synth.normal(f"rowsW{i}", (n_in, n_out), 0.02, device="cuda") for i in range(reps)]
    ws_ = [q.qlora_quantize_nf4(W) for W in W0s]
    torch.cuda.synchronize()

    def timed(fn, which, iters):
        return graph_timed(fn, which, iters)

    iters = 30
    if "quantize" in want:
        qf = lambda i: q.qlora_quantize_nf4(W0s[i % reps], out=ws_[i % reps])
        t = timed(qf, q.KERNEL_QUANTIZE, iters)
        b = n * (4 + 0.5 + 1 / 64) + 4 * math.ceil(n / 64 / 256)
        tb = graph_per_call(qf, iters)
        bb = hbm_fracs(b, tb, pk)
        rows["quantize"] = {"shape": [n_in, n_out], "ms": t, **hbm_fracs(b, t, pk), "bytes_per_weight": 4.516,
                            "back_to_back": {"ms_per_call": tb, "gbs": bb["gbs"], "frac_hbm": bb["frac_hbm"],
                                             "note": "graph of back-to-back quantisations of the rotating "
                                                     "weights, device time per call"}}
    if "dequantize" in want:
        outs = [torch.empty((n_in, n_out), dtype=torch.bfloat16, device="cuda") for _ in range(reps)]
        df = lambda i: q.qlora_dequantize(ws_[i % reps], torch.bfloat16, out=outs[i % reps])
        t = timed(df, q.KERNEL_DEQUANTIZE, iters)
        b = n * (0.5 + 1 / 64 + 2) + 4 * math.ceil(n / 64 / 256)
        tb = graph_per_call(df, iters)
        bb = hbm_fracs(b, tb, pk)
        rows["dequantize_bf16"] = {"shape": [n_in, n_out], "ms": t, **hbm_fracs(b, t, pk),
                                   "back_to_back": {"ms_per_call": tb, "gbs": bb["gbs"], "frac_hbm": bb["frac_hbm"]}}
        del outs
    if "merge" in want:
        r = wl["r"]
        A = synth.normal("rowsA", (n_in, r), 1 / math.sqrt(n_in), torch.bfloat16, "cuda")
        B = synth.normal("rowsB", (r, n_out), 0.01, torch.bfloat16, "cuda")
        outs32 = [torch.empty((n_in, n_out), dtype=torch.float32, device="cuda") for _ in range(reps)]
        mf = lambda i: q.qlora_merge(ws_[i % reps], A, B, torch.float32, out=outs32[i % reps])
        t = timed(mf, q.KERNEL_MERGE, iters)
        b = n * (0.5 + 1 / 64 + 4) + 2 * r * (n_in + n_out)
        tb = graph_per_call(mf, iters)
        bb = hbm_fracs(b, tb, pk)
        rows["merge_f32"] = {"shape": [n_in, n_out], "r": r, "ms": t, **hbm_fracs(b, t, pk),
                             "back_to_back": {"ms_per_call": tb, "gbs": bb["gbs"], "frac_hbm": bb["frac_hbm"]}}
        del outs32
    del W0s, ws_
    torch.cuda.synchronize()
    return rows


def time_int16_rows(wl, pk):
    """The INT base of the pages' simulation (qlora_quantize_int: symmetric
    integers, one fp32 scale per 16 weights), 4 bits, on the workload's first
    weight shape: quantize and dequantize (GB/s against HBM), and the fused
    forward GEMM on that weight at the workload's M (TFLOP/s), next to the NF4
    weight's forward GEMM measured the same way."""
    import torch
    import quantized_rank_fine_b200 as q
    import synth
    n_in, n_out = wl["shapes"][0]
    M, r = wl["M"], wl["r"]
    n = n_in * n_out
    reps = max(3, math.ceil(3 * L2_BYTES / (4 * n)))
    W0s = [synth.normal(f"intW{i}", (n_in, n_out), 0.02, device="cuda") for i in range(reps)]
    ints = [q.qlora_quantize_int(W, 4) for W in W0s]
    torch.cuda.synchronize()
    out = {"bits": 4, "shape": [n_in, n_out]}
    t = graph_timed(lambda i: q.qlora_quantize_int(W0s[i % reps], 4, out=ints[i % reps]), q.KERNEL_QUANTIZE, 30)
    b = n * (4 + 0.5 + 0.25)
    out["quantize"] = {"ms": t, **hbm_fracs(b, t, pk), "bytes_per_weight": 4.75}
    dq = [torch.empty((n_in, n_out), dtype=torch.bfloat16, device="cuda") for _ in range(reps)]
    t = graph_timed(lambda i: q.qlora_dequantize_int(*ints[i % reps], n_in, n_out, torch.bfloat16, out=dq[i % reps]),
                    q.KERNEL_DEQUANTIZE, 30)
    b = n * (0.5 + 0.25 + 2)
    out["dequantize_bf16"] = {"ms": t, **hbm_fracs(b, t, pk)}
    del dq
    # forward GEMM: INT16 weights against NF4 weights of the same W0, inputs rotated
    wts_int = [q.int_weight(c, s, n_in, n_out) for c, s in ints]
    wts_nf4 = [q.qlora_quantize_nf4(W) for W in W0s]
    del W0s
    X = [synth.normal(f"intX{i}", (M, n_in), 1.0, torch.bfloat16, "cuda") for i in range(2)]
    A = synth.normal("intA", (n_in, r), 1 / math.sqrt(n_in), torch.bfloat16, "cuda")
    B = synth.normal("intB", (r, n_out), 0.01, torch.bfloat16, "cuda")
    Y = torch.empty((M, n_out), dtype=torch.bfloat16, device="cuda")
    V = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    ws = q.Workspace()
    fl = flops_fwd_gemm(n_in, n_out, M, r)
    for name, wts in (("fwd_gemm_int16", wts_int), ("fwd_gemm_nf4", wts_nf4)):
        t = graph_timed(lambda i: q.qlora_linear_fwd(wts[i % reps], X[i % 2], A, B, ws, Y=Y, V=V),
                        q.KERNEL_FWD_GEMM, 20)
        out[name] = {"ms": t, "tflops": fl / t / 1e9}
    if ws.status() != 0:
        raise RuntimeError("a kernel wait timed out in the INT rows")
    del ints, wts_int, wts_nf4
    torch.cuda.synchronize()
    return out


def tensor_fracs(flops, ms, pk):
    """TFLOP/s of `flops` in ms, as fractions of the measured burst and sustained
    bf16 peaks and of the datasheet's dense bf16 peak."""
    tf = flops / ms / 1e9
    return {"tflops": tf, "frac_burst": tf / pk["bf16_tflops"], "frac_sustained": tf / pk["bf16_tflops_sustained"],
            "frac_spec": tf / SPEC_BF16_TFLOPS}


def time_mlp_row(pk):
    """The Llama-7B MLP projections (4096 -> 11008 and 11008 -> 4096, r = 64) at
    M = 8192 tokens, the size the fused GEMM's throughput target is stated at.
    Three CUDA graphs of back-to-back fwd + bwd steps over input sets larger than
    L2: one with the forward GEMM's launches bracketed by events, one with the dX
    GEMM's, one plain for the whole step.  Each GEMM is reported per projection
    shape (mean over its launches) and both together."""
    import torch
    import quantized_rank_fine_b200 as q
    wl = WORKLOADS["mlp4096x11008_m8192_r64"]
    M, r = wl["M"], wl["r"]
    shapes = wl["shapes"]
    nsets = max(2, math.ceil(3 * L2_BYTES / set_bytes(wl)))
    sets = build_sets(wl, nsets, seed_base=11)
    ws = q.Workspace()
    steps = 2 * nsets
    for i in range(3):
        run_step(sets[i % nsets], ws)
    torch.cuda.synchronize()

    def graph(timer):
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
                for i in range(steps):
                    run_step(sets[i % nsets], ws)
        torch.cuda.current_stream().wait_stream(side)
        if timer is not None:
            timer.disarm()
        return g

    out = {"M": M, "r": r}
    for name, kind in (("fwd_gemm", q.KERNEL_FWD_GEMM), ("dx_gemm", q.KERNEL_DX_GEMM)):
        tm = q.KernelTimer(kind, steps * len(shapes))
        g = graph(tm)
        g.replay()
        torch.cuda.synchronize()
        ts = tm.times_ms()
        del g
        per = {}
        for j, (a, b) in enumerate(shapes):
            t = statistics.mean(ts[j::len(shapes)])
            fl = flops_fwd_gemm(a, b, M, r) if name == "fwd_gemm" else flops_fwd_gemm(b, a, M, r)
            per[f"{a}x{b}"] = {"ms": t, **tensor_fracs(fl, t, pk)}
        t_all = sum(per[f"{a}x{b}"]["ms"] for a, b in shapes)
        fl_all = sum(flops_fwd_gemm(a, b, M, r) for a, b in shapes)   # the dX GEMMs have the same total
        per["both"] = {"ms": t_all, **tensor_fracs(fl_all, t_all, pk)}
        out[name] = per
    g = graph(None)
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / steps)
    del g
    t = statistics.median(times)
    out["fwd_bwd"] = {"ms_per_step": t, "tokens_per_s": M / (t * 1e-3),
                      **tensor_fracs(sum(flops_fwd_bwd(a, b, M, r) for a, b in shapes), t, pk)}
    out["note"] = ("fractions of the measured bf16 burst / sustained peaks (MEASURED_PEAKS.json) and of the "
                   f"{SPEC_BF16_TFLOPS:.0f} TFLOP/s datasheet peak; fwd + bwd = both projections")
    if ws.status() != 0:
        raise RuntimeError("a kernel wait timed out in the MLP row")
    del sets
    torch.cuda.synchronize()
    return out


def time_train_step(wl):
    """A whole training step of the workload's layer: forward, then the backward
    with the fused Adam step on the adapters (qlora_linear_bwd_adam), against the
    plain forward + backward of the headline step; both captured in CUDA graphs
    of back-to-back steps over rotated input sets larger than L2."""
    import torch
    import quantized_rank_fine_b200 as q
    M = wl["M"]
    nsets = max(2, math.ceil(3 * L2_BYTES / set_bytes(wl)))
    sets = build_sets(wl, nsets, seed_base=7)
    states = [[q.adam_state(t["A"], t["B"]) for (_, t, _) in layers] for layers in sets]
    ws = q.Workspace()
    iters = 20

    def plain(i):
        run_step(sets[i % nsets], ws)

    def adam_step(i):
        for li, (w, t, o) in enumerate(sets[i % nsets]):
            q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, Y=o["Y"], V=o["V"])
            q.qlora_linear_bwd_adam(w, t["X"], o["V"], t["dY"], t["A"], t["B"], states[i % nsets][li],
                                    5 + i, ws, dX=o["dX"])

    out = {}
    for name, fn in (("fwd_bwd", plain), ("fwd_bwd_adam", adam_step)):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                for i in range(iters):
                    fn(i)
        torch.cuda.current_stream().wait_stream(side)
        graph.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / iters)
        del graph
        t = statistics.median(times)
        out[name] = {"ms_per_step": t, "tokens_per_s": M / (t * 1e-3)}
    if ws.status() != 0:
        raise RuntimeError("a kernel wait timed out in the training-step row")
    out["adam_overhead_ms"] = out["fwd_bwd_adam"]["ms_per_step"] - out["fwd_bwd"]["ms_per_step"]
    return out


def graph_per_call(fn, iters):
    """Device time (ms) per call of a CUDA graph of `iters` back-to-back calls of
    fn(i): the throughput of a sequence of launches, where each kernel's set-up
    overlaps the one before (programmatic dependent launch)."""
    import torch
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side, capture_error_mode="relaxed"):
            for i in range(iters):
                fn(i)
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    best = None
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / iters
        best = t if best is None else min(best, t)
    del graph
    return best


def graph_timed(fn, which, iters):
    """Median duration (ms) of kernel `which` over `iters` calls of fn(i), the
    calls captured in one CUDA graph and replayed, so that the device never
    waits for the host between launches (short kernels would otherwise be timed
    together with the host's launch overhead)."""
    import torch
    import quantized_rank_fine_b200 as q
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    tm = q.KernelTimer(which, iters)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side, capture_error_mode="relaxed"):
            for i in range(iters):
                fn(i)
    torch.cuda.current_stream().wait_stream(side)
    tm.disarm()
    graph.replay()
    torch.cuda.synchronize()
    t = statistics.median(tm.times_ms())
    del graph
    return t


def time_gemv(pk):
    """Small-M forward (M = 1, 4, 16) on the 4096 x 4096 and 4096 x 11008 shapes,
    r = 16, through qlora_linear_fwd: device time per call of a CUDA graph of
    back-to-back calls (the X A kernel and the dequant-GEMV, which overlap through
    programmatic dependent launch), weights rotated over sets larger than L2.
    Algorithmic bytes: codes, absmax codes and scales, A and B, X, V and Y."""
    import torch
    import quantized_rank_fine_b200 as q
    import synth
    out = {}
    r = 16
    iters = 60
    for n_in, n_out in ((4096, 4096), (4096, 11008)):
        wbytes = n_in * n_out * (0.5 + 1 / 64)
        reps = max(3, math.ceil(3 * L2_BYTES / wbytes))
        wts = [q.qlora_quantize_nf4(synth.normal(f"gemvW{i}", (n_in, n_out), 0.02, device="cuda")) for i in range(reps)]
        A = synth.normal("gemvA", (n_in, r), 1 / math.sqrt(n_in), torch.bfloat16, "cuda")
        B = synth.normal("gemvB", (r, n_out), 0.01, torch.bfloat16, "cuda")
        for M in (1, 4, 16):
            X = synth.normal(f"gemvX{M}", (M, n_in), 1.0, torch.bfloat16, "cuda")
            Y = torch.empty((M, n_out), dtype=torch.bfloat16, device="cuda")
            V = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
            ws = q.Workspace()
            for i in range(3):
                q.qlora_linear_fwd(wts[i % reps], X, A, B, ws, Y=Y, V=V)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                with torch.cuda.graph(graph, stream=side):
                    for i in range(iters):
                        q.qlora_linear_fwd(wts[i % reps], X, A, B, ws, Y=Y, V=V)
            torch.cuda.current_stream().wait_stream(side)
            graph.replay()
            torch.cuda.synchronize()
            times = []
            for _ in range(5):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                graph.replay()
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1) / iters)
            t = statistics.median(times)
            del graph
            if ws.status() != 0:
                raise RuntimeError("a kernel wait timed out in the small-M forward")
            b = n_in * n_out * (0.5 + 1 / 64) + 4 * math.ceil(n_in * n_out / 16384) + 2 * r * (n_in + n_out) \
                + 2 * M * (n_in + n_out) + 2 * M * r
            out[f"{n_in}x{n_out}_m{M}"] = {"us_per_forward": t * 1e3, **hbm_fracs(b, t, pk), "launches": 2}
        del wts
        torch.cuda.synchronize()
    return out


def arm_ours(args, world, rank, local):
    import torch
    import quantized_rank_fine_b200 as q

    wl = WORKLOADS[args.workload]
    pk, pk_src = peaks()
    M, r = wl["M"], wl["r"]
    quantize_pass = None
    if "layer" in wl:
        # one set of the stack streams 23 GB per step: nothing stays in L2
        sets, quantize_pass = build_stack(wl, 100 * rank, pk)
        nsets = 1
    else:
        nsets = max(2, math.ceil(3 * L2_BYTES / set_bytes(wl)))
        sets = build_sets(wl, nsets, seed_base=100 * rank)
    ws = q.Workspace()
    nl = len(wl["shapes"])

    for i in range(args.warmup):
        run_step(sets[i % nsets], ws)
    torch.cuda.synchronize()
    if ws.status() != 0:
        raise RuntimeError("a kernel wait timed out during warm-up")

    # The K timed steps run as CUDA-graph replays (no host launch gaps): graph G
    # holds one step on each of the nsets input sets, graph R the K mod nsets
    # steps left over, so that exactly K steps are timed.  GT is G with the
    # library's timing hook armed: it records events around each fwd GEMM into
    # the graph.  GT runs as the last replay inside the timed region (event
    # nodes between kernels cost a little, so the other replays run G).
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream()

    def capture(count, timed):
        timer_ = q.KernelTimer(q.KERNEL_FWD_GEMM, count * nl) if timed else None
        g = torch.cuda.CUDAGraph()
        side.wait_stream(stream)
        c0 = q.qlora_launch_count()
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
                for i in range(count):
                    run_step(sets[i % nsets], ws)
        stream.wait_stream(side)
        if timer_ is not None:
            timer_.disarm()
        return g, timer_, (q.qlora_launch_count() - c0) // count

    if args.steps >= nsets:
        n_rep, n_gt, n_rem = args.steps // nsets, nsets, args.steps % nsets
    else:
        n_rep, n_gt, n_rem = 1, args.steps, 0
    G = capture(nsets, False)[0] if n_rep > 1 else None
    GT, timer, launches_per_step = capture(n_gt, True)
    R = capture(n_rem, False)[0] if n_rem else None
    for g in (G, GT, R):
        if g is not None:
            g.replay()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = clock_sampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    ev0.record(stream)
    if R is not None:
        R.replay()
    for _ in range(n_rep - 1):
        G.replay()
    if GT is not None:
        GT.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    launches = launches_per_step * args.steps
    ms_local = ev0.elapsed_time(ev1)
    gemm_ms = timer.times_ms()
    del G, GT, R
    if ws.status() != 0:
        raise RuntimeError("a kernel wait timed out in the timed region")
    ms = max_over_ranks(ms_local, world)

    tokens = M * args.steps * world
    value = tokens / (ms / 1e3)
    step_flops = sum(flops_fwd_bwd(a, b, M, r) for a, b in wl["shapes"])
    gemm_flops = [flops_fwd_gemm(a, b, M, r) for a, b in wl["shapes"]] * n_gt
    achieved = sum(gemm_flops) / (sum(gemm_ms) / 1e3) / 1e12
    timed_s = ms / 1e3
    peak, sustained, power_capped = gemm_peak(pk, timed_s, clk.get("reasons"))   # both fractions are reported
    traffic = None   # DRAM bytes per launch from the last ncu capture, if gemm.cu is unchanged since
    tp = os.path.join(ROOT, "profiles", "traffic.txt")
    if os.path.exists(tp):
        with open(tp) as f:
            for line in f:
                fields = line.split("#", 1)[0].split()
                if len(fields) == 4 and fields[0] == args.workload and fields[1] == "fwd_gemm" \
                        and fields[3] == src_hash(*GEMM_SOURCES):
                    traffic = int(fields[2])

    line = {
        "metric": "QLoRA linear fwd+bwd tokens/s",
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; W0 ~ N(0,0.02) fp32 quantised on device, X/dY ~ N(0,1) bf16)",
        "config": {**workload_config(args.workload),
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"{nsets} rotating input sets of {set_bytes(wl) / 2**20:.0f} MiB each (> L2 per cycle)"
                   if nsets > 1 else f"one input set of {set_bytes(wl) / 2**30:.1f} GiB per step (> L2)"},
        "tflops": step_flops * args.steps * world / (ms / 1e3) / 1e12,
        "roofline": {"kernel": "nf4_gemm_kernel<fwd> (fused dequant GEMM, tcgen05)", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "frac_burst": achieved / pk["bf16_tflops"],
                     "frac_sustained": achieved / pk["bf16_tflops_sustained"],
                     "frac_spec": achieved / SPEC_BF16_TFLOPS,
                     "peak_source": f"{pk_src} {'sustained' if sustained else 'burst'} bf16"
                                    + (" (sw_power_cap in the timed region)" if power_capped else ""),
                     "flops_per_launch": gemm_flops[0] if nl == 1 else
                     {f"{a}x{b}": flops_fwd_gemm(a, b, M, r) for a, b in wl["shapes"]},
                     "mean_launch_ms": statistics.mean(gemm_ms), "traffic": traffic},
        "gpu_launches": launches,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"],
                   "samples": clk["samples"], "source": clk.get("source")},
    }

    # end to end through the public API with host buffers
    line["e2e"] = e2e(args, sets, ws, wl, world)

    if world == 1 and not args.no_rows:
        line["rows"] = time_rows(wl, pk, args.rows)
    if quantize_pass is not None:
        # per GPU (each rank quantises its own replica of the stack); slowest rank
        slow = max_over_ranks(quantize_pass["ms"], world) / quantize_pass["ms"]
        quantize_pass.update(ms=quantize_pass["ms"] * slow, gbs=quantize_pass["gbs"] / slow,
                             frac_hbm=quantize_pass["frac_hbm"] / slow,
                             frac_hbm_spec=quantize_pass["frac_hbm_spec"] / slow)
        line.setdefault("rows", {})["quantize_pass"] = quantize_pass
    if world == 1 and rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=20.0)
    return line


def e2e_slots(sets):
    """Two device slots of per-step data for the end-to-end leg: slot s holds the
    inputs X and dY and the gradient outputs dA and dB that step i (with
    i % 2 = s) uses; weights, adapters and the other outputs are shared.  With
    one input set (the stack) the second slot gets its own X, dY, dA and dB."""
    import torch
    if len(sets) >= 2:
        return [sets[0], sets[1]]
    fresh = {}

    def twin(d):
        if d.data_ptr() not in fresh:
            fresh[d.data_ptr()] = torch.empty_like(d)
        return fresh[d.data_ptr()]

    second = []
    for w, t, o in sets[0]:
        t2 = dict(t, X=twin(t["X"]), dY=twin(t["dY"]))
        o2 = dict(o, dA=torch.empty_like(o["dA"]), dB=torch.empty_like(o["dB"]))
        second.append((w, t2, o2))
    return [sets[0], second]


def e2e(args, sets, ws, wl, world):
    """Same metric through the public API from host memory: every step copies its
    inputs (each distinct X and dY) from pinned host memory to the device and the
    adapter gradients dA, dB back to pinned host memory.  The copies run on their
    own streams (host-to-device, device-to-host) and overlap the layer calls of
    the neighbouring steps; two device slots alternate, and events order each
    slot's copy-in, layer calls and copy-out."""
    import torch
    M = wl["M"]
    slots = e2e_slots(sets)
    ins, outs = [], []          # per slot: [(device input, pinned host source)], [(device grad, pinned host dest)]
    host_src = {}               # one pinned host copy per distinct input of slot 0, the source of both slots
    for s, layers in enumerate(slots):
        seen, si = set(), []
        for j, (w, t, o) in enumerate(layers):
            for k in ("X", "dY"):
                d = t[k]
                if d.data_ptr() in seen:          # the stack's shared activations are copied once
                    continue
                seen.add(d.data_ptr())
                key = (j, k)
                if key not in host_src:
                    host_src[key] = torch.empty(d.shape, dtype=d.dtype, pin_memory=True).copy_(slots[0][j][1][k])
                si.append((d, host_src[key]))
        ins.append(si)
        outs.append([(o[k], torch.empty(o[k].shape, dtype=torch.float32).pin_memory())
                     for w, t, o in layers for k in ("dA", "dB")])
    h2d = sum(d.numel() * d.element_size() for d, _ in ins[0])
    d2h = sum(d.numel() * d.element_size() for d, _ in outs[0])
    steps = 10 if "layer" in wl else max(10, args.steps // 4)
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def run(n, e_start=None):
        ev = lambda: torch.cuda.Event()
        h_done, c_done, d_done = [], [], []
        if e_start is not None:
            up.wait_event(e_start)
        for i in range(n):
            s = i % 2
            if i >= 2:
                up.wait_event(c_done[i - 2])      # slot s's inputs were read by step i - 2
            with torch.cuda.stream(up):
                for d, h in ins[s]:
                    d.copy_(h, non_blocking=True)
            h_done.append(ev())
            h_done[i].record(up)
            comp.wait_event(h_done[i])
            if i >= 2:
                comp.wait_event(d_done[i - 2])    # slot s's gradients were copied out after step i - 2
            run_step(slots[s], ws)
            c_done.append(ev())
            c_done[i].record(comp)
            down.wait_event(c_done[i])
            with torch.cuda.stream(down):
                for d, h in outs[s]:
                    h.copy_(d, non_blocking=True)
            d_done.append(ev())
            d_done[i].record(down)
        comp.wait_event(d_done[-1])

    run(3)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(comp)
    run(steps, e0)
    e1.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    return {"value": M * steps * world / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "overlap": "copy-in, layer calls and copy-out of neighbouring steps on three streams, two device slots"}


# ------------------------------------------------------------------ the oracle (CPU baseline / reference arm)

def oracle_cores():
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        threadpool_limits(n)
        used = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        used = n
    return n, used


def oracle_inputs(workload, rows_frac, tokens):
    """Oracle inputs of a bounded sample: the first rows_frac of each weight's
    input rows (whole double-quant groups) and `tokens` tokens, quantised by the
    oracle itself.  For the stack the sample is one decoder layer's seven
    projections (all 32 layers have the same shapes)."""
    import synth
    from oracle import nf4
    wl = WORKLOADS[workload]
    r = wl["r"]
    shapes = [(a, b) for _, a, b, _ in wl["layer"]] if "layer" in wl else wl["shapes"]
    layers = []
    for li, (n_in, n_out) in enumerate(shapes):
        rows_per_group = max(1, (64 * 256) // n_out)
        n_rows = max(rows_per_group, int(n_in * rows_frac) // rows_per_group * rows_per_group)
        t = synth.layer_inputs(n_rows, n_out, tokens, r, tag=f"oracle{li}:")
        codes, dqc, dqs = nf4.quantize_nf4(t["W0"].numpy())
        layers.append((t, (codes, dqc, dqs), n_rows, n_out, n_in))
    return layers


def oracle_step(layers):
    """One oracle forward + backward over the sample (dequantisation included)."""
    from oracle import linear, nf4
    for t, (codes, dqc, dqs), n_rows, n_out, _ in layers:
        Wq = nf4.dequantize_bf16(codes, dqc, dqs, n_rows, n_out)
        linear.forward(t["X"], t["A"], t["B"], Wq)
        linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])


def oracle_sample_time(workload, budget_s):
    """Pick a sample that costs about budget_s per step; returns (layers, seconds
    per step, fraction of the full step's work)."""
    wl = WORKLOADS[workload]
    M = wl["M"]
    tokens = min(M, 256)
    frac = 1.0 / 16
    while True:
        layers = oracle_inputs(workload, frac, tokens)
        t0 = time.perf_counter()
        oracle_step(layers)
        dt = time.perf_counter() - t0
        if dt * 2 > budget_s or frac >= 1.0:
            break
        frac = min(1.0, frac * 2)
    # the sampled share of the whole step's work (work ~ rows x columns x tokens)
    row_frac = sum(l[2] * l[3] for l in layers) / sum(l[4] * l[3] for l in layers) / wl.get("layers", 1)
    return layers, dt, row_frac, tokens


def sample_layers(workload):
    wl = WORKLOADS[workload]
    return f" (of the whole stack: one layer's 7 projections, x {wl['layers']} layers)" if "layer" in wl else ""


def cpu_baseline(workload, budget_s=20.0):
    cores, used = oracle_cores()
    layers, dt, row_frac, tokens = oracle_sample_time(workload, budget_s / 4)
    reps = max(1, int(budget_s / max(dt, 1e-3) / 2))
    ts = []
    for _ in range(min(reps, 5)):
        t0 = time.perf_counter()
        oracle_step(layers)
        ts.append(time.perf_counter() - t0)
    dt = statistics.median(ts)
    value = tokens * row_frac / dt   # tokens/s of the full step (work scales with the weights' size)
    return {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"float64 oracle fwd+bwd incl. dequantisation: {tokens} tokens through the leading input "
                      f"rows of each weight{sample_layers(workload)}, {row_frac:.5f} of the step's weights; "
                      f"median of {len(ts)} runs, scaled to the full step"}


def arm_reference(args, world, rank):
    """The reference arm: the float64 oracle on the host cores, K timed steps."""
    if rank != 0:
        return None
    wl = WORKLOADS[args.workload]
    budget = max(0.05, 150.0 / max(1, args.steps + args.warmup))
    layers, _, row_frac, tokens = oracle_sample_time(args.workload, budget)
    for _ in range(args.warmup):
        oracle_step(layers)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(layers)
    dt = time.perf_counter() - t0
    cores, used = oracle_cores()
    value = tokens * row_frac * args.steps / dt
    sample = (f"float64 oracle fwd+bwd incl. dequantisation, per step {tokens} tokens through the leading "
              f"input rows of each weight{sample_layers(args.workload)}, {row_frac:.5f} of the step's weights; "
              f"scaled to the full step")
    return {
        "impl": "reference", "metric": "QLoRA linear fwd+bwd tokens/s", "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.workload),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world, rank, local = dist_init(args)
    if args.impl == "reference":
        line = arm_reference(args, world, rank)
    elif args.rows_only:
        pk, _ = peaks()
        line = {"rows": time_rows(WORKLOADS[args.workload], pk, args.rows)} if rank == 0 else None
    else:
        line = arm_ours(args, world, rank, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
