#!/usr/bin/env python
"""Benchmark of the W6A6 / W6A8 group-quantized linear layers of LLaMA-2-70B.

Workload (one "step"): for every M in {1, 16, 512, 8192} and every linear layer
of the LLaMA-2-70B configuration -- q and o (8192x8192, 6-bit activations),
gate and up (28672x8192, 6-bit activations), down (8192x28672, 8-bit
activations) -- quantize the layer's FP16 activations to group codes (group
size 128) and run the group GEMM against 6-bit packed weights.  Inputs are
seeded synthetic tensors of those shapes (weights N(0, 0.015); activations
N(0, 1) with 0.5% outlier channels x50, one input per site: attention input,
attention output, MLP input, MLP activation); every step streams 629 MB of
distinct packed weights per M, far more than the 126 MB L2, so each GEMM reads
its weights from HBM.

Output: one JSON line (rank 0).  `value` is whole-job TOPS (2*M*N*K summed over
the step, divided by the device time), measured over CUDA-graph replays of the
step with inputs resident in HBM.  `roofline` covers both halves of the
metric: the tensor-bound GEMM launches at M >= 512 against the int8 peak, and
the HBM-bound layers at M <= 16 against the measured copy bandwidth.  `e2e` is
the same metric through the public Python API with host buffers (pinned H2D
copy of every layer input, D2H copy of every output) inside the timed region,
copies and layer calls on three streams.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl flexq|reference]

`--impl reference` times the CPU oracle (the plain restatement of the method
used by the tests) on a bounded sample of the same workload.  With --gpus N > 1
(launched by torchrun) every rank runs its own replica of the workload (weak
scaling, no collective on the data path); ranks meet only for the barrier and
the max-over-ranks timing.
"""

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("W6A6/W6A8 linear-layer TOPS and % of roofline "
          "(HBM at small M, INT8 peak at large M)")
UNIT = "TOPS"
GS = 128
ACT_BITS = 6
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0          # nominal dense ratio (4.5 vs 2.25 PFLOP/s)


# ------------------------------------------------------------- workload ----
HEADLINE_LAYERS = ("q", "o", "gate", "up", "down")
WEIGHT_STD = 0.015
OUTLIER_FRAC, OUTLIER_SCALE = 0.005, 50.0
TENSOR_MIN_M = 512            # launches at or above this M are tensor-bound
DECODE_MAX_M = 16             # launches at or below this M are HBM-bound


def workload_shapes(ms=None, layers=None):
    """M values and [(name, N, K, act_bits, site)] of the LLaMA-2-70B step."""
    from bit_group_quantized_flexq_b200 import inputs, stack
    ms = list(ms) if ms else list(inputs.LLAMA2_70B_M)
    bits = stack.LLAMA2_70B_MIXED["act_bits"]
    lay = [(n, N, K, bits[n], site) for (n, N, K, site) in inputs.LLAMA2_70B_BLOCK
           if n in HEADLINE_LAYERS and (not layers or n in layers)]
    return ms, lay


def step_ops(ms, layers):
    return sum(2.0 * M * l[1] * l[2] for M in ms for l in layers)


def gemm_bytes(M, N, K, gs=GS):
    """Algorithmic HBM bytes of one GEMM launch: packed weights (0.75 B per
    element), weight scales, int8 activation codes and scales, FP16 output."""
    return 0.75 * N * K + 2.0 * N * K / gs + M * K + 2.0 * M * K / gs + 2.0 * M * N


def workload_name(ms, layers):
    return ("LLaMA-2-70B linear layers, W6A6 q/o/gate/up + W6A8 down ("
            + ",".join(f"{l[0]}:{l[1]}x{l[2]}:A{l[3]}" for l in layers)
            + f"), group 128, M in {{{','.join(map(str, ms))}}}")


# ------------------------------------------------------------ distributed --
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def dist_init(backend):
    import datetime
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(x, device=None):
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(units_per_rank, world, t_max_s):
    """Whole-job throughput: the units all ranks processed over the max time."""
    return units_per_rank * world / t_max_s


# ----------------------------------------------------------------- clocks --
class ClockSampler:
    """SM clocks and throttle reasons of one GPU, polled every few
    milliseconds from a thread through NVML while the timed region runs
    (nvidia-smi's ~100 ms period can miss a region of a few tens of ms);
    falls back to nvidia-smi when NVML is not importable."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.002

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.nvml = None
        self.lines = []
        self.samples = []            # (sm_mhz, max_mhz, reasons bitmask)
        self._stop = threading.Event()
        self.thread = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.nvml = (pynvml, h)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        except Exception:            # no NVML: sample with nvidia-smi instead
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _poll(self):
        pynvml, h = self.nvml
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, self.max_mhz, rs))
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        self._stop.set()
        if self.nvml is not None:
            self.thread.join(timeout=5)
            return self.summary_nvml()
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        return self.summary()

    def summary_nvml(self):
        pynvml, _ = self.nvml
        if not self.samples:
            return None
        bits = {"hw_slowdown": getattr(pynvml, "nvmlClocksEventReasonHwSlowdown", 0x8),
                "hw_thermal_slowdown": getattr(pynvml, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                "sw_thermal_slowdown": getattr(pynvml, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                "sw_power_cap": getattr(pynvml, "nvmlClocksEventReasonSwPowerCap", 0x4)}
        reasons = sorted(n for n, b in bits.items() if any(r & b for _, _, r in self.samples))
        return {"sm_mhz": statistics.median(sm for sm, _, _ in self.samples),
                "sm_max_mhz": max(mx for _, mx, _ in self.samples),
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi"}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_digest():
    """Digest of the GEMM sources' code: comments and whitespace removed, so
    that only a change of the code itself marks a profiled figure stale."""
    h = hashlib.sha256()
    for f in ("flexq_gemm.cuh", "flexq_gemm_wide.cuh", "flexq_ptx.cuh", "flexq_api.cu"):
        with open(os.path.join(ROOT, "bit_group_quantized_flexq_b200", "csrc", f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


TRAFFIC_SUMMARY = os.path.join("profiles", "gemm_w6ax_wide_70b_step_traffic.md")


def profiled_traffic():
    """DRAM bytes per launch of the dominant GEMM from the committed ncu
    summary of the bench step's wide launches (its `dram_bytes_per_launch`
    and `kernel_src_sha` lines), or None when that summary is missing or the
    kernel sources changed since the capture."""
    p = os.path.join(ROOT, TRAFFIC_SUMMARY)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        text = f.read()
    sha = re.search(r"kernel_src_sha:\s*([0-9a-f]+)", text)
    nbytes = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not sha or not nbytes or sha.group(1) != kernel_source_digest():
        return None
    return int(nbytes.group(1))


# ------------------------------------------------------------ flexq arm ----
class Layers:
    """Device-resident workload: packed weights, per-site activations, their
    codes and scales, outputs.  Layer tuples: (name, N, K, bits, site, wp, ws)."""

    def __init__(self, ms, layers, device):
        import torch
        from bit_group_quantized_flexq_b200 import flexq, inputs
        self.ms, self.layers, self.dev = ms, layers, device
        self.w = []
        for name, N, K, bits, site in layers:
            w16 = inputs.weights(N, K, std=WEIGHT_STD, seed=inputs.layer_seed("70b", name),
                                 device=device)
            wp, ws = flexq.quantize_weight(w16, GS)
            del w16
            self.w.append((name, N, K, bits, site, wp, ws))
        # layers that read the same input at the same width share one call
        # (flexq.linear_group / one quantization): gate and up
        self.groups = []
        by_q = {}
        for layer in self.w:
            q = (layer[4], layer[3])
            if q in by_q:
                self.groups[by_q[q]].append(layer)
            else:
                by_q[q] = len(self.groups)
                self.groups.append([layer])
        self.x, self.xq, self.xs, self.y = {}, {}, {}, {}
        sites = {site: K for (_, _, K, _, site) in layers}
        for M in ms:
            for site, K in sites.items():
                x = inputs.activations(M, K, outlier_frac=OUTLIER_FRAC,
                                       outlier_scale=OUTLIER_SCALE,
                                       seed=inputs.layer_seed("70b-x", M, site))
                self.x[(M, site)] = x.to(device)
            for (name, N, K, bits, site, _, _) in self.w:
                self.xq[(M, name)] = torch.empty(M, K, dtype=torch.int8, device=device)
                self.xs[(M, name)] = torch.empty(K // GS, flexq.act_scales_ld(M),
                                                 dtype=torch.float16, device=device)
                self.y[(M, name)] = torch.empty(M, N, dtype=torch.float16, device=device)
        torch.cuda.synchronize(device)

    def packed_bytes(self):
        return sum(l[5].numel() for l in self.w)

    def split_m(self, M):
        """The tensor-bound M run the quantizer and the GEMM as separate
        launches, so that events bracket every GEMM launch."""
        return M >= TENSOR_MIN_M

    def launches_per_step(self):
        from bit_group_quantized_flexq_b200 import flexq
        n = 0
        for M in self.ms:
            for g in self.groups:
                if self.split_m(M):
                    n += 1 + len(g)
                else:
                    n += flexq.group_plan(M, g[0][2], GS, [l[1] for l in g])[3]
        return n

    def quant(self, M, group):
        """One quantization of the group's input (codes kept under its first layer)."""
        from bit_group_quantized_flexq_b200 import flexq
        name, _, _, bits, site, _, _ = group[0]
        flexq.quantize_act(self.x[(M, site)], GS, bits,
                           out=(self.xq[(M, name)], self.xs[(M, name)]))

    def gemm(self, M, group, layer):
        from bit_group_quantized_flexq_b200 import flexq
        first = group[0][0]
        name, N, K, bits, _, wp, ws = layer
        flexq.gemm(self.xq[(M, first)], self.xs[(M, first)], wp, ws, N, GS, bits,
                   out=self.y[(M, name)])

    def linear(self, M, group):
        """The group's layers from FP16 activations: one flexq.linear, or one
        grouped call (flexq.linear_group) for layers sharing their input."""
        from bit_group_quantized_flexq_b200 import flexq
        if len(group) == 1:
            name, N, K, bits, site, wp, ws = group[0]
            flexq.linear(self.x[(M, site)], wp, ws, N, GS, bits, out=self.y[(M, name)])
            return
        bits, site = group[0][3], group[0][4]
        flexq.linear_group(self.x[(M, site)], [(l[5], l[6], l[1]) for l in group], GS, bits,
                           outs=[self.y[(M, l[0])] for l in group])

    def run_m(self, M):
        for group in self.groups:
            self.linear(M, group)

    def segments(self):
        """The step cut into replayable pieces: at the HBM-bound M all layers
        of an M are one piece (flexq.linear per layer, flexq.linear_group for
        gate and up); at the tensor-bound M every quantization (one per input)
        and every GEMM is its own piece so that events can bracket the GEMM
        launches."""
        segs = []
        for M in self.ms:
            if self.split_m(M):
                for group in self.groups:
                    segs.append(("quant", M, group[0], (lambda M=M, g=group: self.quant(M, g))))
                    for layer in group:
                        segs.append(("gemm", M, layer,
                                     (lambda M=M, g=group, l=layer: self.gemm(M, g, l))))
            else:
                segs.append(("all", M, None, (lambda M=M: self.run_m(M))))
        return segs


def run_flexq(args, rank, world):
    import torch
    from bit_group_quantized_flexq_b200 import flexq
    _, _, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    flexq.lib()                                   # fail loudly if not built
    ms, layers = workload_shapes(args.ms, args.layers)
    W = Layers(ms, layers, device)
    ops = step_ops(ms, layers)

    # eager warm-up (first calls set kernel attributes; nothing is captured yet)
    for M in ms:
        W.run_m(M)
    torch.cuda.synchronize(device)

    stream = torch.cuda.Stream(device)
    segs = W.segments()
    runners = []
    if args.graph:
        for (_, _, _, fn) in segs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    fn()
            runners.append(g.replay)
        graphs = runners
        torch.cuda.synchronize(device)
    else:
        runners = [fn for (_, _, _, fn) in segs]
        graphs = []

    def new_event():
        return torch.cuda.Event(enable_timing=True)

    # one event before the first piece and one after every piece, per step
    evs = [[new_event() for _ in range(len(segs) + 1)] for _ in range(args.steps)]

    def run_step(ev):
        if ev is not None:
            ev[0].record(stream)
        for k, run in enumerate(runners):
            run()
            if ev is not None:
                ev[k + 1].record(stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            run_step(None)
        torch.cuda.synchronize(device)
        barrier(device)
        torch.cuda.synchronize(device)
        clocks = ClockSampler(device.index if device.index is not None else 0)
        clocks.start()
        time.sleep(0.05)                          # sampler running before timing
        t0, t1 = new_event(), new_event()
        t0.record(stream)
        for i in range(args.steps):
            run_step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(device)
        clock_summary = clocks.stop()
    barrier(device)
    elapsed_ms = t0.elapsed_time(t1)
    t_max_s = max_over_ranks(elapsed_ms / 1e3, device)
    status, msg = flexq.device_status(device)
    if status != flexq.FLEXQ_OK:
        raise RuntimeError(f"device status after the timed region: {msg}")

    def seg_ms(k):
        return statistics.mean(evs[i][k].elapsed_time(evs[i][k + 1]) for i in range(args.steps))

    peaks, peak_src = measured_peaks()
    long_region = elapsed_ms > 1000.0
    bf16 = peaks.get("bf16_tflops_sustained" if long_region else "bf16_tflops",
                     peaks.get("bf16_tflops"))
    int8_peak = bf16 * INT8_OVER_BF16
    hbm = peaks["hbm_gbs"]

    # per M: device time of its pieces, TOPS, and the GEMM launches alone
    per_m = []
    gemm_ops = gemm_ms = 0.0
    dec_bytes = dec_ms = 0.0
    for M in ms:
        ks = [k for k, sg in enumerate(segs) if sg[1] == M]
        m_ms = statistics.mean(evs[i][ks[0]].elapsed_time(evs[i][ks[-1] + 1])
                               for i in range(args.steps))
        m_ops = sum(2.0 * M * l[1] * l[2] for l in layers)
        row = {"M": M, "ms": round(m_ms, 5), "tops": round(m_ops / (m_ms / 1e3) / 1e12, 3)}
        gk = [k for k in ks if segs[k][0] == "gemm"]
        if gk:
            g_ms = sum(seg_ms(k) for k in gk)
            row["gemm_ms"] = round(g_ms, 5)
            row["gemm_tops"] = round(m_ops / (g_ms / 1e3) / 1e12, 3)
            row["gemm_frac_int8"] = round(m_ops / (g_ms / 1e3) / 1e12 / int8_peak, 4)
            row["gemm_us_by_layer"] = {segs[k][2][0]: round(seg_ms(k) * 1e3, 2) for k in gk}
            gemm_ops += m_ops
            gemm_ms += g_ms
        if M <= DECODE_MAX_M:
            nbytes = sum(linear_bytes(M, l[1], l[2]) for l in layers)
            gbs = nbytes / (m_ms / 1e3) / 1e9
            row["GB/s"] = round(gbs, 1)
            row["frac_hbm"] = round(gbs / hbm, 4)
            dec_bytes += nbytes
            dec_ms += m_ms
        per_m.append(row)
    achieved_tops = gemm_ops / (gemm_ms / 1e3) / 1e12 if gemm_ms else 0.0
    n_gemm = sum(1 for sg in segs if sg[0] == "gemm")
    dec_gbs = dec_bytes / (dec_ms / 1e3) / 1e9 if dec_ms else 0.0

    # GEMM-only diagnostics per M (after the timed region, not part of value)
    diag = gemm_diagnostics(W, device, hbm, int8_peak) if args.diag else None

    traffic = profiled_traffic()
    result = {
        "metric": METRIC,
        "value": round(aggregate(ops * args.steps, world, t_max_s) / 1e12, 3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t_max_s * 1e3 / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic",
        "config": {
            "workload": workload_name(ms, layers),
            "group_size": GS, "weight_bits": 6,
            "act_bits": {l[0]: l[3] for l in layers},
            "shapes": [[l[0], l[1], l[2]] for l in layers], "M": ms,
            "ops_per_step": ops,
            "l2": (f"inputs larger than L2: each M streams {W.packed_bytes() / 1e6:.0f} MB of "
                   "distinct packed weights"),
            "timing": "CUDA-graph replay of each step" if args.graph else "eager launches",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "per_m": per_m,
        "roofline": {
            "bound": "tensor",
            "kernel": (f"gemm_w6ax_wide_kernel (GEMM launches at M >= {TENSOR_MIN_M}, "
                       f"{n_gemm} per step)"),
            "achieved": round(achieved_tops, 2),
            "peak": round(int8_peak, 1),
            "unit": "TFLOP/s",
            "frac": round(achieved_tops / int8_peak, 4) if int8_peak else None,
            "peak_source": (f"{peak_src}: {'sustained' if long_region else 'burst'} bf16 x "
                            f"{INT8_OVER_BF16:g} (nominal int8/bf16 dense ratio)"),
            "avg_launch_us": round(gemm_ms * 1e3 / max(1, n_gemm), 2),
            "traffic": traffic,
            "decode": {
                "bound": "hbm",
                "kernel": f"whole layers (quantization + GEMM) at M <= {DECODE_MAX_M}",
                "achieved": round(dec_gbs, 1), "peak": round(hbm, 1), "unit": "GB/s",
                "frac": round(dec_gbs / hbm, 4),
                "bytes": "0.75 B per weight element + FP16 weight scales + FP16 input and output",
                "peak_source": f"{peak_src}: copy bandwidth",
            },
        },
        "gpu_launches": W.launches_per_step() * args.steps,
        "clocks": clock_summary,
    }
    if args.graph:
        result["config"]["timing"] = (f"CUDA-graph replay: one graph per M below {TENSOR_MIN_M}, "
                                      "one per launch above; events between graph launches")
    if diag:
        result["gemm_by_m"] = diag
    if args.diag and rank == 0:
        result["int8_library_context"] = int8_library_context(W, device, max(ms))
        result["act_quant"] = act_quant_diagnostics(device, hbm)
        result["mixed_stack"] = stack_diagnostics(device, hbm, int8_peak)
        result["other_configs"] = run_sweep(device, hbm, int8_peak, subset=True)
        result["layout_ab"] = layout_ab(device, hbm)
    if args.e2e:
        result["e2e"] = run_e2e(W, args, device, world)
    if rank == 0 and world == 1 and args.cpu_baseline:
        result["cpu_baseline"] = run_cpu_baseline(args.cpu_budget_s)
    if rank == 0:
        print(json.dumps(result), flush=True)
    graphs.clear()
    runners.clear()


def roofline(ops, nbytes, us, hbm_gbs, int8_peak_tops):
    """(bound, fraction) of a launch against the attainable rate
    min(int8 peak, HBM bandwidth x ops per algorithmic byte)."""
    intensity = ops / nbytes
    mem_tops = hbm_gbs * 1e9 * intensity / 1e12
    bound = "hbm" if mem_tops < int8_peak_tops else "tensor"
    achieved = ops / (us * 1e-6) / 1e12
    return bound, achieved / min(mem_tops, int8_peak_tops)


def linear_bytes(M, N, K, gs=GS):
    """Algorithmic HBM bytes of one whole linear layer from FP16 activations:
    packed weights, weight scales, FP16 activations read once, FP16 output."""
    return 0.75 * N * K + 2.0 * N * K / gs + 2.0 * M * K + 2.0 * M * N


def _graph_time_us(body, device, stream, reps):
    """Device time of one `body()` from a CUDA graph of `reps` bodies."""
    import torch
    with torch.cuda.stream(stream):
        body()                                    # eager pass: sets attributes, workspace
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                body()
        g.replay()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize(device)
    t_us = e0.elapsed_time(e1) * 1e3 / reps
    del g
    return t_us


def gemm_diagnostics(W, device, hbm_gbs, int8_peak_tops, reps=None):
    """Per-M times and fractions of the attainable roofline (min(int8 peak,
    HBM x intensity): HBM-bound at decode sizes, tensor-bound at M = 512 and
    above) of the step's layers, each timed from a CUDA graph that holds
    `reps` rounds of them back to back (the other layers' weights stream in
    between, so each launch reads its weights cold); events bracket the graph
    replay, so host launch work is not timed.  `gemm_*`: the GEMM alone on
    quantized activations; `linear_*`: the whole layers from FP16 activations
    through flexq.linear (flexq.linear_group for gate and up)."""
    import torch
    from bit_group_quantized_flexq_b200 import flexq
    out = []
    stream = torch.cuda.Stream(device)
    for M in W.ms:
        for group in W.groups:
            W.quant(M, group)                     # the GEMMs' quantized inputs
        n_reps = reps or (2 if M >= 4096 else 5)

        def gemm_body():
            for group in W.groups:
                for layer in group:
                    W.gemm(M, group, layer)

        def linear_body():
            for group in W.groups:
                W.linear(M, group)

        t_us = _graph_time_us(gemm_body, device, stream, n_reps)
        l_us = _graph_time_us(linear_body, device, stream, n_reps)
        flops = sum(2.0 * M * l[1] * l[2] for l in W.w)
        row = {"M": M}
        for key, us, nbytes in (("gemm", t_us, sum(gemm_bytes(M, l[1], l[2]) for l in W.w)),
                                ("linear", l_us, sum(linear_bytes(M, l[1], l[2]) for l in W.w))):
            gbs = nbytes / (us * 1e-6) / 1e9
            tops = flops / (us * 1e-6) / 1e12
            bound, frac = roofline(flops, nbytes, us, hbm_gbs, int8_peak_tops)
            row["bound"] = bound
            row[f"{key}_us"] = round(us, 2)
            row[f"{key}_GB/s"] = round(gbs, 1)
            row[f"{key}_TOPS"] = round(tops, 2)
            row[f"{key}_frac"] = round(frac, 4)
        row["plan"] = [list(flexq.plan(M, l[1], l[2], GS)) for l in W.w]
        out.append(row)
    return out


def act_quant_diagnostics(device, hbm_gbs, K=8192, ms=(1, 2048, 16384), reps=20):
    """The activation quantizer alone on FP16 [M, 8192] inputs with the
    workload's outlier channels (the sweep configuration's separate timing):
    device time per call from a CUDA graph of `reps` calls, and its HBM
    roofline at 2 B read + 1 B written per element + 2 B per group scale."""
    import torch
    from bit_group_quantized_flexq_b200 import flexq, inputs
    out = []
    stream = torch.cuda.Stream(device)
    for M in ms:
        x = inputs.activations(M, K, outlier_frac=0.005, outlier_scale=50.0,
                               seed=inputs.layer_seed("act-sweep", M, K)).to(device)
        xq = torch.empty(M, K, dtype=torch.int8, device=device)
        xs = torch.empty(K // GS, flexq.act_scales_ld(M), dtype=torch.float16, device=device)
        with torch.cuda.stream(stream):
            flexq.quantize_act(x, GS, ACT_BITS, out=(xq, xs))
            torch.cuda.synchronize(device)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    flexq.quantize_act(x, GS, ACT_BITS, out=(xq, xs))
            g.replay()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize(device)
        us = e0.elapsed_time(e1) * 1e3 / reps
        del g
        nbytes = 3.0 * M * K + 2.0 * M * K / GS
        gbs = nbytes / (us * 1e-6) / 1e9
        out.append({"M": M, "K": K, "us": round(us, 2), "GB/s": round(gbs, 1),
                    "bound": "hbm", "frac": round(gbs / hbm_gbs, 4)})
    return out


def stack_diagnostics(device, hbm_gbs, int8_peak_tops, ms=(1, 16)):
    """The mixed W6A6/W6A8 layer stack (stack.LayerStack) on one LLaMA-2-70B
    block (q, k, v, o, gate, up, down; 8-bit activations for down), seeded
    synthetic weights drawn on the device, at the decode sizes (the step
    above measures the large ones): per M, the device time of one block
    forward from FP16 activations (CUDA graph of a few forwards), with the
    attainable roofline min(int8 peak, HBM x intensity).  Three ways to run
    it: the layers of one input site as one grouped launch, each with its
    own packed weights (`by_m`, the default); every layer its own launch
    (`by_m_single_launches`); the layers of a site merged into one weight
    matrix (`by_m_fused_sites`, a different weight layout).  The same for
    the LLaMA-2-7B block, W6A6 (`llama2_7b_block`; two copies of the block
    run in turn, 311 MB of packed weights, so that they do not sit in L2)."""
    import torch
    from bit_group_quantized_flexq_b200 import inputs, stack
    res = {}
    for key, kw in (("by_m", {}), ("by_m_single_launches", {"group_sites": False}),
                    ("by_m_fused_sites", {"fuse_sites": True})):
        st = stack.LayerStack(inputs.LLAMA2_70B_BLOCK, stack.LLAMA2_70B_MIXED, device=device, **kw)
        res[key] = _stack_rows([st], device, hbm_gbs, int8_peak_tops, ms)
        bits, gs, packed = st.bits, st.gs, st.packed_bytes()
        del st
        torch.cuda.empty_cache()
    cfg7 = {"group_size": 128, "act_bits": {name: 6 for name, _, _, _ in inputs.LLAMA2_7B_BLOCK}}
    res7 = {}
    for key, kw in (("by_m", {}), ("by_m_single_launches", {"group_sites": False})):
        sts = [stack.LayerStack(inputs.LLAMA2_7B_BLOCK, cfg7, device=device, seed=c, **kw)
               for c in range(2)]
        res7[key] = _stack_rows(sts, device, hbm_gbs, int8_peak_tops, ms)
        del sts
        torch.cuda.empty_cache()
    return {"block": "LLaMA-2-70B (q, k, v, o, gate, up, down)",
            "act_bits": bits, "group_size": gs, "packed_MB": round(packed / 1e6, 1), **res,
            "llama2_7b_block": {"act_bits": 6, "group_size": 128, "copies": 2, **res7}}


def _stack_rows(stacks, device, hbm_gbs, int8_peak_tops, ms):
    """Per M, one forward of every stack in `stacks` in turn (each its own
    weights) per timed pass; figures for the whole pass."""
    import torch
    from bit_group_quantized_flexq_b200 import inputs
    stream = torch.cuda.Stream(device)
    rows = []
    st0 = stacks[0]
    for M in ms:
        acts = {site: inputs.activations(M, K, outlier_frac=0.005, outlier_scale=50.0,
                                         seed=inputs.layer_seed("70b-x", M, site)).to(device)
                for site, K in st0.sites().items()}
        out = {name: torch.empty(M, N, dtype=torch.float16, device=device)
               for name, N, K, _ in st0.layers}

        def passes():
            for st in stacks:
                st.forward(acts, out)
        reps = 2 if M >= 4096 else 5
        us = _graph_time_us(passes, device, stream, reps)
        flops = len(stacks) * sum(2.0 * M * N * K for _, N, K, _ in st0.layers)
        nbytes = len(stacks) * sum(linear_bytes(M, N, K, st0.gs) for _, N, K, _ in st0.layers)
        gbs = nbytes / (us * 1e-6) / 1e9
        tops = flops / (us * 1e-6) / 1e12
        bound, frac = roofline(flops, nbytes, us, hbm_gbs, int8_peak_tops)
        rows.append({"M": M, "us": round(us, 2), "TOPS": round(tops, 2), "GB/s": round(gbs, 1),
                     "bound": bound, "frac": round(frac, 4),
                     "launches": len(stacks) * st0.launches(M)})
        del acts, out
    return rows


def run_sweep(device, hbm_gbs, int8_peak_tops, subset=False):
    """The other measured configurations, one JSON line (`--sweep`; not part
    of the default run): the LLaMA-2-13B W6A8 layers at M in {1, 64, 4096}
    and the N = K = 8192 sweep over group size {32, 64, 128, 256}, W6A6 and
    W6A8, M in {1, 8, 32, 128, 1024, 4096, 16384}.  Per case the GEMM alone
    (codes given) and the whole layer from FP16 activations (flexq.linear),
    device time per call from a CUDA graph that rotates over enough copies
    of the packed weights to exceed L2, against the attainable rate
    min(int8 peak, HBM bandwidth x arithmetic intensity).  With subset=True
    (the default run's extra key): the 13B layers at all their M, and the
    sweep at M in {1, 4096} for every group size, W6A6 and W6A8."""
    import torch
    from bit_group_quantized_flexq_b200 import flexq, inputs
    stream = torch.cuda.Stream(device)

    def case(M, N, K, gs, bits, wp0, ws0, copies):
        x = inputs.activations(M, K, outlier_frac=0.01, outlier_scale=20.0,
                               seed=inputs.layer_seed("sweep-x", M, K)).to(device)
        xq, xs = flexq.quantize_act(x, gs, bits)
        y = torch.empty(M, N, dtype=torch.float16, device=device)
        reps = 1 if M >= 4096 else 3

        def gemm():
            for wp, ws in copies:
                flexq.gemm(xq, xs, wp, ws, N, gs, bits, out=y)

        def lin():
            for wp, ws in copies:
                flexq.linear(x, wp, ws, N, gs, bits, out=y)
        row = {"M": M, "N": N, "K": K, "gs": gs, "act_bits": bits,
               "plan": list(flexq.plan(M, N, K, gs)),
               "linear_launches": flexq.linear_launches(M, N, K, gs)}
        for key, body, nbytes in (("gemm", gemm, gemm_bytes(M, N, K, gs)),
                                  ("linear", lin, linear_bytes(M, N, K, gs))):
            us = _graph_time_us(body, device, stream, reps) / len(copies)
            tops = 2.0 * M * N * K / (us * 1e-6) / 1e12
            bound, frac = roofline(2.0 * M * N * K, nbytes, us, hbm_gbs, int8_peak_tops)
            row[f"{key}_us"] = round(us, 2)
            row[f"{key}_TOPS"] = round(tops, 2)
            row[f"{key}_frac"] = round(frac, 4)
            row["bound"] = bound
        del x, xq, xs, y
        return row

    def weights(N, K, gs, std):
        w = inputs.weights(N, K, std=std, seed=inputs.layer_seed("sweep-w", N, K), device=device)
        wp, ws = flexq.quantize_weight(w, gs)
        del w
        n = max(2, int((400 << 20) // wp.numel()) + 1)
        return wp, ws, [(wp, ws)] + [(wp.clone(), ws.clone()) for _ in range(n - 1)]

    out = {"13b_w6a8": [], "sweep_8192": []}
    for N, K in [(5120, 5120), (13824, 5120), (5120, 13824)]:
        wp, ws, copies = weights(N, K, 128, 0.02)
        for M in (1, 64, 4096):
            out["13b_w6a8"].append(case(M, N, K, 128, 8, wp, ws, copies))
        del copies
        torch.cuda.empty_cache()
    sweep_m = (1, 4096) if subset else tuple(inputs.SWEEP_M)
    for gs in (32, 64, 128, 256):
        wp, ws, copies = weights(8192, 8192, gs, 0.02)
        for bits in (6, 8):
            for M in sweep_m:
                out["sweep_8192"].append(case(M, 8192, 8192, gs, bits, wp, ws, copies))
        del copies
        torch.cuda.empty_cache()
    return out


def layout_ab(device, hbm_gbs, ms=(1, 16)):
    """A/B of the two packed-weight layouts at decode sizes on the three
    LLaMA-2-70B layer shapes of the step: the byte-aligned device form and
    the "4+2" bit-plane form hold the same codes and run the same kernels,
    only the unpack differs.  Per (shape, M, layout): the GEMM alone on
    quantized activations and the whole layer, device time per call from a
    CUDA graph rotating over enough weight copies to exceed L2, and the
    fraction of the HBM roofline; `ratio` = byte-aligned time / 4+2 time
    (above 1: 4+2 faster)."""
    import torch
    from bit_group_quantized_flexq_b200 import flexq, inputs
    stream = torch.cuda.Stream(device)
    rows = []
    for (N, K, bits) in ((8192, 8192, 6), (28672, 8192, 6), (8192, 28672, 8)):
        w = inputs.weights(N, K, std=WEIGHT_STD, seed=inputs.layer_seed("ab", N, K), device=device)
        n_copies = max(2, int((400 << 20) // (N * K * 3 // 4)) + 1)
        packed = {lay: [flexq.quantize_weight(w, GS, layout=lay) for _ in range(n_copies)]
                  for lay in (flexq.LAYOUT_BYTE_ALIGNED, flexq.LAYOUT_4_2)}
        del w
        for M in ms:
            x = inputs.activations(M, K, outlier_frac=OUTLIER_FRAC, outlier_scale=OUTLIER_SCALE,
                                   seed=inputs.layer_seed("ab-x", M, K)).to(device)
            xq, xs = flexq.quantize_act(x, GS, bits)
            y = torch.empty(M, N, dtype=torch.float16, device=device)
            row = {"M": M, "N": N, "K": K, "act_bits": bits}
            for lay, name in ((flexq.LAYOUT_BYTE_ALIGNED, "byte_aligned"), (flexq.LAYOUT_4_2, "4+2")):
                cps = packed[lay]

                def g_body(cps=cps, lay=lay):
                    for wp, ws in cps:
                        flexq.gemm(xq, xs, wp, ws, N, GS, bits, out=y, layout=lay)

                def l_body(cps=cps, lay=lay):
                    for wp, ws in cps:
                        flexq.linear(x, wp, ws, N, GS, bits, out=y, layout=lay)
                g_us = _graph_time_us(g_body, device, stream, 3) / len(cps)
                l_us = _graph_time_us(l_body, device, stream, 3) / len(cps)
                row[f"{name}_gemm_us"] = round(g_us, 2)
                row[f"{name}_gemm_frac_hbm"] = round(gemm_bytes(M, N, K) / (g_us * 1e-6) / 1e9 / hbm_gbs, 4)
                row[f"{name}_linear_us"] = round(l_us, 2)
            row["ratio_gemm"] = round(row["byte_aligned_gemm_us"] / row["4+2_gemm_us"], 4)
            row["ratio_linear"] = round(row["byte_aligned_linear_us"] / row["4+2_linear_us"], 4)
            rows.append(row)
            del x, xq, xs, y
        del packed
        torch.cuda.empty_cache()
    return rows


def int8_library_context(W, device, M, reps=20):
    """Context only, never the target: the library int8 GEMM (torch._int_mm,
    plain W8A8 without group scales) on this GPU at the dominant M's shapes,
    and its rate on an 8192^3 problem (an on-box int8 tensor figure to set
    beside the nominal ratio used for the roofline)."""
    import torch

    def time_mm(m, n, k):
        a = torch.randint(-127, 128, (m, k), dtype=torch.int8, device=device)
        b = torch.randint(-127, 128, (n, k), dtype=torch.int8, device=device).t()
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize(device)
        us = e0.elapsed_time(e1) * 1e3 / reps
        return round(us, 2), round(2.0 * m * n * k / (us * 1e-6) / 1e12, 1)

    try:
        shapes = []
        for (name, N, K, _, _, _, _) in W.w:
            us, tops = time_mm(M, N, K)
            shapes.append({"layer": name, "M": M, "N": N, "K": K, "us": us, "TOPS": tops})
        us, tops = time_mm(8192, 8192, 8192)
        return {"kernel": "torch._int_mm (int8 x int8 -> int32, no group scales)",
                "layers": shapes, "int8_8192_cube_TOPS": tops}
    except (RuntimeError, AttributeError) as exc:       # not available in this torch build
        return {"unavailable": str(exc).splitlines()[0][:200]}


def gpu_local_cpus(index):
    """The host CPUs NVML reports as local to GPU `index` (its NUMA node), or
    None when NVML cannot tell."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(index)
        ncpu = os.cpu_count() or 1
        words = pynvml.nvmlDeviceGetCpuAffinity(h, (ncpu + 63) // 64)
        cpus = {64 * w + b for w, mask in enumerate(words) for b in range(64) if (mask >> b) & 1}
        return cpus or None
    except Exception:
        return None


def run_e2e(W, args, device, world):
    """Pins this process to the GPU's local CPUs while the host buffers are
    allocated and the copies run (so the pinned pages sit on the GPU's NUMA
    node), then restores the previous affinity."""
    saved = os.sched_getaffinity(0)
    local = gpu_local_cpus(device.index if device.index is not None else 0)
    pinned = sorted(local & saved) if local else []
    if pinned:
        os.sched_setaffinity(0, pinned)
    try:
        res = _run_e2e(W, args, device, world)
    finally:
        os.sched_setaffinity(0, saved)
    res["host_cpus"] = (f"{len(pinned)} CPUs local to the GPU (NVML)" if pinned
                        else "unpinned (NVML gave no CPU affinity)")
    return res


def _run_e2e(W, args, device, world):
    """The same metric through the public API with host buffers: every step
    copies each layer's FP16 input from pinned host memory and each output
    back to pinned host memory.  Copies in, layer calls and copies out run
    on three streams joined by events (each layer waits for its input, each
    copy out for its layer; a buffer is refilled only after its last reader
    of the previous step), so the two copy directions and the kernels
    overlap as the hardware's copy engines allow."""
    import torch
    from bit_group_quantized_flexq_b200 import flexq
    keys = [(M, layer) for M in W.ms for layer in W.w]
    hx = {(M, l[0]): W.x[(M, l[4])].cpu().pin_memory() for M, l in keys}
    hy = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in W.y.items()}
    dx = {(M, l[0]): torch.empty_like(W.x[(M, l[4])]) for M, l in keys}
    h2d = sum(v.numel() * 2 for v in hx.values())
    d2h = sum(v.numel() * 2 for v in W.y.values())
    s_in, s_c, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    done_in = {k: ev() for k in hx}
    done_c = {k: ev() for k in hx}
    done_out = {k: ev() for k in hx}
    started = [False]

    def step():
        for M, (name, N, K, bits, site, wp, ws) in keys:
            k = (M, name)
            if started[0]:
                s_in.wait_event(done_c[k])        # the previous step's layer has read dx
            with torch.cuda.stream(s_in):
                dx[k].copy_(hx[k], non_blocking=True)
                done_in[k].record(s_in)
            s_c.wait_event(done_in[k])
            if started[0]:
                s_c.wait_event(done_out[k])       # the previous step's copy out has read y
            with torch.cuda.stream(s_c):
                flexq.linear(dx[k], wp, ws, N, GS, bits, out=W.y[k])
                done_c[k].record(s_c)
            s_out.wait_event(done_c[k])
            with torch.cuda.stream(s_out):
                hy[k].copy_(W.y[k], non_blocking=True)
                done_out[k].record(s_out)
        started[0] = True

    main = torch.cuda.current_stream(device)

    def run(n):
        for stream in (s_in, s_c, s_out):
            stream.wait_stream(main)
        for _ in range(n):
            step()
        for stream in (s_in, s_c, s_out):
            main.wait_stream(stream)

    run(args.warmup)
    torch.cuda.synchronize(device)
    barrier(device)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(main)
    run(args.steps)
    t1.record(main)
    torch.cuda.synchronize(device)
    t_max = max_over_ranks(t0.elapsed_time(t1) / 1e3, device)
    ops = step_ops(W.ms, W.layers)
    return {"value": round(aggregate(ops * args.steps, world, t_max) / 1e12, 3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(t_max * 1e3 / args.steps, 4),
            "streams": "copies in, layer calls and copies out on three streams"}


# ------------------------------------------------------- CPU oracle arm ----
def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OracleSample:
    """A bounded sample of the step for the CPU oracle: for every M of the
    step, `rows` seeded rows of that M's activations (all of them where M is
    smaller) through all five layers.  The oracle's cost is linear in the
    rows, so a larger M's time is the sample's time scaled by M / rows
    (extrapolated); the weights are quantized once, outside the timing, as
    the method does offline."""

    def __init__(self, rows=1):
        from bit_group_quantized_flexq_b200 import inputs
        from oracle import flexq_oracle as orc
        self.orc = orc
        self.ms, self.layers = workload_shapes()
        self.rows = rows
        self.w = []
        for name, N, K, bits, site in self.layers:
            w16 = inputs.weights(N, K, std=WEIGHT_STD,
                                 seed=inputs.layer_seed("70b", name)).numpy()
            qw, sw = orc.quantize_weight(w16, GS)      # offline step, not timed
            self.w.append((name, N, K, bits, site, qw, sw))
        self.x = {}
        for M in self.ms:
            r = min(M, rows)
            for site, K in {l[4]: l[2] for l in self.layers}.items():
                x = inputs.activations(r, K, outlier_frac=OUTLIER_FRAC,
                                       outlier_scale=OUTLIER_SCALE,
                                       seed=inputs.layer_seed("70b-x-cpu", M, site))
                self.x[(M, site)] = x.numpy()
        self.jobs = [(M, l) for M in self.ms for l in self.w]
        # operations the sample computes, and those of the M it stands for
        self.ops_sample = sum(2.0 * min(M, rows) * l[1] * l[2] for M, l in self.jobs)
        self.ops_full = step_ops(self.ms, self.layers)

    def job(self, item):
        M, (name, N, K, bits, site, qw, sw) = item
        orc = self.orc
        qa, sa = orc.quantize_act(self.x[(M, site)], GS, bits)
        orc.to_fp16(orc.gemm_fp64(qa, sa, qw, sw, GS))

    def step(self, threads=1):
        if threads <= 1:
            for item in self.jobs:
                self.job(item)
            return
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(self.job, self.jobs))


def run_cpu_baseline(budget_s=30.0):
    """The oracle on the host cores: one pass of the sample on one thread and
    passes on every core (numpy releases the GIL inside its array loops, so
    threads run the (M, layer) jobs in parallel)."""
    s = OracleSample(rows=1)
    cores = os.cpu_count() or 1
    t0 = time.perf_counter()
    s.step(1)
    dt1 = time.perf_counter() - t0
    n, t0 = 0, time.perf_counter()
    while True:
        s.step(cores)
        n += 1
        if time.perf_counter() - t0 > budget_s / 3 or n >= 3:
            break
    dtn = (time.perf_counter() - t0) / n
    return {"value": round(s.ops_sample / dtn / 1e12, 9), "unit": UNIT, "cores": cores,
            "kind": "oracle", "cpu_model": cpu_model(),
            "one_thread": {"value": round(s.ops_sample / dt1 / 1e12, 9), "cores": 1},
            "step_s_extrapolated": round(dtn * s.ops_full / s.ops_sample, 1),
            "sample": (f"oracle (numpy: int64 group dot products + FP64 rescale, activation "
                       f"quantization included) on one seeded row of each M in {s.ms} through "
                       f"all five layers ({s.ops_sample / 1e9:.1f} GOP); {n} passes of "
                       f"{dtn:.2f} s on {cores} threads, {dt1:.2f} s on one; the whole step "
                       f"scales linearly in the rows (extrapolated)")}


def run_reference(args, rank, world):
    if rank != 0:
        return
    s = OracleSample(rows=1)
    cores = os.cpu_count() or 1
    for _ in range(args.warmup):
        s.step(cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s.step(cores)
    dt = time.perf_counter() - t0
    value = s.ops_sample * args.steps / dt / 1e12
    ms, layers = workload_shapes()
    sample = (f"each step: one seeded row of each M in {s.ms} through all five layers "
              f"({s.ops_sample / 1e9:.1f} GOP), on {cores} threads")
    out = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 9), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int64", "data": "synthetic",
        "config": {"workload": workload_name(ms, layers), "sample": sample},
        "cpu_baseline": {"value": round(value, 9), "unit": UNIT, "cores": cores,
                         "kind": "oracle", "cpu_model": cpu_model(), "sample": sample},
        "e2e": {"value": round(value, 9), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ main ---
def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["flexq", "reference"], default="flexq")
    p.add_argument("--ms", type=lambda s: [int(v) for v in s.split(",")], default=None,
                   help="subset of M values (profiling)")
    p.add_argument("--layers", type=lambda s: s.split(","), default=None,
                   help="subset of layer names (profiling)")
    p.add_argument("--no-graph", dest="graph", action="store_false")
    p.add_argument("--no-e2e", dest="e2e", action="store_false")
    p.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    p.add_argument("--no-diag", dest="diag", action="store_false")
    p.add_argument("--cpu-budget-s", type=float, default=30.0)
    p.add_argument("--sweep", action="store_true",
                   help="measure the 13B W6A8 layers and the N = K = 8192 group-size sweep "
                        "instead of the step (one JSON line)")
    a = p.parse_args(argv)
    if a.warmup < 3 and a.impl == "flexq" and not (a.ms or a.layers):
        p.error("--warmup must be >= 3")
    return a


def main(argv=None):
    args = parse_args(argv)
    rank, world = dist_init("nccl" if args.impl == "flexq" else "gloo")
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.sweep:
            import torch
            _, _, local = dist_env()
            device = torch.device("cuda", local)
            torch.cuda.set_device(device)
            peaks, src = measured_peaks()
            res = run_sweep(device, peaks["hbm_gbs"], peaks["bf16_tflops"] * INT8_OVER_BF16)
            if rank == 0:
                print(json.dumps({"sweep": res, "peaks": src,
                                  "int8_peak_tops": peaks["bf16_tflops"] * INT8_OVER_BF16,
                                  "hbm_gbs": peaks["hbm_gbs"]}), flush=True)
        else:
            run_flexq(args, rank, world)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
