"""Benchmark of the fused MoE expert layer on B200s: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one full forward of the layer (route -> permute -> gate/up GEMM with the
activation -> down GEMM -> combine) over one batch of seeded synthetic inputs. The
default workload is the largest one-GPU workload, the DeepSeek-shaped BF16 prefill
(T=8192, H=7168, I=2048, E=256 plus 16 redundant slots, top-8). With N GPUs (torchrun,
one process per GPU; `--gpus N` alone relaunches itself that way) every rank runs its
own replica of the layer on its own batch: there is no data-path collective ("weak"
scaling); the time is the max over ranks of the device time.

value   tokens/s over all ranks, inputs resident in HBM, CUDA events on the stream.
e2e     the same through the public call with pinned host buffers: every step copies x
        and the router logits host -> device and the output device -> host inside the
        timed region, double-buffered on two copy streams so that the copies of one step
        overlap the layer of the previous one.
roofline  the dominant kernel (the gate/up grouped GEMM), algorithmic FLOPs or bytes per
        launch over its event-timed duration, against MEASURED_PEAKS.json.
cpu_baseline  the CPU oracle on a bounded token sample, rank 0, N = 1 only.

--impl reference times the CPU oracle alone (the only reference there is: the pages
describe closed or library kernels), rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "MoE layer tokens/s on 1 B200; grouped-GEMM TFLOP/s & HBM GB/s as % roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2 ** 20


# ---------------------------------------------------------------------------- accounting

def weight_bytes_per_row(ws: W.WeightSet) -> int:
    """Bytes of one weight row [N,K] including its scales and alpha."""
    b = ws.data[0].numel() * ws.data.element_size()
    if ws.scale is not None:
        b += ws.scale[0].numel()
    if ws.alpha is not None:
        b += 4
    return b


def segment_stats(cfg: W.MoEConfig, topk_ids: torch.Tensor, replica_src: torch.Tensor):
    """Non-empty weight rows and the largest segment of one step, from the top-k ids the
    library produced (bookkeeping for the roofline, outside the timed region): expert e
    with n_e assignments and R_e rows (itself plus its used replicas) fills min(n_e, R_e)
    rows, the largest holding ceil(n_e / R_e)."""
    n = torch.bincount(topk_ids.reshape(-1).long().cpu(), minlength=cfg.E).numpy()
    R = np.ones(cfg.E, dtype=np.int64)
    for s in replica_src.tolist():
        if s >= 0:
            R[s] += 1
    nonempty = int(np.minimum(n, R).sum())
    max_seg = int(np.max(-(-n // R))) if cfg.E else 0
    return nonempty, max_seg


def accounting(cfg: W.MoEConfig, inp: W.MoEInputs, nonempty: int, max_seg: int) -> dict:
    NvS = cfg.NvS
    wg, wu, wd = (weight_bytes_per_row(inp.w_gate), weight_bytes_per_row(inp.w_up),
                  weight_bytes_per_row(inp.w_down))
    # activation operand bytes per value as the GEMMs read them
    a_in = {0: 2.0, 1: 9.0 / 16.0, 2: 1.0 + 1.0 / 32.0}[cfg.act_quant]
    if cfg.wfmt == "mxfp4" and not cfg.act_quant:
        a_in = 2.0 + 1.0 / 32.0           # two e4m3 terms and a scale per 32 values
    # gate/up output: bf16 (BF16), f16 (NVFP4 weights, bf16 activations, SITU), the down
    # GEMM's e4m3 records (MXFP4), else fp32
    act_out = 2 if cfg.wfmt == "bf16" or (cfg.wfmt == "nvfp4" and cfg.act == "situ" and not cfg.act_quant) else 4
    if cfg.wfmt == "mxfp4":
        act_out = a_in
    fc1_flops = 4.0 * NvS * cfg.H * cfg.I
    fc2_flops = 2.0 * NvS * cfg.H * cfg.I
    fc1_bytes = nonempty * (wg + wu) + NvS * cfg.H * a_in + NvS * cfg.I * act_out
    fc2_bytes = nonempty * wd + NvS * cfg.I * a_in + NvS * cfg.H * 4
    bias_bytes = nonempty * (2 * cfg.I + cfg.H) * 4 if cfg.bias else 0
    if cfg.bias:
        # the epilogues read each non-empty expert's bias rows: gate and up, then down
        fc1_bytes += nonempty * 2 * cfg.I * 4
        fc2_bytes += nonempty * cfg.H * 4
    layer_bytes = nonempty * (wg + wu + wd) + bias_bytes + cfg.T * cfg.H * 2 * 2 + cfg.T * cfg.E * 4
    return dict(nonempty=nonempty, max_seg=max_seg,
                fc1_flops=fc1_flops, fc2_flops=fc2_flops, fc1_bytes=fc1_bytes, fc2_bytes=fc2_bytes,
                layer_flops=fc1_flops + fc2_flops, layer_bytes=layer_bytes,
                weight_bytes_total=nonempty * (wg + wu + wd))


def tensor_peak_ratio(cfg) -> tuple[float, str]:
    """Tensor peak of the path's MMA kind relative to the measured bf16 one (the nominal
    dense ratios: fp8 2x, fp4 4x bf16)."""
    if cfg.wfmt == "nvfp4" and cfg.act_quant == 1:
        return 4.0, "bf16 x 4 (kind::mxf4nvf4, the nominal fp4/bf16 ratio)"
    if cfg.wfmt == "mxfp4" and cfg.act_quant == 2:
        return 2.0, "bf16 x 2 (kind::mxf8f6f4, the nominal fp8/bf16 ratio)"
    if cfg.wfmt == "mxfp4":
        return 1.0, ("bf16 x 1 (kind::mxf8f6f4 at the fp8 rate, two e4m3 products per "
                     "multiply-add for the hi/lo activations)")
    return 1.0, "bf16 (kind::f16)"


def routing_config(cfg) -> dict:
    """The routing method in the config record (only when it is not the default)."""
    if cfg.routing == "renormalize":
        return {}
    return {"routing": cfg.routing, "n_group": cfg.n_group, "topk_group": cfg.topk_group,
            "routed_scaling_factor": cfg.routed_scaling_factor}


def act_config(cfg) -> dict:
    """SWIGLUOAI's parameters and the GEMM biases in the config record, when used."""
    d = {}
    if cfg.act == "swigluoai":
        d.update(swiglu_alpha=cfg.swiglu_alpha, swiglu_beta=cfg.swiglu_beta, swiglu_limit=cfg.swiglu_limit)
    if cfg.bias:
        d["gemm_biases"] = True
    return d


def compute_dtype(cfg) -> str:
    """The operand types the grouped GEMMs' tensor cores multiply."""
    if cfg.wfmt == "bf16":
        return "bf16"
    if cfg.wfmt == "nvfp4":
        return "nvfp4 x nvfp4 (e2m1, e4m3 block scales)" if cfg.act_quant == 1 else "f16"
    return "mxfp4 x mxfp8 (e2m1 x e4m3, e8m0 block scales)" + ("" if cfg.act_quant else ", activations as hi+lo")


def load_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            measured = json.load(f)
        missing = [k for k in FALLBACK_PEAKS if not isinstance(measured.get(k), (int, float))]
        peaks = {**FALLBACK_PEAKS, **{k: measured[k] for k in FALLBACK_PEAKS if k not in missing}}
        return peaks, "measured" + (f" (fallback for {', '.join(missing)})" if missing else "")
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak_key(clocks: dict) -> tuple[str, str]:
    """Which bf16 tensor peak bounds a GEMM timed inside the step loop: the sustained
    figure (a seconds-long cuBLAS loop under the power cap) when the clock record of the
    timed region shows the power cap active, else the burst figure."""
    if "sw_power_cap" in (clocks.get("reasons") or []):
        return "bf16_tflops_sustained", "sustained: sw_power_cap active in the timed region"
    return "bf16_tflops", "burst"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for name in ("gemm.cu", "common.cuh", "internal.h"):
        with open(os.path.join(ROOT, "mixture_experts_layer_21_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str) -> float | None:
    """DRAM bytes per launch of the gate/up GEMM from the committed ncu summary, if the
    summary was taken on the kernel source as it is now; else None."""
    p = os.path.join(ROOT, "profiles", f"grouped_gemm_fc1_{workload}.md")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha") != kernel_source_sha():
        return None
    try:
        return float(vals["dram_bytes_per_launch_full"])
    except (KeyError, ValueError):
        return None


def needs_l2_flush(weight_bytes_touched: float) -> bool:
    """A step whose weights fit in L2 would find them there on the next step."""
    return weight_bytes_touched <= L2_BYTES


def config_record(cfg, weight_bytes_touched: float) -> dict:
    """The workload's record, the same in both arms: its shapes and modes, and how the L2 is
    handled between timed steps (not flushed when the weights a step touches exceed it, else
    flushed by a 2 x L2 write between individually timed steps)."""
    l2 = (f"flushed between steps: weights touched per step {weight_bytes_touched / 1e6:.1f} MB "
          f"<= L2 {L2_BYTES / 2 ** 20:.0f} MiB" if needs_l2_flush(weight_bytes_touched) else
          f"no flush: weights touched per step {weight_bytes_touched / 1e9:.2f} GB > L2 {L2_BYTES / 2 ** 20:.0f} MiB")
    return {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "B": cfg.B,
            "topk": cfg.topk, "act": cfg.act, "weights": cfg.wfmt, "act_quant": cfg.act_quant,
            **routing_config(cfg), **act_config(cfg), "l2": l2}


# ---------------------------------------------------------------------------- ranks

def reduce_max(v: float, world: int, device) -> float:
    """Max of a per-rank value over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank runs its own replica on its own batch."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            p = torch.cuda.get_device_properties(index)
            ids = [getattr(p, n, None) for n in ("pci_domain_id", "pci_bus_id", "pci_device_id")]
            if all(isinstance(v, int) for v in ids):
                bus = "%08X:%02X:%02X.0" % tuple(ids)   # NVML wants the string form
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            else:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML unavailable: report it
            self.err = str(e)
        self.period = period_s
        self.samples = []
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = self._reasons(self.h)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((mhz, reasons, util))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self) -> dict:
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        busy = [s for s in self.samples if s[2] > 0] or self.samples
        mhz = [s[0] for s in busy]
        reasons = set()
        for _, r, _ in busy:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(busy), "source": "nvml"}


# ---------------------------------------------------------------------------- CPU oracle

def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(cfg, inp, tokens):
    from oracle import moe_oracle as O
    t0 = time.perf_counter()
    bias = inp.extra.get("routing_bias")
    O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                  inp.w_down, tokens=tokens, routing_bias=None if bias is None else bias.numpy(),
                  biases=inp.extra.get("biases"))
    return time.perf_counter() - t0


def default_sample(cfg) -> int:
    """Token sample for one oracle call: 1.5e12 FLOPs of the layer, about 10-15 s of fp64
    work on the GPU host's 16 cores (measured: 1.5e11 took 1.3 s)."""
    flops_per_token = 6.0 * cfg.topk * cfg.H * cfg.I
    return int(max(1, min(cfg.T, 1.5e12 // flops_per_token)))


# ---------------------------------------------------------------------------- arms

def kernel_launches(cfg) -> int:
    # route and permutation (one kernel for at most 256 tokens with the default routing; else
    # the routing, then the count, scan and scatter, or one kernel for at most 256 tokens),
    # gate/up GEMM, down GEMM, combine
    if cfg.T <= 256:
        n = (1 if cfg.routing == "renormalize" else 2) + 1 + 1 + 1
    else:
        n = 1 + 3 + 1 + 1 + 1
    # the gate/up operand in segment order: a gather (BF16; NVFP4 weights with bf16
    # activations, as f16) or one staging / quantisation pass over the gathered rows (MXFP4;
    # NVFP4 activations when H % 256 == 0, else quantisation then a gather)
    n += 2 if (cfg.wfmt == "nvfp4" and cfg.act_quant == 1 and cfg.H % 256) else 1
    # the down operand: a row pass for NVFP4 weights (NVFP4 quantisation, or f16 staging
    # unless SITU bounds h); the MXFP4 gate/up epilogue writes its records itself
    if cfg.wfmt == "nvfp4" and (cfg.act_quant == 1 or cfg.act != "situ"):
        n += 1
    return n


def roofline_records(cfg, acc: dict, fc1_ms: float, clocks: dict, traffic) -> tuple[dict, float]:
    """The gate/up GEMM's roofline record (its algorithmic FLOPs or bytes over its measured
    time, against the bound that is larger) and the layer's roofline time in seconds."""
    peaks, peak_src = load_peaks()
    tensor_mult, tensor_note = tensor_peak_ratio(cfg)
    tensor_key, tensor_regime = tensor_peak_key(clocks)
    tensor_peak = peaks[tensor_key] * tensor_mult
    t_fc1_tensor = acc["fc1_flops"] / (tensor_peak * 1e12)
    t_fc1_hbm = acc["fc1_bytes"] / (peaks["hbm_gbs"] * 1e9)
    if t_fc1_tensor >= t_fc1_hbm:
        ach = acc["fc1_flops"] / (fc1_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": ach / tensor_peak}
    else:
        ach = acc["fc1_bytes"] / (fc1_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"]}
    kname = "grouped GEMM gate+up (fused activation" + (", biases)" if cfg.bias else ")")
    roof.update({"traffic": traffic, "kernel": kname,
                 "algorithmic_flops": acc["fc1_flops"], "algorithmic_bytes": acc["fc1_bytes"],
                 "kernel_ms": fc1_ms,
                 "peak_source": f"{peak_src} peaks: HBM {peaks['hbm_gbs']:.0f} GB/s (copy); bf16 tensor "
                                f"{peaks[tensor_key]:.0f} TFLOP/s ({tensor_regime}); this path's tensor peak "
                                f"= {tensor_note}"})
    t_layer_roof = max(acc["layer_flops"] / (tensor_peak * 1e12),
                       acc["layer_bytes"] / (peaks["hbm_gbs"] * 1e9))
    return roof, t_layer_roof


def run_ours(args, cfg, rank, world):
    import mixture_experts_layer_21_b200 as m
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = W.gen_inputs(cfg)
    ws = [m.Weight.from_host(w, dev) for w in (inp.w_gate, inp.w_up, inp.w_down)]
    bias = inp.extra.get("routing_bias")
    layer = m.MoEForward(*ws, cfg.E, cfg.topk, cfg.B,
                         inp.replica_src.to(dev) if cfg.B else None, cfg.act, cfg.situ_alpha,
                         cfg.situ_beta, cfg.act_quant, True, T_max=cfg.T, routing=cfg.routing,
                         routing_bias=None if bias is None else bias.to(dev), n_group=cfg.n_group,
                         topk_group=cfg.topk_group, routed_scaling_factor=cfg.routed_scaling_factor,
                         swiglu_alpha=cfg.swiglu_alpha, swiglu_beta=cfg.swiglu_beta, swiglu_limit=cfg.swiglu_limit,
                         biases=tuple(b.float().to(dev) for b in inp.extra["biases"]) if cfg.bias else None)
    x_d, l_d = inp.x.to(dev), inp.logits.to(dev)
    out_d = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    K, Wm = args.steps, args.warmup

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
            torch.cuda.synchronize()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, world, dev)

    ids_d = torch.empty(cfg.T, cfg.topk, dtype=torch.int32, device=dev)
    for _ in range(Wm):
        layer(x_d, l_d, out=out_d, topk_ids=ids_d)
    assert layer.device_error() == 0, "device error in warm-up"
    acc = accounting(cfg, inp, *segment_stats(cfg, ids_d, inp.replica_src))

    # ---- device-resident timed region. Only the two events around the gate/up GEMM are
    # recorded (on the launching stream): every other kernel boundary keeps its
    # programmatic-dependent-launch overlap.
    nst = m.MOE_FWD_STAGE_EVENTS

    def new_events():
        row = [torch.cuda.Event(enable_timing=True) for _ in range(nst)]
        for e in row:
            e.record(stream)  # creates the handle
        return row

    fc1_evs = [new_events() for _ in range(K)]
    flush = needs_l2_flush(acc["weight_bytes_total"])
    scrub = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if flush else None
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record(stream)
        for i in range(K):
            ev = fc1_evs[i]
            if flush:                     # outside the step's own events
                scrub.fill_(float(i))
                step_evs[i][0].record(stream)
            layer(x_d, l_d, out=out_d, stage_events=[None, None, ev[2], ev[3], None, None, None])
            if flush:
                step_evs[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    if flush:
        ms_total = max_over_ranks(sum(a.elapsed_time(b) for a, b in step_evs))
    else:
        ms_total = max_over_ranks(t0.elapsed_time(t1))
    fc1_ms = float(np.mean([fc1_evs[i][2].elapsed_time(fc1_evs[i][3]) for i in range(K)]))
    assert layer.device_error() == 0, "device error in timed region"

    # ---- stage breakdown (separate pass, all seven events; not part of the value)
    br_evs = [new_events() for _ in range(min(K, 10))]
    for row in br_evs:
        layer(x_d, l_d, out=out_d, stage_events=row)
    torch.cuda.synchronize()
    stage_ms = np.array([[row[j].elapsed_time(row[j + 1]) for j in range(nst - 1)] for row in br_evs]).mean(axis=0)

    # ---- end to end through the public call, host buffers
    e2e = None
    if not args.no_e2e:
        # Two device buffer sets: step i copies its inputs into set i % 2 on the H2D stream
        # while the layer of step i - 1 runs, and its output leaves on the D2H stream while
        # step i + 1 runs. Events order each buffer's reuse.
        x_h = inp.x.pin_memory()
        l_h = inp.logits.pin_memory()
        o_h = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        xs = [x_d, torch.empty_like(x_d)]
        ls = [l_d, torch.empty_like(l_d)]
        outs = [out_d, torch.empty_like(out_d)]
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        loaded, computed, drained = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        used = [False, False]

        def e2e_step(i):
            b = i % 2
            with torch.cuda.stream(h2d):
                if used[b]:
                    h2d.wait_event(computed[b])           # the layer of step i-2 read this set
                xs[b].copy_(x_h, non_blocking=True)
                ls[b].copy_(l_h, non_blocking=True)
                loaded[b].record(h2d)
            stream.wait_event(loaded[b])
            if used[b]:
                stream.wait_event(drained[b])             # step i-2's output has left
            layer(xs[b], ls[b], out=outs[b])
            computed[b].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(computed[b])
                o_h[b].copy_(outs[b], non_blocking=True)
                drained[b].record(d2h)
            used[b] = True

        for i in range(Wm):
            e2e_step(i)
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        h2d.wait_event(a0)
        for i in range(Wm, Wm + K):
            e2e_step(i)
        for b in range(2):
            stream.wait_event(drained[b])
        a1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(a0.elapsed_time(a1))
        assert layer.device_error() == 0, "device error in the end-to-end pass"
        e2e = {"value": job_tokens_per_s(world, cfg.T, K, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": int(x_h.numel() * 2 + l_h.numel() * 4),
               "d2h_bytes_per_step": int(o_h[0].numel() * 2),
               "overlap": "double-buffered: H2D and D2H on their own streams overlap the layer"}

    clocks = clk.summary()
    ms_step = ms_total / K
    roof, t_layer_roof = roofline_records(cfg, acc, fc1_ms, clocks, profiled_traffic(args.config))
    tok_s = job_tokens_per_s(world, cfg.T, K, ms_total)

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        S = default_sample(cfg)
        toks = list(range(S))
        dt = oracle_sample(cfg, inp, toks)
        cpu = {"value": S / dt, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{S} of {cfg.T} tokens (routing and permutation of all {cfg.T}), "
                         f"fp64 NumPy, {dt:.1f} s"}

    res = {
        "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": compute_dtype(cfg),
        "data": "synthetic (seeded; random weights of the workload's shapes)",
        "config": config_record(cfg, acc["weight_bytes_total"]),
        "parallelism": f"replicas x{world} (one process per GPU, no data-path collective)",
        "workload_stats": {"nonempty_segments": acc["nonempty"], "max_segment": acc["max_seg"]},
        "roofline": roof,
        "layer_roofline": {"t_roof_ms": t_layer_roof * 1e3, "frac": t_layer_roof * 1e3 / ms_step,
                           "flops": acc["layer_flops"], "bytes": acc["layer_bytes"],
                           "tflops": acc["layer_flops"] / (ms_step * 1e-3) / 1e12,
                           "gbs": acc["layer_bytes"] / (ms_step * 1e-3) / 1e9},
        "stage_ms": {n: float(v) for n, v in zip(
            ["route", "permute_gather", "gate_up_gemm", "act_row_pass", "down_gemm", "combine"], stage_ms)},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": kernel_launches(cfg) * K,
        "clocks": clocks,
    }
    return res


def run_reference(args, cfg):
    """The CPU oracle on the host cores, each step a bounded token sample."""
    from oracle import moe_oracle as O

    inp = W.gen_inputs(cfg)
    bias = inp.extra.get("routing_bias")
    ids, _ = O.route(cfg, inp.logits.numpy(), None if bias is None else bias.numpy())
    acc = accounting(cfg, inp, *segment_stats(cfg, torch.from_numpy(ids), inp.replica_src))
    S = max(1, default_sample(cfg) // 4)
    K, Wm = args.steps, args.warmup
    # keep the whole run within a few minutes: shrink the sample if a calibration step is slow
    dt0 = oracle_sample(cfg, inp, list(range(min(S, cfg.T))))
    while S > 1 and dt0 * (K + Wm) > 240:
        S = max(1, S // 2)
        dt0 = oracle_sample(cfg, inp, list(range(min(S, cfg.T))))
    for i in range(Wm):
        oracle_sample(cfg, inp, [(i * S + j) % cfg.T for j in range(S)])
    t = 0.0
    for i in range(K):
        t += oracle_sample(cfg, inp, [((Wm + i) * S + j) % cfg.T for j in range(S)])
    val = S * K / t
    cores = cpu_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": 1,
        "steps": K, "warmup": Wm, "ms_per_step": t / K * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": config_record(cfg, acc["weight_bytes_total"]),
        "workload_stats": {"nonempty_segments": acc["nonempty"], "max_segment": acc["max_seg"]},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{S} tokens per step of {cfg.T} (routing of all), fp64 NumPy"},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="deepseek_prefill", choices=sorted(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (smaller cases for profiling; not a bench line)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E, with no redundant slots (smaller cases for profiling; not a bench line)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    cfg = W.CONFIGS[args.config]
    if args.tokens:
        cfg = cfg.with_(T=args.tokens, name=f"{cfg.name}_T{args.tokens}")
    if args.experts:
        cfg = cfg.with_(E=args.experts, B=0, B_used=0, name=f"{cfg.name}_E{args.experts}")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: relaunch under the torch launcher on this node
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr=127.0.0.1", f"--master-port={29500 + os.getpid() % 1000}",
               os.path.abspath(__file__), *(argv if argv is not None else sys.argv[1:])]
        os.execv(sys.executable, cmd)
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        return 2

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, cfg)), flush=True)
        return 0

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    try:
        res = run_ours(args, cfg, rank, world)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
