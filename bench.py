"""Benchmark of the GPTQ layer solver (Hessian + prepare + sweep + pack per layer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload opt175b]
    python bench.py --op hessian|prepare|quantize|layer --rows R --cols C --tokens T

One step quantizes every layer of the workload once: Hessian accumulation over
all calibration tokens, damping / ordering / inverse Cholesky factor, the
blocked column sweep, and bit packing.  The default workload is the largest that
fits one GPU: the OPT-175B-shaped layers (12288 x 12288, 49152 x 12288 and
12288 x 49152, 262144 calibration tokens each, 38.6 GB of fp16 activations).
Inputs are seeded synthetic tensors resident in HBM before timing; every layer's
calibration set is larger than L2, so no flush is needed between steps.

``--op`` times one stage of one layer on device-drawn inputs (X ~ N(0, 1) fp16,
W ~ N(0, 0.02^2) fp16) and prints one text line: a small fixed command to put
under a profiler (the untimed repeats are the warm-up a profiler skips with -s).

Multi-GPU: one process per GPU (torchrun).  The path has no exchange step, so
every rank quantizes its own replica of the workload (weak scaling); the only
collectives are the timing barrier and the max-over-ranks of the elapsed time.

Prints one JSON line on rank 0.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from post_weight_quantization_20_b200 import synthetic as S  # noqa: E402
from post_weight_quantization_20_b200.workloads import WORKLOADS  # noqa: E402

METRIC = "ms per linear layer quantized (H+Cholesky+sweep); GEMM TFLOP/s vs B200 peak"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of the Hessian launch at the given column count, per
# calibration token, or None when the kernel has changed since the counters were
# taken.  Estimated from two ncu captures of the CTA-pair kernel at 24576 columns
# (8192 and 16384 tokens): X's re-reads per flop at 16384 tokens (1.99 GB per TFLOP)
# times the launch's 6.33e14 flop, plus H's triangle read and written once
# (2 x 4.83 GB): 1271 GB per 262144-token launch.
HESSIAN_TRAFFIC = {"cols": 49152, "bytes_per_token": 1271e9 / 262144,
                   "how": "estimate scaled from ncu captures of the CTA-pair kernel at 24576 "
                          "columns, 8192 and 16384 tokens (X re-reads per flop, plus the H "
                          "triangle read and written once)"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


L2_BYTES = 126 * 2 ** 20


def l2_note(wl):
    """Whether each layer's calibration input alone outgrows the L2 (so that no
    flush is needed between timed steps)."""
    esize = {"f32": 4, "f16": 2, "bf16": 2}
    smallest = min(wl.tokens * l.cols * esize[wl.xdtype] for l in wl.layers)
    if smallest > L2_BYTES:
        return f"inputs larger than L2 (each layer's X >= {smallest / 2 ** 20:.0f} MiB > 126 MiB), no flush"
    return (f"inputs smaller than L2 (X {smallest / 2 ** 20:.1f} MiB), not flushed: "
            "a parity-size case, not a timing workload")


def workload_config(wl, n_gpus):
    shapes = ", ".join(f"{l.rows}x{l.cols}" for l in wl.layers)
    q = wl.quant[0]
    return {
        "workload": f"{wl.name}: W {shapes} {wl.wdtype}; X {wl.tokens} tokens x cols {wl.xdtype} "
                    f"({wl.xspec.dist}, {wl.xspec.outlier_frac:.0%} outlier channels x{wl.xspec.outlier_mult:g}); "
                    f"{q.label()} B={q.block_size} damp={q.damp}",
        "layers": len(wl.layers),
        "calib_tokens": wl.tokens,
        "l2": l2_note(wl),
        "parallelism": f"replicas x{n_gpus} (no data-path collective)",
    }


def gen_inputs(wl, seed=1234):
    out = []
    for l in wl.layers:
        W = S.gen_weight(l.rows, l.cols, wl.wdtype, wl.wspec, seed=seed, tag=l.tag)
        X = S.gen_activations(wl.tokens, l.cols, wl.xdtype, wl.xspec, seed=seed, tag=l.tag)
        out.append((l, W, X))
    return out


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled while a region runs.

    NVML is polled from a thread every few milliseconds (the timed regions are
    tens of milliseconds); without NVML, nvidia-smi is run in the background.
    The device is matched by PCI bus id, so CUDA_VISIBLE_DEVICES does not matter.
    """
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.005

    def __init__(self, device):
        import torch
        pr = torch.cuda.get_device_properties(device)
        self.bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        self.rows = []
        self.nv = None
        self.thread = None
        self.proc = None
        self.path = None
        self.stop_evt = None

    def _nvml_sample(self):
        nv, h, mx, bits = self.nv
        try:
            sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            return
        try:
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            reasons = [k for k, b in bits.items() if rs & b]
        except Exception:
            reasons = ["unreadable"]
        self.rows.append((sm, mx, reasons))

    def _nvml_loop(self):
        while not self.stop_evt.is_set():
            self._nvml_sample()
            self.stop_evt.wait(self.PERIOD_S)

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByPciBusId(self.bus.encode())
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            self.nv = (nv, h, float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)), bits)
            self._nvml_sample()                  # one sample at the start of the region
            if not self.rows:
                raise RuntimeError("NVML gave no clock reading")
            self.stop_evt = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
            self.rows = []
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.bus}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            self._nvml_sample()                      # and one at its end
            rows = self.rows
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            rows = []
            with open(self.path) as f:
                for line in f:
                    r = [p.strip() for p in line.split(",")]
                    if len(r) >= 9 and r[1].replace(".", "").isdigit():
                        rows.append((float(r[1]), float(r[2]) if r[2].replace(".", "").isdigit() else 0.0,
                                     [names[i] for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]]))
            os.unlink(self.path)
        else:
            return None
        if not rows:
            return None
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted({x for r in rows for x in r[2]}), "samples": len(rows)}


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(vals, world, device):
    """Each entry's value on the slowest rank (the job ends when its last rank does)."""
    if world == 1:
        return [float(v) for v in vals]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def status_over_ranks(local_status, world, device):
    """A device status word that is nonzero on any rank, on every rank (every rank
    takes this collective, so all of them raise together on an error)."""
    if world == 1:
        return int(local_status)
    import torch
    import torch.distributed as dist
    t = torch.tensor([int(local_status)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return int(local_status) or int(t.item())


def job_ms_per_layer(ms_timed, steps, layers_per_rank, world):
    """Whole-job ms per layer: every rank quantizes `layers_per_rank` layers per step
    (replicas, weak scaling), all finished within the slowest rank's time."""
    return ms_timed / steps / (layers_per_rank * world)


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    from post_weight_quantization_20_b200 import gptq as G

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    G.load_library()
    wl = WORKLOADS[args.workload]
    q = wl.quant[0]
    cfg = G.make_config(q.bits, q.group_size, q.sym, q.act_order, q.damp, q.block_size)
    host = gen_inputs(wl)
    torch_dt = {S.F32: torch.float32, S.F16: torch.float16, S.BF16: torch.bfloat16}

    def to_dev(a, dt):
        if dt == S.BF16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    def to_pinned(a, dt):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if dt == S.BF16 else torch.from_numpy(a)
        return t.pin_memory()

    stream = torch.cuda.current_stream(dev)
    # The layers run one after another on one stream, so they share one set of
    # Hessian, factor and workspace buffers sized for the largest layer; only
    # each layer's W, X and outputs are its own.
    Rmax = max(l.rows for l, _, _ in host)
    Cmax = max(l.cols for l, _, _ in host)
    shared = {
        "H": torch.empty(Cmax * Cmax, device=dev), "U": torch.empty(Cmax * Cmax, device=dev),
        "wsp": G.alloc_workspace(G.GPTQ_OP_PREPARE, Rmax, Cmax, cfg, dev),
        "wsq": torch.empty(max(G.gptq_workspace_size(G.GPTQ_OP_QUANTIZE, l.rows, l.cols, cfg)
                               for l, _, _ in host), dtype=torch.uint8, device=dev),
    }
    layers = []
    for l, W, X in host:
        R, C = l.rows, l.cols
        Gn = G.n_groups(C, cfg.group_size)
        b = {
            "R": R, "C": C,
            "W": to_dev(W, wl.wdtype), "X": to_dev(X, wl.xdtype),
            "H": shared["H"][:C * C].view(C, C), "U": shared["U"][:C * C].view(C, C),
            "perm": torch.empty(C, dtype=torch.int32, device=dev),
            "wsp": shared["wsp"],
            "wsq": shared["wsq"][:G.gptq_workspace_size(G.GPTQ_OP_QUANTIZE, R, C, cfg)],
            "codes": torch.empty(R, C, dtype=torch.uint8, device=dev),
            "scales": torch.empty(R, Gn, device=dev), "zeros": torch.empty(R, Gn, device=dev),
            "g_idx": torch.empty(C, dtype=torch.int32, device=dev),
            "losses": torch.empty(C, device=dev),
            "packed": torch.empty(R, G.packed_words(C, cfg.bits), dtype=torch.int32, device=dev),
            "status": torch.zeros(1, dtype=torch.int32, device=dev),
        }
        layers.append(b)

    hess_ev = []
    phase_ev = []   # per layer: events around hessian / prepare / quantize / pack

    def step(record=False):
        for b in layers:
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)] if record else None
            if record:
                ev[0].record(stream)
            G.gptq_hessian_accumulate(b["H"], 0, b["X"], b["status"], stream)
            if record:
                ev[1].record(stream)
                hess_ev.append((ev[0], ev[1], b["X"].shape[0], b["C"]))
            G.gptq_prepare(b["H"], cfg, b["U"], b["perm"], b["wsp"], b["status"], stream)
            if record:
                ev[2].record(stream)
            G.gptq_quantize_layer(b["W"], b["U"], b["perm"], cfg, b["codes"], b["scales"],
                                  b["zeros"], b["g_idx"], b["losses"], b["wsq"], b["status"], stream)
            if record:
                ev[3].record(stream)
            G.gptq_pack(b["codes"], cfg.bits, b["packed"], stream)
            if record:
                ev[4].record(stream)
                phase_ev.append((b["R"], b["C"], ev))

    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()

    def check_status(where):
        # a device condition (a bounded wait that gave up, a non-PD pivot) makes the
        # kernels finish early, so the run's times would not be of the whole work;
        # every rank takes the same collective here and raises together
        st = 0
        for b in layers:
            st |= int(b["status"].item())
        st = status_over_ranks(st, world, dev)
        if st:
            raise RuntimeError(f"device status {G.status_names(st)} {where}")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    check_status("after the warm-up steps")

    clocks = ClockSampler(dev)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    launches0 = G.gptq_launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step(record=True)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    launches = G.gptq_launch_count() - launches0
    barrier()
    cl = clocks.stop()
    check_status("in the timed steps")
    ms = t0.elapsed_time(t1)
    hess_ms = sum(a.elapsed_time(b) for a, b, _, _ in hess_ev)
    # per phase, summed over the layers of one step, and each phase's useful
    # flop rate (Hessian N C (C+1); Cholesky + triangular inverse 2/3 C^3; lazy
    # trailing update R C^2)
    names = ("hessian", "prepare", "quantize", "pack")
    tot = {n: 0.0 for n in names}
    flop = {"hessian": 0.0, "prepare": 0.0, "quantize": 0.0}
    for (R_, C_, ev), (_, _, m, _) in zip(phase_ev, hess_ev):
        for i, n in enumerate(names):
            tot[n] += ev[i].elapsed_time(ev[i + 1])
        flop["hessian"] += float(m) * C_ * (C_ + 1)
        flop["prepare"] += 2.0 * C_ ** 3 / 3.0
        flop["quantize"] += float(R_) * C_ * C_
    basis = {"hessian": "N*C*(C+1)", "prepare": "2/3*C^3",
             "quantize": "R*C^2 (lazy trailing update; the phase also runs the sweep)"}
    phases = {}
    for n in names:
        phases[n] = {"ms_per_step": tot[n] / args.steps}
        if n in flop and tot[n] > 0:
            phases[n]["tflops"] = flop[n] / (tot[n] * 1e-3) / 1e12
            phases[n]["flop"] = basis[n]
    hess_flop = sum(float(m) * C * (C + 1) for _, _, m, C in hess_ev)
    n_hess = len(hess_ev)

    stored = stored_form_product(G, layers, cfg, dev, stream, args)
    group = shared_input_group(G, layers[0], wl, cfg, dev, stream, args, to_dev)

    # end to end through the public API from pinned host buffers; the device-resident
    # inputs and buffers of the timed steps are released first (the host path
    # allocates its own)
    n_layers_rank = len(layers)
    layers.clear()
    shared.clear()
    torch.cuda.empty_cache()
    pinned = [(l, to_pinned(W, wl.wdtype), to_pinned(X, wl.xdtype)) for l, W, X in host]
    h2d = sum(w.numel() * w.element_size() + x.numel() * x.element_size() for _, w, x in pinned)

    def e2e_step():
        outs = []
        for l, Wh, Xh in pinned:
            r = G.quantize_layer_host(Wh, Xh, cfg, device=dev)
            outs.append(r)
        return outs

    # two untimed steps: each step's pinned outputs stay alive while the next one
    # runs, so the caching host allocator holds two sets before the timed region
    outs = e2e_step()
    outs = e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_steps = max(1, min(args.steps, 5))
    for _ in range(e2e_steps):
        outs = e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    d2h = sum(o.nbytes for o in outs)
    e2e_status = 0
    for o_ in outs:
        e2e_status |= int(o_.status.item())
    if status_over_ranks(e2e_status, world, dev):
        raise RuntimeError(f"device status {G.status_names(e2e_status)} in the end-to-end steps")
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], world, dev)

    n_layers = len(layers) * world
    peaks = load_peaks()
    achieved = hess_flop / (hess_ms * 1e-3) / 1e12 if hess_ms > 0 else None
    # the Hessian runs inside a step of seconds at the power cap: the sustained peak
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    traffic = None
    if HESSIAN_TRAFFIC:
        toks = [m for _, _, m, C in hess_ev if C == HESSIAN_TRAFFIC["cols"]]
        if toks:
            traffic = HESSIAN_TRAFFIC["bytes_per_token"] * toks[0]
    out = {
        "metric": METRIC,
        "value": job_ms_per_layer(ms, args.steps, n_layers_rank, world),
        "unit": "ms",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; stands in for the pages' calibration text)",
        "config": workload_config(wl, world),
        "phases": phases,
        "hessian": {"ms_per_launch": hess_ms / max(n_hess, 1), "tflops": achieved,
                    "launches": n_hess},
        "roofline": {"bound": "tensor", "kernel": "hessian accumulate (X^T X)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                     "traffic_scope": (f"bytes per C={HESSIAN_TRAFFIC['cols']} launch: "
                                       f"{HESSIAN_TRAFFIC['how']}")
                     if traffic is not None else
                     "null: the kernel changed after its last ncu capture",
                     "peak_source": (f"{peaks['source']} bf16 dense, sustained (a seconds-long "
                                     f"loop at the power cap), as the Hessian runs inside a "
                                     f"step of seconds; burst {float(peaks['bf16_tflops']):g}")},
        "e2e": {"value": e2e_ms / n_layers_rank, "unit": "ms", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        "stored_form": stored,
        "shared_input_group": group,
        "gpu_launches": int(launches),
        "clocks": cl,
    }
    return out


# ----------------------------------------------------------------------------- stored form
def stored_form_product(G, layers, cfg, dev, stream, args):
    """The inference side of the quantized layers: Y = X Q^T for one decode token from
    each layer's packed codes (repacked to sweep order once), timed over all layers
    with CUDA events.  HBM-bound: per layer it reads R C b/8 bytes of codes and R G 8
    of grids (plus the token and the output)."""
    import torch
    peaks = load_peaks()
    items, nbytes = [], 0
    gen = torch.Generator(device=dev)
    gen.manual_seed(1)
    for b in layers:
        R, C = b["R"], b["C"]
        qp = torch.empty(R, G.sweep_words(C, cfg.bits), dtype=torch.int32, device=dev)
        G.gptq_repack_sweep_order(b["packed"], cfg.bits, b["perm"], qp, stream)
        x = torch.randn(1, C, device=dev, generator=gen).half()
        y = torch.empty(1, R, device=dev)
        items.append((qp, b["scales"], b["zeros"], b["perm"], x, y))
        nbytes += R * C * cfg.bits // 8 + b["scales"].numel() * 8 + C * 2 + R * 4
    reps = max(3, min(args.steps, 20))

    def run():
        for qp, sc, ze, pm, x, y in items:
            G.gptq_dequant_matmul(x, qp, sc, ze, cfg.bits, cfg.group_size, pm, y, stream=stream)
    for _ in range(3):
        run()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(reps):
        run()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / reps
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"op": f"Y = x Q^T, one fp16 token, from the packed {cfg.bits}-bit codes of every "
                  f"layer (sweep-order repack, fp32 sums)",
            "ms_per_step": ms, "bytes_per_step": int(nbytes), "achieved_gbs": gbs,
            "peak_gbs": float(peaks["hbm_gbs"]), "frac": gbs / float(peaks["hbm_gbs"]),
            "peak_source": f"{peaks['source']} HBM copy"}


# ----------------------------------------------------------------------------- shared input
def shared_input_group(G, b, wl, cfg, dev, stream, args, to_dev):
    """Layers that read the same input (the q, k and v projections of one attention
    block): one Hessian and one factorization, then one sweep per weight, against the
    same three layers quantized one by one.  The first layer of the workload and two
    more weights of its shape, drawn from the same distribution."""
    import torch
    R, C = b["R"], b["C"]
    l = wl.layers[0]
    Ws = [b["W"]] + [to_dev(S.gen_weight(R, C, wl.wdtype, wl.wspec, seed=1234, tag=l.tag + 500 + k),
                            wl.wdtype) for k in range(2)]

    def sweep(W):
        G.gptq_quantize_layer(W, b["U"], b["perm"], cfg, b["codes"], b["scales"], b["zeros"],
                              b["g_idx"], b["losses"], b["wsq"], b["status"], stream)
        G.gptq_pack(b["codes"], cfg.bits, b["packed"], stream)

    def factor():
        G.gptq_hessian_accumulate(b["H"], 0, b["X"], b["status"], stream)
        G.gptq_prepare(b["H"], cfg, b["U"], b["perm"], b["wsp"], b["status"], stream)

    def shared():
        factor()
        for W in Ws:
            sweep(W)

    def separate():
        for W in Ws:
            factor()
            sweep(W)

    reps = max(1, min(args.steps, 3))
    out = {}
    for name, fn in (("shared", shared), ("separate", separate)):
        fn()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(reps):
            fn()
        t1.record(stream)
        torch.cuda.synchronize(dev)
        out[name] = t0.elapsed_time(t1) / reps
    if int(b["status"].item()):
        raise RuntimeError(f"device status {G.status_names(int(b['status'].item()))} "
                           "in the shared-input group")
    return {"layers": f"3 x {R}x{C} reading one {wl.tokens}-token input",
            "ms_per_layer_shared": out["shared"] / 3, "ms_per_layer_separate": out["separate"] / 3}


# ----------------------------------------------------------------------------- oracle arm
# The float64 oracle cannot run a full-size layer in a bounded time (at 49152
# columns its factorization alone is ~3e14 flop and its matrices 19 GB each), so
# each step runs one sub-problem, drawn from the workload's largest layer, and
# every layer's time is extrapolated from it by each phase's work formula:
#   Hessian      SAMPLE_TOKENS tokens x SAMPLE_COLS columns; work N C^2, scaled by
#                (N / m) (C / Cs)^2;
#   prepare      damping, order and factor of that Cs x Cs Hessian; work C^3,
#                scaled by (C / Cs)^3;
#   sweep        SAMPLE_ROWS rows at Cs/2 and at Cs columns, fitted as a C + b C^2
#                (per-column vector work and the lazy trailing update) and
#                evaluated at C, scaled by R / r;
#   pack         r rows x Cs columns, scaled by (R / r)(C / Cs).
SAMPLE_TOKENS = 8192
SAMPLE_COLS = 3072
SAMPLE_ROWS = 768


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] + [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_sample(wl):
    """One sub-problem of the workload's largest layer: (layer, W sample r x Cs, X sample
    m x Cs, m, Cs, r)."""
    l = max(wl.layers, key=lambda x: x.rows * x.cols * x.cols)
    m = min(wl.tokens, SAMPLE_TOKENS)
    cs = min(l.cols, SAMPLE_COLS)
    r = min(l.rows, SAMPLE_ROWS)
    W = S.gen_weight(r, l.cols, wl.wdtype, wl.wspec, seed=1234, tag=l.tag)[:, :cs]
    X = S.gen_activations(m, l.cols, wl.xdtype, wl.xspec, seed=1234, tag=l.tag)[:, :cs]
    return l, np.ascontiguousarray(W), np.ascontiguousarray(X), m, cs, r


def oracle_phases(W, X, wl, q):
    """Seconds the oracle spends on the sample: Hessian, prepare, sweep at Cs/2 and at
    Cs columns, pack."""
    from oracle import gptq_ref as o
    t0 = time.perf_counter()
    H, n = o.hessian(S.to_f64(X, wl.xdtype))
    t1 = time.perf_counter()
    perm, Hp, U = o.prepare(H, q.damp, q.act_order)
    t2 = time.perf_counter()
    Wp = S.to_f64(W, wl.wdtype)[:, perm]
    half = max(1, W.shape[1] // 2)
    o.sweep(Wp[:, :half], U[:half, :half], q.bits, q.group_size, q.sym, q.block_size)
    t3 = time.perf_counter()
    res = o.sweep(Wp, U, q.bits, q.group_size, q.sym, q.block_size)
    t4 = time.perf_counter()
    o.pack(res["codes"], q.bits)
    t5 = time.perf_counter()
    return t1 - t0, t2 - t1, t3 - t2, t4 - t3, t5 - t4


def sweep_model(t_half, t_full, c_half, c_full, C):
    """Fit t(c) = a c + b c^2 through the two sweep samples (a, b >= 0) and evaluate it
    at C."""
    # solve [c1 c1^2; c2 c2^2] [a b]^T = [t1 t2]^T
    det = c_half * c_full ** 2 - c_full * c_half ** 2
    if det <= 0:
        return t_full * C / c_full
    a = (t_half * c_full ** 2 - t_full * c_half ** 2) / det
    b = (c_half * t_full - c_full * t_half) / det
    if a < 0 or b < 0:       # timing noise: keep the single-term fit that stays non-negative
        a, b = (t_full / c_full, 0.0) if b < 0 else (0.0, t_full / c_full ** 2)
    return a * C + b * C * C


def layer_ms_from_sample(times, l, wl, m, cs, r):
    """One full layer's oracle time (ms), extrapolated from the sample's phase times."""
    th, tp, ts1, ts2, tk = times
    C, R, N = l.cols, l.rows, wl.tokens
    half = max(1, cs // 2)
    total = (th * (N / m) * (C / cs) ** 2 + tp * (C / cs) ** 3 +
             sweep_model(ts1, ts2, half, cs, C) * (R / r) + tk * (R / r) * (C / cs))
    return total * 1e3


def cpu_step_ms_per_layer(wl, sample):
    """One oracle step: the sample timed once, every layer extrapolated from it; the
    mean over the workload's layers (ms per layer)."""
    _, W, X, m, cs, r = sample
    times = oracle_phases(W, X, wl, wl.quant[0])
    return sum(layer_ms_from_sample(times, l, wl, m, cs, r) for l in wl.layers) / len(wl.layers)


def cpu_sample_text(wl, sample):
    l, _, _, m, cs, r = sample
    return (f"per step one sub-problem of the {l.rows}x{l.cols} layer ({m} tokens, {cs} cols, "
            f"{r} rows of its inputs); every layer of the workload extrapolated from it by "
            f"each phase's work: Hessian x (N/m)(C/Cs)^2, prepare x (C/Cs)^3, sweep fitted as "
            f"a C + b C^2 from Cs/2 and Cs columns and x R/r, pack x (R/r)(C/Cs); float64 "
            f"NumPy oracle on host cores")


def run_cpu_baseline(wl):
    sample = cpu_sample(wl)
    v = cpu_step_ms_per_layer(wl, sample)
    return {"value": v, "unit": "ms per layer", "cores": blas_threads(), "kind": "oracle",
            "sample": "one step: " + cpu_sample_text(wl, sample)}


def run_reference(args):
    wl = WORKLOADS[args.workload]
    sample = cpu_sample(wl)
    for _ in range(args.warmup):
        cpu_step_ms_per_layer(wl, sample)
    v = sum(cpu_step_ms_per_layer(wl, sample) for _ in range(args.steps)) / max(args.steps, 1)
    cores = blas_threads()
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "ms", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v * len(wl.layers),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": workload_config(wl, 1),
            "cpu_baseline": {"value": v, "unit": "ms per layer", "cores": cores, "kind": "oracle",
                             "sample": cpu_sample_text(wl, sample)},
            "e2e": {"value": v, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- one stage
def run_op(args):
    """Time one stage of one layer on device-drawn inputs; one text line."""
    import torch
    from post_weight_quantization_20_b200 import gptq as G
    dev = torch.device("cuda", torch.cuda.current_device())
    G.load_library()
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    R, C, T = args.rows, args.cols, args.tokens
    X = torch.randn(T, C, device=dev, generator=gen).half()
    W = (0.02 * torch.randn(R, C, device=dev, generator=gen)).half()
    cfg = G.make_config(args.bits, args.group, act_order=args.act_order)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    H = torch.empty(C, C, device=dev)
    U = torch.empty(C, C, device=dev)
    perm = torch.empty(C, dtype=torch.int32, device=dev)
    wsp = G.alloc_workspace(G.GPTQ_OP_PREPARE, R, C, cfg, dev)
    G.gptq_hessian_accumulate(H, 0, X, status)
    if args.op == "hessian":
        def run():
            G.gptq_hessian_accumulate(H, 0, X, status)
        work = f"{float(T) * C * (C + 1) / 1e12:.4f} TFLOP per call"
    elif args.op == "prepare":
        def run():
            G.gptq_prepare(H, cfg, U, perm, wsp, status)
        work = f"{2.0 * C ** 3 / 3e12:.4f} TFLOP per call (2/3 C^3)"
    elif args.op == "dequant":
        # the stored form's product for args.tokens (<= 8) decode tokens on random codes
        Gn = G.n_groups(C, cfg.group_size)
        words = torch.randint(-2 ** 31, 2 ** 31 - 1, (R, G.sweep_words(C, cfg.bits)),
                              dtype=torch.int32, device=dev, generator=gen)
        sc = torch.rand(R, Gn, device=dev, generator=gen) * 0.01
        ze = torch.randint(0, 2 ** cfg.bits, (R, Gn), device=dev, generator=gen).float()
        pm = torch.randperm(C, device=dev, generator=gen).int()
        x = torch.randn(min(T, 8), C, device=dev, generator=gen).half()
        y = torch.empty(x.shape[0], R, device=dev)

        def run():
            G.gptq_dequant_matmul(x, words, sc, ze, cfg.bits, cfg.group_size, pm, y)
        nbytes = R * C * cfg.bits // 8 + R * Gn * 8 + x.numel() * 2 + y.numel() * 4
        work = f"{nbytes / 1e6:.1f} MB of codes, grids, tokens and outputs per call"
    elif args.op == "quantize":
        G.gptq_prepare(H, cfg, U, perm, wsp, status)
        Gn = G.n_groups(C, cfg.group_size)
        codes = torch.empty(R, C, dtype=torch.uint8, device=dev)
        scales = torch.empty(R, Gn, device=dev)
        zeros = torch.empty(R, Gn, device=dev)
        g_idx = torch.empty(C, dtype=torch.int32, device=dev)
        losses = torch.empty(C, device=dev)
        packed = torch.empty(R, G.packed_words(C, cfg.bits), dtype=torch.int32, device=dev)
        wsq = G.alloc_workspace(G.GPTQ_OP_QUANTIZE, R, C, cfg, dev)

        def run():
            G.gptq_quantize_layer(W, U, perm, cfg, codes, scales, zeros, g_idx, losses, wsq, status)
            G.gptq_pack(codes, cfg.bits, packed)
        work = f"sweep + lazy updates + pack, {float(R) * C * C / 1e12:.4f} TFLOP of update per call"
    else:
        def run():
            G.quantize_layer(W, X, cfg, check=False)
        work = "Hessian + prepare + sweep + pack, with their allocations"
    for _ in range(args.repeat):
        run()
    torch.cuda.synchronize(dev)
    G.check_status(status, args.op)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.repeat):
        run()
    e1.record()
    torch.cuda.synchronize(dev)
    G.check_status(status, args.op)
    ms = e0.elapsed_time(e1) / args.repeat
    print(f"op={args.op} rows={R} cols={C} tokens={T}: {ms:.3f} ms per call ({work})", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="opt175b", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default="step", choices=["step", "hessian", "prepare", "quantize",
                                                     "layer", "dequant"])
    ap.add_argument("--rows", type=int, default=768)
    ap.add_argument("--cols", type=int, default=3072)
    ap.add_argument("--tokens", type=int, default=16384)
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--bits", type=int, default=4)
    ap.add_argument("--group", type=int, default=128)
    ap.add_argument("--act-order", action="store_true")
    args = ap.parse_args()
    if args.op != "step":
        run_op(args)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    out = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = run_cpu_baseline(WORKLOADS[args.workload])
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
