#!/usr/bin/env python
"""Benchmark: GPTQ+QEP layers quantised per second on one Llama-2-7B-shaped layer.

One step = the whole per-layer path on one synthetic layer already resident in
HBM: H = 2 Xhat^T Xhat, the QEP correction with that H and GPTQ with packing,
through the library's one-call layer entry point (oc_quantize_layer, one
factorisation of the dampened Hessian).  The same layer through the three
separate calls (oc_hessian_accumulate, oc_qep_correct, oc_gptq_quantize) is
timed as well and reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun every rank quantises its own
layer (independent problems, no collective on the data path): weak scaling,
value = layers of all ranks / max-over-ranks device time.  ``--impl reference``
times the float64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPTQ+QEP layers quantized/sec (Llama-7B shapes, 4-bit g128); % of roofline"
UNIT = "layers/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SM_COUNT = 148
L2_BYTES = 126 * 1024 * 1024
CPU_SAMPLE_TOKENS = 16384
CPU_SAMPLE_ROWS = 2048
# The recorded DRAM traffic of the dominant kernel: dram__bytes_read.sum +
# dram__bytes_write.sum per launch from one ncu capture of a smaller case of the
# same workload, scaled to a full-size launch, with the SHA-256 of the kernel's
# source at capture time.  If the source has changed since, the traffic is
# reported as null.
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "atb16_q_proj_4096_traffic.json")
KERNEL_SOURCE = os.path.join(ROOT, "post_weight_quantization_07_b200", "csrc", "k_atb16.cu")


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


WORKLOAD_TITLES = {
    "layer_512": "single 512x512 linear layer",
    "q_proj_4096": "Llama-2-7B q_proj layer",
    "down_proj_11008": "Llama-2-7B MLP down_proj layer",
    "down_proj_28672": "Llama-3-70B-shaped MLP down_proj layer",
}
X_KINDS = {"normal": "N(0,1)", "t": "Student-t({nu:g})", "swiglu": "SiLU(z1)*z2"}


def workload_config(spec):
    xk = X_KINDS.get(spec.x_kind, spec.x_kind).format(nu=spec.nu)
    outl = f"{spec.outlier_count()} channels x{spec.outlier_scale:g}"
    noise = (f"Xhat = X + N(0, {spec.noise_abs:g}^2)" if spec.noise_abs > 0
             else f"Xhat = X + {100 * spec.noise_rel:g}% channel noise")
    x_bytes = spec.n_tok * spec.d_in * 2
    return {
        "workload": (f"{spec.name}: {WORKLOAD_TITLES.get(spec.name, 'linear layer')} "
                     f"{spec.d_out}x{spec.d_in}, {spec.n_tok} calibration tokens (bf16 {xk}, "
                     f"{outl}, {noise}), QEP alpha {spec.alpha}, GPTQ {spec.wbits}-bit "
                     f"g{spec.groupsize} asymmetric, damp {spec.damp}, "
                     f"act_order {'on' if spec.act_order else 'off'}"),
        "d_out": spec.d_out, "d_in": spec.d_in, "n_tok": spec.n_tok, "wbits": spec.wbits,
        "groupsize": spec.groupsize, "act_order": spec.act_order,
        "l2": (f"inputs larger than L2 (X and Xhat are {x_bytes / 1e9:.2f} GB each), no flush needed"
               if x_bytes > L2_BYTES else "inputs fit in L2: L2 flushed between steps"),
    }


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs.

    NVML is polled every 10 ms from a thread (the same counters nvidia-smi
    prints, often enough to see a region of a few hundred milliseconds);
    without NVML, nvidia-smi is sampled every 200 ms instead.
    """

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index, pci_bus_id=None, period_s=0.01):
        self.gpu_index = gpu_index
        self.pci_bus_id = pci_bus_id
        self.period_s = period_s
        self.proc = None
        self.thread = None
        self.samples = []  # (sm_mhz, sm_max_mhz, set of reasons)
        self.source = None

    def _nvml_start(self):
        import threading

        import pynvml as nv
        nv.nvmlInit()
        h = None
        if self.pci_bus_id:
            try:
                h = nv.nvmlDeviceGetHandleByPciBusId(self.pci_bus_id)
            except nv.NVMLError:
                h = None
        if h is None:
            h = nv.nvmlDeviceGetHandleByIndex(self.gpu_index)
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        bits = {}
        for nm, attr in zip(self.NAMES, ("HwSlowdown", "HwThermalSlowdown", "SwThermalSlowdown",
                                         "SwPowerCap")):
            bits[nm] = getattr(nv, "nvmlClocksEventReason" + attr,
                               getattr(nv, "nvmlClocksThrottleReason" + attr, 0))
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    r = get_reasons(h) if get_reasons else 0
                    self.samples.append((float(sm), float(smax),
                                         {nm for nm, b in bits.items() if b and (r & b)}))
                except nv.NVMLError:
                    pass
                self._stop.wait(self.period_s)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()
        self.source = f"NVML every {self.period_s * 1e3:.0f} ms"

    def __enter__(self):
        try:
            self._nvml_start()
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi every 200 ms"
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            for ln in out.splitlines():
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 7:
                    continue
                try:
                    sm, smax = float(parts[0]), float(parts[1])
                except ValueError:
                    continue
                self.samples.append((sm, smax, {nm for nm, v in zip(self.NAMES, parts[3:7])
                                                if v.lower().startswith("active")}))
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "source": self.source}
        reasons = set()
        for _, _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples), "reasons": sorted(reasons),
                "samples": len(self.samples), "source": self.source}


def gpu_index_for(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


# ----------------------------------------------------------------------------- algorithmic work

def phase_work(spec, factorisations=1):
    """Algorithmic work of each phase of one layer: (amount, unit, bound)."""
    n, m, N = spec.d_in, spec.d_out, spec.n_tok
    G = spec.d_in if spec.groupsize == -1 else spec.groupsize
    trailing = sum(2 * m * min(128, n - j1) * (n - j1 - min(128, n - j1)) for j1 in range(0, n, 128))
    return {
        # symmetric half of X^T X: n(n+1)/2 entries x 2N flops
        "hessian_syrk": (n * (n + 1) * N, "flop", "tensor"),
        "qep_cross": (2 * n * n * N, "flop", "tensor"),
        "qep_w_delta": (2 * m * n * n, "flop", "f32"),
        # per factorisation one Cholesky (n^3/3) + one triangular inverse (n^3/3)
        "factor": (factorisations * (2 * n ** 3 // 3), "flop", "f32"),
        "qep_apply": (2 * m * n * n, "flop", "f32"),
        "gptq_trailing": (trailing, "flop", "f32"),
        # read W (fp32) once, write codes (u8) and block errors (fp32)
        "gptq_sweep": (m * n * 4 + m * n + m * n * 4, "byte", "hbm"),
        "gptq_prep": (2 * m * n * 4, "byte", "hbm"),
        "gptq_pack": (m * n + m * n * spec.wbits // 8 + m * (n // G) * 8, "byte", "hbm"),
        # clear H (4n^2 written), mirror the upper triangle (2n^2 read + 2n^2 written)
        "hessian_fixup": (8 * n * n, "byte", "hbm"),
        # W (fp32), X and Xhat (bf16) read and written once each
        "hadamard_rotate": (2 * (4 * m * n + 2 * 2 * N * n), "byte", "hbm"),
    }


def cross_slices(spec):
    """Token slices the library runs the QEP cross product in (one launch of
    the product each): 8192 tokens or more per slice, at most 32."""
    return max(1, min(32, spec.n_tok // 8192))


def gemm_bytes(spec):
    """Algorithmic DRAM bytes of the two bf16-input phases of one layer: X and
    Xhat read once (bf16), H and d written once (fp32)."""
    n, N = spec.d_in, spec.n_tok
    return 2 * 2 * N * n + 2 * 4 * n * n


def recorded_traffic(workload):
    """(bytes per launch, description) of the dominant kernel on `workload`,
    or (None, reason) when there is no record or the kernel changed since."""
    import hashlib
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
        with open(KERNEL_SOURCE, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None, "no traffic record"
    if rec.get("workload") != workload:
        return None, f"traffic recorded for {rec.get('workload')}, not {workload}"
    if rec.get("kernel_source_sha256") != sha:
        return None, "kernel source changed since the traffic was captured"
    return int(rec["bytes_per_launch_full_size"]), rec.get("how", "")


# ----------------------------------------------------------------------------- oracle timing

def time_oracle_layer(spec, n_sample=CPU_SAMPLE_TOKENS, m_sample=CPU_SAMPLE_ROWS):
    """Time the float64 oracle on a bounded sample of one layer.

    The oracle's public pieces are timed separately and each is scaled by the
    part of the workload it is proportional to: the Hessian and the QEP cross
    product run on ``n_sample`` tokens (scaled to the workload's tokens); the
    QEP solve/apply and the GPTQ sweep run on ``m_sample`` rows of W (scaled
    to d_out); the factorisations run in full.  Returns (seconds per layer,
    seconds actually measured).
    """
    import numpy as np

    import oracle
    from synthetic import make_layer_host

    L = make_layer_host(spec, n_tok=n_sample)
    W = L["W"].astype(np.float64)
    Ws = W[:m_sample]
    tok_scale = spec.n_tok / n_sample
    row_scale = spec.d_out / m_sample
    clock = time.perf_counter
    t0 = clock()
    H = oracle.hessian(L["Xhat"])
    t_h = clock() - t0
    t0 = clock()
    oracle.qep_cross(L["X"], L["Xhat"])
    t_x = clock() - t0
    t0 = clock()
    oracle.qep_correct(W[:0], L["X"], L["Xhat"], spec.alpha, spec.damp, H=H)
    t_q0 = clock() - t0  # cross product + factorisation, no rows
    t0 = clock()
    Wps = oracle.qep_correct(Ws, L["X"], L["Xhat"], spec.alpha, spec.damp, H=H)
    t_qm = clock() - t0
    t0 = clock()
    prep = oracle.gptq_prepare(Wps, H, spec.damp, spec.act_order)
    U = oracle.inv_chol_upper(prep["Hd"])
    t_f = clock() - t0
    t0 = clock()
    oracle.gptq_sweep(prep["W"], U, spec.wbits, spec.groupsize, prep["perm"])
    t_s = clock() - t0
    total = ((t_h + t_x) * tok_scale + (t_q0 - t_x) + max(0.0, t_qm - t_q0) * row_scale
             + t_f + t_s * row_scale)
    measured = t_h + t_x + t_q0 + t_qm + t_f + t_s
    return total, measured


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        th = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if th:
            return max(th)
    except Exception:
        pass
    return os.cpu_count()


def cpu_sample_text(spec, n_sample=CPU_SAMPLE_TOKENS, m_sample=CPU_SAMPLE_ROWS):
    return (f"{n_sample} of {spec.n_tok} calibration tokens for the Hessian and QEP cross product "
            f"(scaled x{spec.n_tok / n_sample:g}); {m_sample} of {spec.d_out} rows for the QEP "
            f"apply and the GPTQ sweep (scaled x{spec.d_out / m_sample:g}); both factorisations of "
            f"the {spec.d_in}x{spec.d_in} Hessian in full; inputs from the host recipe of the workload")


# ----------------------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import torch

    import post_weight_quantization_07_b200 as oc
    from synthetic import CONFIGS, make_layer_device

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    spec = CONFIGS[args.workload]
    if args.n_tok:
        spec = spec.with_(n_tok=args.n_tok)
    spec_r = spec.with_(seed=spec.seed + 1000 * rank)
    L = make_layer_device(spec_r, "cuda")
    W, X, Xh = L["W"], L["X"], L["Xhat"]
    m, n = spec.d_out, spec.d_in
    G = n if spec.groupsize == -1 else spec.groupsize
    H = torch.zeros(n, n, device="cuda")
    Wp = torch.empty_like(W)
    codes = torch.empty(m, n * spec.wbits // 32, dtype=torch.int32, device="cuda")
    scales = torch.empty(m, n // G, device="cuda")
    zeros = torch.empty(m, n // G, device="cuda")
    stream = torch.cuda.current_stream()
    oc.oc_set_sync(False)

    if args.rotate:
        # rotation preprocessing: W, X and Xhat rotated by the same block
        # Hadamard matrix every step, then the layer quantised in that basis
        Wr, Xr, Xhr = torch.empty_like(W), torch.empty_like(X), torch.empty_like(Xh)

    def step():
        if args.rotate:
            oc.oc_hadamard_rotate(W, args.rotate, out=Wr, stream=stream)
            oc.oc_hadamard_rotate(X, args.rotate, out=Xr, stream=stream)
            oc.oc_hadamard_rotate(Xh, args.rotate, out=Xhr, stream=stream)
            w_in, x_in, xh_in = Wr, Xr, Xhr
        else:
            w_in, x_in, xh_in = W, X, Xh
        oc.oc_quantize_layer(w_in, x_in, xh_in, spec.alpha, spec.damp, spec.wbits, spec.groupsize,
                             spec.act_order, H=H, W_out=Wp, codes=codes, scales=scales,
                             zeros=zeros, stream=stream)

    def step_three_calls():
        H.zero_()
        oc.oc_hessian_accumulate(Xh, H, stream=stream)
        oc.oc_qep_correct(W, X, Xh, spec.alpha, spec.damp, H_opt=H, W_out=Wp, stream=stream)
        oc.oc_gptq_quantize(Wp, H, spec.wbits, spec.groupsize, spec.damp, spec.act_order,
                            codes=codes, scales=scales, zeros=zeros, stream=stream)

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x):
        if dist is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    for _ in range(args.warmup):
        step()
    st = oc.oc_stream_status(stream)
    if st != oc.OC_OK:
        raise RuntimeError(f"warm-up failed: {oc.oc_status_string(st)}")

    # ---- device-timed region: inputs resident in HBM
    oc.oc_profile_read()
    oc.oc_profile_enable(True)
    launches0 = oc.oc_launch_count()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(local_rank)
    bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    # Inputs smaller than L2 would be re-read from cache: then every step is
    # timed alone, after a write of a buffer larger than L2 outside its events.
    fits_l2 = X.numel() * X.element_size() <= L2_BYTES
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda") if fits_l2 else None
    step_ms = 0.0
    with ClockSampler(gpu_index_for(local_rank), bus) as clk:
        if fits_l2:
            for _ in range(args.steps):
                flush.fill_(1.0)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                step()
                b.record(stream)
                b.synchronize()
                step_ms += a.elapsed_time(b)
        else:
            e0.record(stream)
            for _ in range(args.steps):
                step()
            e1.record(stream)
        barrier()
    launches = oc.oc_launch_count() - launches0
    oc.oc_profile_enable(False)
    phases = oc.oc_profile_read()
    st = oc.oc_stream_status(stream)
    if st != oc.OC_OK:
        raise RuntimeError(f"timed steps failed: {oc.oc_status_string(st)}")
    ms_total = max_over_ranks(step_ms if fits_l2 else e0.elapsed_time(e1))
    ms_per_step = ms_total / args.steps
    value = world * args.steps / (ms_total / 1e3)

    # ---- the same layer through the three separate calls (two factorisations)
    step_three_calls()
    barrier()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(args.steps):
        step_three_calls()
    g1.record(stream)
    barrier()
    # A failure in this or the later side measurements is reported in the line
    # (with no figure for that measurement); only the timed steps' own failure
    # stops the run.  Every rank still takes the same collective steps.
    st = oc.oc_stream_status(stream)
    three_err = None if st == oc.OC_OK else f"three-call steps failed: {oc.oc_status_string(st)}"
    ms_three = max_over_ranks(g0.elapsed_time(g1)) / args.steps

    # ---- end to end: pinned host inputs copied in and results read back every step
    e2e = None
    if not args.no_e2e:
        Xh_h = torch.empty(Xh.shape, dtype=Xh.dtype, pin_memory=True)
        X_h = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
        W_h = torch.empty(W.shape, dtype=W.dtype, pin_memory=True)
        Xh_h.copy_(Xh)
        X_h.copy_(X)
        W_h.copy_(W)
        codes_h = torch.empty(codes.shape, dtype=codes.dtype, pin_memory=True)
        scales_h = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
        zeros_h = torch.empty(zeros.shape, dtype=zeros.dtype, pin_memory=True)

        def e2e_step():
            Xh.copy_(Xh_h, non_blocking=True)
            X.copy_(X_h, non_blocking=True)
            W.copy_(W_h, non_blocking=True)
            step()
            codes_h.copy_(codes, non_blocking=True)
            scales_h.copy_(scales, non_blocking=True)
            zeros_h.copy_(zeros, non_blocking=True)

        e2e_step()
        barrier()
        k2 = max(1, min(args.steps, 5))
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(k2):
            e2e_step()
        f1.record(stream)
        barrier()
        st = oc.oc_stream_status(stream)
        ms_e2e = max_over_ranks(f0.elapsed_time(f1))
        h2d = Xh.numel() * Xh.element_size() + X.numel() * X.element_size() + W.numel() * 4
        d2h = codes.numel() * 4 + scales.numel() * 4 + zeros.numel() * 4
        e2e = {"value": world * k2 / (ms_e2e / 1e3), "unit": UNIT, "steps": k2,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}
        if st != oc.OC_OK:
            e2e["value"] = None
            e2e["error"] = f"end-to-end steps failed: {oc.oc_status_string(st)}"

    # ---- the 224 layers of a 7B-shaped model, each on its own inputs
    model = None
    if not args.no_model_pass:
        model = model_pass(args, rank, world, stream, barrier, max_over_ranks)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    clocks = clk.summary()
    work = phase_work(spec)
    phase_out = {}
    for name, (ms, nl) in phases.items():
        if nl == 0 and ms == 0.0:
            continue
        amt, unit, bound = work.get(name, (0, "", ""))
        ms_step = ms / args.steps
        entry = {"ms_per_step": round(ms_step, 4), "launches_per_step": nl / args.steps}
        if amt and ms_step > 0:
            if unit == "flop":
                entry["achieved_tflops"] = round(amt / (ms_step / 1e3) / 1e12, 2)
            else:
                entry["achieved_gbs"] = round(amt / (ms_step / 1e3) / 1e9, 1)
            entry["bound"] = bound
        phase_out[name] = entry

    # Dominant kernel: the persistent tcgen05 product atb16_kernel, launched
    # once for the Hessian (bf16) and once per token slice of the QEP cross
    # product (fp16 operands; B200's dense fp16 and bf16 rates are the same).
    # Its phases hold those launches plus a few small ones (the first slice's
    # operand pass, column scales, two no-op fallback launches), so
    # achieved = the phases' algorithmic flops over the phases' CUDA-event
    # time, a lower bound on the kernel's own rate.  Peak: the measured bf16
    # burst figure (the timed region is a fraction of a second); the
    # sustained one is given beside it.
    gemm_phases = [p for p in ("hessian_syrk", "qep_cross") if p in phase_out]
    gemm_ms = sum(phase_out[p]["ms_per_step"] for p in gemm_phases)
    gemm_flop = sum(work[p][0] for p in gemm_phases)
    n_launch = 1 + (cross_slices(spec) if "qep_cross" in gemm_phases else 0)
    per_launch = gemm_flop / n_launch
    ms_launch = gemm_ms / n_launch
    peak_b = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_s = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    achieved = gemm_flop / (gemm_ms / 1e3) / 1e12
    traffic, traffic_how = recorded_traffic(spec.name) if not args.n_tok else (None, "reduced token count")
    sm_mhz = clocks.get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
    roof = {"bound": "tensor", "unit": "TFLOP/s", "kernel": "atb16_kernel", "phases": gemm_phases,
            "achieved": round(achieved, 2), "peak": round(peak_b, 2),
            "peak_source": f"bf16_tflops (burst) of {peak_src}", "frac": round(achieved / peak_b, 4),
            "frac_of_sustained_peak": round(achieved / peak_s, 4), "sm_mhz_median": sm_mhz,
            "traffic": traffic, "traffic_source": traffic_how,
            "per_launch": {"launches": n_launch, "flop": per_launch, "ms": round(ms_launch, 4),
                           "algorithmic_bytes": gemm_bytes(spec) / n_launch}}

    # Whole-layer roofline: every phase at the peak of the unit it needs,
    # taken in sequence: the bf16 products at the measured bf16 burst peak, the
    # fp32-accurate products (3xTF32 on the tensor cores) at tf32's dense
    # peak, taken as half the measured bf16 figure (the B200's nominal ratio,
    # 1.1 vs 2.25 PFLOP/s), counting each product once, and the memory-bound
    # phases at the measured copy bandwidth.
    peak_tf32 = peak_b / 2.0
    t_roof = 0.0
    for name, (amt, unit, bound) in work.items():
        if name == "hadamard_rotate" and not args.rotate:
            continue
        if bound == "tensor":
            t_roof += amt / (peak_b * 1e12)
        elif bound == "f32":
            t_roof += amt / (peak_tf32 * 1e12)
        else:
            t_roof += amt / (peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]) * 1e9)
    layer_roof = {"t_roof_ms": round(t_roof * 1e3, 3), "t_measured_ms": round(ms_per_step, 3),
                  "frac": round(t_roof * 1e3 / ms_per_step, 4),
                  "peaks": {"bf16_tflops": peak_b, "tf32_tflops": peak_tf32, "tf32_from": "half the measured bf16 burst",
                            "hbm_gbs": peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), "source": peak_src}}
    for name, entry in phase_out.items():
        amt, unit, bound = work.get(name, (0, "", ""))
        if "achieved_tflops" in entry:
            pk = peak_b if bound == "tensor" else peak_tf32
            entry["frac_of_peak"] = round(entry["achieved_tflops"] / pk, 4)
            if bound == "f32":
                entry["tensor_issue_frac"] = round(3 * entry["achieved_tflops"] / pk, 4)
        elif "achieved_gbs" in entry:
            entry["frac_of_peak"] = round(entry["achieved_gbs"] / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), 4)

    line = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16+f32",
        "data": "synthetic",
        "config": dict(workload_config(spec),
                       parallelism=(f"{world} independent layers, one per rank" if world > 1
                                    else "single GPU")),
        "seconds_per_7b_model": model.get("seconds") if model else None,
        "model_pass": model,
        "seconds_per_224_layers_of_this_shape": round(224 * ms_per_step / 1e3, 3),
        "three_calls_ms_per_step": round(ms_three, 3) if three_err is None else None,
        "roofline": roof, "layer_roofline": layer_roof, "phases": phase_out, "gpu_launches": int(launches),
        "clocks": clocks, "e2e": e2e,
    }
    if three_err is not None:
        line["three_calls_error"] = three_err
    if args.rotate:
        line["config"]["rotation"] = (f"block-{args.rotate} Hadamard rotation of W, X and Xhat in every step "
                                      f"(oc_hadamard_rotate), the layer quantised in the rotated basis")
    if world == 1 and not args.no_cpu_baseline:
        t_layer, t_meas = time_oracle_layer(spec)
        line["cpu_baseline"] = {"value": round(1.0 / t_layer, 6), "unit": UNIT,
                                "cores": blas_threads(), "kind": "oracle",
                                "sample": cpu_sample_text(spec),
                                "cpu_seconds_measured": round(t_meas, 2)}
    print(json.dumps(line), flush=True)


def model_pass(args, rank, world, stream, barrier, max_over_ranks):
    """All 224 linear layers of a 32-block Llama-2-7B-shaped model, each with its
    own seeded synthetic calibration inputs (131072 tokens, Student-t(4) with 1%
    of channels x20, Xhat = X + 2% channel noise) and weight (bf16 N(0, 0.02^2)),
    attention layers at 4 bits and MLP layers at 3 bits, g128, QEP alpha 0.5,
    damp 0.01, act_order off: one oc_quantize_layer call per layer.  Inputs are
    drawn on the device before each layer, outside its CUDA events; the
    reported seconds are the sum of the layers' device times (max over ranks;
    rank r takes layers r, r + N, ...)."""
    import torch

    import post_weight_quantization_07_b200 as oc
    from synthetic import llama7b_layers, make_layer_device

    specs = llama7b_layers(args.model_tokens)
    total_ms = 0.0
    done = 0
    launches0 = oc.oc_launch_count()
    t_wall = time.perf_counter()
    for i, spec in enumerate(specs):
        if i % world != rank:
            continue
        L = make_layer_device(spec, "cuda")
        m, n, G = spec.d_out, spec.d_in, spec.groupsize
        outs = dict(H=torch.empty(n, n, device="cuda"), W_out=torch.empty_like(L["W"]),
                    codes=torch.empty(m, n * spec.wbits // 32, dtype=torch.int32, device="cuda"),
                    scales=torch.empty(m, n // G, device="cuda"), zeros=torch.empty(m, n // G, device="cuda"))
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        oc.oc_quantize_layer(L["W"], L["X"], L["Xhat"], spec.alpha, spec.damp, spec.wbits, spec.groupsize,
                             spec.act_order, stream=stream, **outs)
        b.record(stream)
        b.synchronize()
        total_ms += a.elapsed_time(b)
        done += 1
        del L, outs
    st = oc.oc_stream_status(stream)
    barrier()
    ms = max_over_ranks(total_ms)
    if st != oc.OC_OK:
        return {"seconds": None, "error": f"model pass failed: {oc.oc_status_string(st)}", "layers": len(specs)}
    return {"seconds": round(ms / 1e3, 3), "layers": len(specs), "layers_per_rank": done,
            "layers_per_s": round(len(specs) / (ms / 1e3), 3), "calibration_tokens": args.model_tokens,
            "gpu_launches": int(oc.oc_launch_count() - launches0),
            "wall_s_including_input_generation": round(time.perf_counter() - t_wall, 1),
            "what": ("224 layers (32 blocks x q/k/v/o 4096x4096 4-bit, gate/up 4096->11008 and down "
                     "11008->4096 3-bit, g128), each on its own seeded inputs, one oc_quantize_layer call "
                     "per layer; sum of the layers' device times, input generation excluded")}


# ----------------------------------------------------------------------------- one layer over N GPUs

def run_shard_layer(args, rank, world, local_rank):
    """One layer split over the ranks: rank r takes token shard r (its share of
    H and the cross term, all-reduced over NCCL) and row shard r of W (QEP and
    GPTQ of those rows).  The whole job quantises one layer per step, so the
    value is layers/s of the job (strong scaling)."""
    import torch

    import post_weight_quantization_07_b200 as oc
    from post_weight_quantization_07_b200.sharded import quantize_layer_sharded, shard_range
    from synthetic import CONFIGS, make_layer_device

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    spec = CONFIGS[args.workload]
    if args.n_tok:
        spec = spec.with_(n_tok=args.n_tok)
    L = make_layer_device(spec, "cuda")  # the same layer on every rank
    t0, t1 = shard_range(spec.n_tok, rank, world, align=64)
    r0, r1 = shard_range(spec.d_out, rank, world)
    X, Xh = L["X"][t0:t1].contiguous(), L["Xhat"][t0:t1].contiguous()
    W = L["W"][r0:r1].contiguous()
    del L
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream()
    oc.oc_set_sync(False)
    reduce = (lambda t: dist.all_reduce(t)) if dist is not None else (lambda t: None)

    def step():
        quantize_layer_sharded(W, X, Xh, spec.alpha, spec.damp, spec.wbits, spec.groupsize, spec.act_order,
                               all_reduce=reduce)

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    st = oc.oc_stream_status(stream)
    if st != oc.OC_OK:
        raise RuntimeError(f"sharded steps failed: {oc.oc_status_string(st)}")
    ms = e0.elapsed_time(e1)
    if dist is not None:
        t = torch.tensor([ms], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(args.steps / (ms / 1e3), 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16+f32",
        "data": "synthetic",
        "config": dict(workload_config(spec),
                       parallelism=f"one layer over {world} rank(s): tokens and rows sharded, "
                                   f"H and the cross term all-reduced"),
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- one 7B block

BLOCK_GROUPS = ((0, 1, 2), (3,), (4, 5), (6,))  # q/k/v, o, gate/up, down of llama7b_layers()


def run_block(args, rank, world, local_rank):
    """One Llama-2-7B-shaped transformer block: q/k/v quantised as one group on
    their shared input, o alone, gate/up as one group, down alone (7 layers,
    4 calls).  Each group's X, Xhat follow its first layer's recipe; every
    layer has its own seeded W ~ N(0, 0.02^2) rounded to bf16."""
    import torch

    import post_weight_quantization_07_b200 as oc
    from synthetic import llama7b_layers, make_layer_device

    torch.cuda.set_device(local_rank)
    n_tok = args.n_tok or 131072
    specs = llama7b_layers(n_tok)[:7]
    groups = []
    for g in BLOCK_GROUPS:
        lead = specs[g[0]]
        L = make_layer_device(lead.with_(seed=lead.seed + 1000 * rank), "cuda")
        Ws = []
        for j in g:
            gen = torch.Generator(device="cuda").manual_seed(specs[j].seed + 1000 * rank)
            w = torch.randn(specs[j].d_out, specs[j].d_in, generator=gen, device="cuda") * specs[j].w_std
            Ws.append(w.to(torch.bfloat16).float().contiguous())
        groups.append((lead, Ws, L["X"], L["Xhat"]))
        del L
    stream = torch.cuda.current_stream()
    oc.oc_set_sync(False)
    outs = []
    for lead, Ws, X, Xh in groups:
        n = lead.d_in
        G = lead.groupsize
        outs.append(dict(H=torch.empty(n, n, device="cuda"), W_outs=[torch.empty_like(w) for w in Ws],
                         codes=[torch.empty(w.shape[0], n * lead.wbits // 32, dtype=torch.int32, device="cuda")
                                for w in Ws],
                         scales=[torch.empty(w.shape[0], n // G, device="cuda") for w in Ws],
                         zeros=[torch.empty(w.shape[0], n // G, device="cuda") for w in Ws]))

    def step():
        for (lead, Ws, X, Xh), o in zip(groups, outs):
            oc.oc_quantize_layer_group(Ws, X, Xh, lead.alpha, lead.damp, lead.wbits, lead.groupsize,
                                       lead.act_order, stream=stream, **o)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    launches0 = oc.oc_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(local_rank)
    bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    with ClockSampler(gpu_index_for(local_rank), bus) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    st = oc.oc_stream_status(stream)
    if st != oc.OC_OK:
        raise RuntimeError(f"block steps failed: {oc.oc_status_string(st)}")
    ms_block = e0.elapsed_time(e1) / args.steps
    layers = sum(len(g) for g in BLOCK_GROUPS)
    line = {
        "metric": METRIC, "value": round(layers / (ms_block / 1e3), 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_block, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16+f32",
        "data": "synthetic",
        "config": {"workload": (f"block_7b: one Llama-2-7B-shaped block (q/k/v/o 4096x4096 4-bit, gate/up "
                                f"4096->11008 and down 11008->4096 3-bit, g128, QEP alpha 0.5, damp 0.01), "
                                f"{n_tok} calibration tokens per input, q/k/v and gate/up sharing their "
                                f"inputs (one Hessian, cross term and factorisation per group)"),
                   "layers_per_step": layers, "calls_per_step": len(BLOCK_GROUPS),
                   "l2": "inputs larger than L2, no flush needed"},
        "seconds_per_32_block_model": round(32 * ms_block / 1e3, 3),
        "gpu_launches": int(oc.oc_launch_count() - launches0), "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_lpcd(args, rank, world, local_rank):
    """LPCD of one Llama-2-7B-shaped V/O pair treated as the linear submodule
    y = x W_v^T W_o^T (4096x4096 each, 4-bit g128, QEP alpha 0.5 start, damp
    0.01): the layer-wise start plus --lpcd-rounds rounds of the projected
    coordinate steps, all inside the timed step.  X, Xhat follow v_proj's
    recipe; W_v, W_o are seeded N(0, 0.02^2) rounded to bf16.  The submodule's
    output error before and after the rounds comes from one more, untimed run."""
    import torch

    import post_weight_quantization_07_b200 as oc
    from synthetic import llama7b_layers, make_layer_device

    torch.cuda.set_device(local_rank)
    n_tok = args.n_tok or 131072
    specs = llama7b_layers(n_tok)
    sv, so = specs[2], specs[3]
    L = make_layer_device(sv.with_(seed=sv.seed + 1000 * rank), "cuda")
    gen = torch.Generator(device="cuda").manual_seed(so.seed + 1000 * rank)
    Wo = (torch.randn(so.d_out, so.d_in, generator=gen, device="cuda") * so.w_std).to(torch.bfloat16).float()
    Wv, X, Xh = L["W"], L["X"], L["Xhat"]
    R = args.lpcd_rounds
    stream = torch.cuda.current_stream()
    oc.oc_set_sync(False)

    def step(track=False):
        return oc.lpcd_pair(Wv, Wo, X, Xh, sv.alpha, sv.damp, sv.wbits, sv.groupsize, sv.act_order, rounds=R,
                            stream=stream, track_error=track)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    launches0 = oc.oc_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(local_rank)
    bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    with ClockSampler(gpu_index_for(local_rank), bus) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    launches = oc.oc_launch_count() - launches0
    st = oc.oc_stream_status(stream)
    if st != oc.OC_OK:
        raise RuntimeError(f"LPCD steps failed: {oc.oc_status_string(st)}")
    ms = e0.elapsed_time(e1) / args.steps
    r = step(track=True)
    rel = [e / r["ref"] for e in r["errors"]]
    line = {
        "metric": "LPCD two-layer submodules quantized/sec (Llama-7B V/O shapes, 4-bit g128)",
        "value": round(world / (ms / 1e3), 4), "unit": "submodules/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16+f32",
        "data": "synthetic",
        "config": {"workload": (f"lpcd_vo: Llama-2-7B v_proj and o_proj (4096x4096 each) as the linear "
                                f"submodule y = x W_v^T W_o^T, {n_tok} calibration tokens (v_proj recipe), "
                                f"4-bit g128, QEP alpha 0.5 start, damp 0.01, {R} LPCD round(s)"),
                   "rounds": R, "l2": "inputs larger than L2, no flush needed"},
        "submodule_rel_error": {"layer_wise_start": round(rel[0], 6),
                                "after_rounds": [round(x, 6) for x in rel[1:]]},
        "gpu_launches": int(launches), "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_gemv(args, rank, world, local_rank):
    """The quantised layers of one Llama-2-7B-shaped block applied at decode
    time straight from packed codes (oc_dequant_gemv): q/k/v/o 4096x4096 at
    4 bits, gate/up 4096->11008 and down 11008->4096 at 3 bits, g128, batch
    --gemv-batch tokens.  Codes, scales and zeros are seeded random values of
    the quantiser's layout (the GEMV's cost does not depend on them).  The
    95 MB of codes and grids fit in L2, so every step is timed alone after a
    write of a buffer larger than L2."""
    import torch

    import post_weight_quantization_07_b200 as oc

    torch.cuda.set_device(local_rank)
    nb = args.gemv_batch
    shapes = [(4096, 4096, 4)] * 4 + [(11008, 4096, 3)] * 2 + [(4096, 11008, 3)]
    gen = torch.Generator(device="cuda").manual_seed(5150 + rank)
    layers = []
    nbytes = 0
    for m, n, b in shapes:
        codes = torch.randint(-2 ** 31, 2 ** 31 - 1, (m, n * b // 32), generator=gen, device="cuda",
                              dtype=torch.int32)
        scales = torch.rand(m, n // 128, generator=gen, device="cuda") * 0.01 + 1e-3
        zeros = torch.randint(0, 2 ** b, (m, n // 128), generator=gen, device="cuda").float()
        x = torch.randn(nb, n, generator=gen, device="cuda").to(torch.bfloat16)
        y = torch.empty(nb, m, device="cuda")
        layers.append((codes, scales, zeros, n, b, x, y))
        nbytes += codes.numel() * 4 + scales.numel() * 4 + zeros.numel() * 4 + x.numel() * 2 + y.numel() * 4
    oc.oc_set_sync(False)

    def step():
        # stream=None: the current stream, which is the capture stream below
        for codes, scales, zeros, n, b, x, y in layers:
            oc.oc_dequant_gemv(codes, scales, zeros, n, b, 128, x, y=y)

    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # A decode loop replays its launches as a CUDA graph; the eager calls'
    # host overhead (Python, ctypes, argument checks) exceeds these kernels.
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    stream = torch.cuda.current_stream()
    graph.replay()
    torch.cuda.synchronize()

    def timed(run):
        total = 0.0
        for _ in range(args.steps):
            flush.fill_(1.0)
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            run()
            e.record(stream)
            e.synchronize()
            total += a.elapsed_time(e)
        return total / args.steps

    props = torch.cuda.get_device_properties(local_rank)
    bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    with ClockSampler(gpu_index_for(local_rank), bus) as clk:
        ms = timed(graph.replay)
    launches = 7 * args.steps  # one kernel per layer per replay (the counter sees host calls only)
    ms_eager = timed(step)
    st = oc.oc_stream_status(stream)
    if st != oc.OC_OK:
        raise RuntimeError(f"GEMV steps failed: {oc.oc_status_string(st)}")
    del graph
    peaks, peak_src = load_peaks()
    peak = peaks.get("hbm_gbs")
    achieved = nbytes / (ms / 1e3) / 1e9
    line = {
        "metric": "dequantising GEMV over packed GPTQ codes: decode steps of one Llama-7B block per second",
        "value": round(world / (ms / 1e3), 2), "unit": "block-steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 (bf16 activations, packed int codes)", "data": "synthetic",
        "config": {"workload": (f"gemv_block: q/k/v/o 4096x4096 4-bit and gate/up/down 4096<->11008 3-bit, "
                                f"g128, {nb} token(s) per step"),
                   "batch": nb, "l2": "flushed before every step (a write of twice L2)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 3) if peak else None, "traffic": None,
                     "peak_source": f"{peak_src} copy bandwidth (of {peak_src})", "bytes_per_step": nbytes},
        "eager_ms_per_step": round(ms_eager, 4), "launch": "CUDA graph replay of the step's 7 calls",
        "gpu_launches": int(launches), "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return
    from synthetic import CONFIGS
    if args.workload not in CONFIGS:
        print(json.dumps({"impl": "reference", "unavailable": (
            f"the float64 oracle arm times single-layer workloads ({', '.join(sorted(CONFIGS))}); "
            f"{args.workload} has none")}), flush=True)
        return
    spec = CONFIGS[args.workload]
    if args.n_tok:
        spec = spec.with_(n_tok=args.n_tok)
    for _ in range(args.warmup):
        time_oracle_layer(spec, n_sample=512, m_sample=64)
    times = []
    measured = 0.0
    for _ in range(args.steps):
        t, tm = time_oracle_layer(spec)
        times.append(t)
        measured += tm
    t = statistics.median(times)
    value = 1.0 / t
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(spec), parallelism="host cores"),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": blas_threads(),
                         "kind": "oracle", "sample": cpu_sample_text(spec),
                         "cpu_seconds_measured": round(measured, 2)},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="q_proj_4096")
    ap.add_argument("--n-tok", type=int, default=None,
                    help="calibration tokens per layer (default: the workload's own)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-model-pass", action="store_true",
                    help="skip the 224-layer 7B-shaped model pass (seconds per model)")
    ap.add_argument("--model-tokens", type=int, default=131072,
                    help="calibration tokens per layer in the model pass")
    ap.add_argument("--rotate", type=int, default=0, metavar="B",
                    help="rotate W, X, Xhat by a block-B Hadamard matrix every step before quantising")
    ap.add_argument("--gemv-batch", type=int, default=1,
                    help="tokens per decode step (--workload gemv_block, 1..8)")
    ap.add_argument("--lpcd-rounds", type=int, default=1,
                    help="LPCD rounds after the layer-wise start (--workload lpcd_vo)")
    ap.add_argument("--shard-layer", action="store_true",
                    help="one layer split over the ranks (tokens and rows) instead of one layer per rank")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.workload == "block_7b":
        run_block(args, rank, world, local_rank)
    elif args.workload == "lpcd_vo":
        run_lpcd(args, rank, world, local_rank)
    elif args.workload == "gemv_block":
        run_gemv(args, rank, world, local_rank)
    elif args.shard_layer:
        run_shard_layer(args, rank, world, local_rank)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
